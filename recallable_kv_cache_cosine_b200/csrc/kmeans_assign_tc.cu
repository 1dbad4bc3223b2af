// Cosine K-means assignment on the 5th-generation tensor cores (sm_100a).
//
// The ClusterKV explainer ("大模型KV Cache压缩技术：ClusterKV的语义空间优化") computes the
// cosine distances of prefill clustering with a half-precision matmul (section 4.1):
//   assign[i] = argmax_c  k_i . mu_hat_c ,   mu_hat_c = bf16(mu_c / |mu_c|)
// (section 3.2; |k_i| does not depend on c, so this is the argmax of the cosine). Ties go
// to the lower c. The n x C score matrix is never written to memory.
//
// Design (one CTA per SM, persistent over the flattened (unit, 128-key tile) list):
//   warp 16     TMA producer: the unit's centroid block mu_hat (<= 512 rows, kept in shared
//               memory while the unit lasts, each 256-row slot sized to its rows), then the
//               128x128 bf16 key tiles through a ring of 3-6 stages (as many as shared
//               memory allows). All loads use the 128-byte swizzle; each CTA loads its own tiles.
//   warp 17     allocates 512 TMEM columns. One thread issues tcgen05.mma (M=128, N<=256,
//               K=16, bf16 x bf16 -> fp32) into two 256-column accumulator slots. With
//               C <= 256, consecutive tiles alternate slots (double buffering). With
//               256 < C <= 512, every tile uses both slots.
//   warps 0..15 epilogue: warp w reads TMEM lanes 32*(w%4).. (its rows) and column quarter
//               w/4 of each slot with tcgen05.ld, frees the slot, takes each 32-column
//               block's maximum with three-input max instructions, then the first column
//               holding the slot's maximum (one search per slot), and merges the four
//               quarters through shared memory. When asked, each
//               key's final cluster is also counted into its 1024-key chunk's histogram
//               (integer atomics), the counting sort's first pass.
// For C > 512 the host launches once per 512-centroid chunk. Each later launch merges into
// the running (best value, index) of the earlier ones, so ties still go to the lower c.
#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

constexpr int kTileM = 128;
constexpr int kSlotCols = 256;
constexpr int kEpiWarps = 16;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr uint32_t kATileBytes = kTileM * kD * 2;       // 32 KB
constexpr uint32_t kAHalfBytes = kTileM * 64 * 2;       // 16 KB (one 64-wide K half)
constexpr int kMaxStages = 6;

struct AssignParams {
    int32_t U;
    int32_t T;             // tiles per unit
    int64_t m;             // keys per unit
    int32_t row0;          // first key row inside each unit
    int32_t c_lo;          // first centroid of this launch
    int32_t nslots;        // 1 or 2
    int32_t valid0, valid1;  // centroids in slot 0 / 1
    int32_t n0, n1;          // MMA N of slot 0 / 1 (multiple of 16) = rows held per slot
    int32_t nst;             // key-tile stages
    int32_t merge;         // merge with the running best of earlier launches
    int32_t store_best;    // write the running best for later launches
    int32_t* assign;
    int64_t assign_ustride;
    float* best;
    int64_t best_ustride;
    int32_t* counts;       // [U][nch][C_all] chunk counts to add to (last launch only), or null
    int32_t nch;
    int32_t C_all;
    uint32_t* err;
};

struct __align__(8) Bars {
    uint64_t a_full[kMaxStages], a_empty[kMaxStages], b_full, b_empty, t_full[2], t_empty[2], done;
};

// Barrier over the 16 epilogue warps that also ORs a per-thread flag, so that every epilogue
// warp takes the same abort decision after it.
CKV_DEV bool epi_bar_any(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred q, a;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred a, 1, 512, q;\n"
        " selp.u32 %0, 1, 0, a;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)flag)
        : "memory");
    return r != 0;
}

CKV_DEV float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Maximum of 32 values with three-input max instructions (17 instructions, depth 4).
CKV_DEV float max32(const float* v) {
    float m[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) m[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    m[10] = fmaxf(v[30], v[31]);
    const float a = fmax3(m[0], m[1], m[2]), b = fmax3(m[3], m[4], m[5]);
    const float c = fmax3(m[6], m[7], m[8]), d = fmaxf(m[9], m[10]);
    return fmaxf(fmax3(a, b, c), d);
}

// Lowest j with v[j] == mx (0 if none, which only a NaN row could give).
CKV_DEV int first_index(const float* v, float mx) {
    uint32_t msk = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) msk |= (v[j] == mx ? 1u : 0u) << j;
    return msk ? __ffs((int)msk) - 1 : 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap map_a,
                     const __grid_constant__ CUtensorMap map_b0,
                     const __grid_constant__ CUtensorMap map_b1, const AssignParams p) {
    pdl_launch_dependents();  // let the next kernel in the stream be scheduled early
    pdl_wait();               // the previous kernel's writes are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // centroid slots: slot h holds n_h rows as two 64-column halves of n_h x 128 B each
    uint8_t* sB = smem;
    const uint32_t b0_bytes = (uint32_t)p.n0 * kD * 2;
    const uint32_t b1_bytes = p.nslots == 2 ? (uint32_t)p.n1 * kD * 2 : 0u;
    uint8_t* sA = sB + b0_bytes + b1_bytes;                   // nst x 32 KB
    float* xval = (float*)(sA + (size_t)p.nst * kATileBytes); // [2][3][128]
    int32_t* xidx = (int32_t*)(xval + 6 * kTileM);            // [2][3][128]
    Bars* bars = (Bars*)(xidx + 6 * kTileM);
    uint32_t* tmem_slot = (uint32_t*)(bars + 1);
    volatile int32_t* abort_flag = (volatile int32_t*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t total = (int64_t)p.U * p.T;
    const int64_t f0 = total * blockIdx.x / gridDim.x;
    const int64_t f1 = total * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.nst; ++s) {
            mbar_init(&bars->a_full[s], 1);
            mbar_init(&bars->a_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->t_full[s], 1);
            mbar_init(&bars->t_empty[s], kEpiWarps);
        }
        mbar_init(&bars->b_full, 1);
        mbar_init(&bars->b_empty, 1);
        mbar_init(&bars->done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kEpiWarps + 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == kEpiWarps) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&map_a);
            tma_prefetch_desc(&map_b0);
            if (p.nslots == 2) tma_prefetch_desc(&map_b1);
            int32_t cur_u = -1;
            uint32_t nb = 0;  // B loads issued
            int64_t i = 0;
            for (int64_t f = f0; f < f1; ++f, ++i) {
                if (*abort_flag) break;
                const int32_t u = (int32_t)(f / p.T);
                const int32_t t = (int32_t)(f % p.T);
                if (u != cur_u) {
                    if (nb > 0 && !mbar_wait(&bars->b_empty, (nb - 1) & 1, p.err)) {
                        *abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->b_full, b0_bytes + b1_bytes);
                    for (int kh = 0; kh < 2; ++kh)
                        tma_load_3d(sB + kh * (b0_bytes / 2), &map_b0, &bars->b_full, kh * 64,
                                    p.c_lo, u);
                    if (p.nslots == 2)
                        for (int kh = 0; kh < 2; ++kh)
                            tma_load_3d(sB + b0_bytes + kh * (b1_bytes / 2), &map_b1, &bars->b_full,
                                        kh * 64, p.c_lo + kSlotCols, u);
                    ++nb;
                    cur_u = u;
                }
                const int s = (int)(i % p.nst);
                if (!mbar_wait(&bars->a_empty[s], ((uint32_t)(i / p.nst) & 1u) ^ 1u, p.err)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(&bars->a_full[s], kATileBytes);
                for (int kh = 0; kh < 2; ++kh)
                    tma_load_3d(sA + s * kATileBytes + kh * kAHalfBytes, &map_a, &bars->a_full[s],
                                kh * 64, p.row0 + t * kTileM, u);
            }
            // Drain: every issued load must land before the CTA may exit.
            const int64_t issued = i;
            for (int64_t j = issued - p.nst < 0 ? 0 : issued - p.nst; j < issued; ++j)
                mbar_wait(&bars->a_full[j % p.nst], (uint32_t)(j / p.nst) & 1u, p.err);
            if (nb > 0) mbar_wait(&bars->b_full, (nb - 1) & 1, p.err);
        }
    } else if (warp == kEpiWarps + 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc0 = umma_idesc_bf16(kTileM, p.n0);
            const uint32_t idesc1 = umma_idesc_bf16(kTileM, p.n1 > 0 ? p.n1 : 16);
            uint32_t use[2] = {0, 0};
            int32_t cur_u = -1;
            uint32_t nb = 0;
            int64_t i = 0;
            for (int64_t f = f0; f < f1; ++f, ++i) {
                if (*abort_flag) break;
                const int32_t u = (int32_t)(f / p.T);
                if (u != cur_u) {
                    if (nb > 0) umma_commit(&bars->b_empty);
                    if (!mbar_wait(&bars->b_full, nb & 1, p.err)) { *abort_flag = 1; break; }
                    ++nb;
                    cur_u = u;
                }
                const int s = (int)(i % p.nst);
                if (!mbar_wait(&bars->a_full[s], (uint32_t)(i / p.nst) & 1u, p.err)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_u32(sA + s * kATileBytes);
                const int nuse = p.nslots == 1 ? 1 : 2;
                bool ok = true;
                for (int k = 0; k < nuse; ++k) {
                    const int h = p.nslots == 1 ? (int)(i & 1) : k;
                    const int hb = p.nslots == 1 ? 0 : h;  // which B slot holds the centroids
                    if (!mbar_wait(&bars->t_empty[h], (use[h] & 1u) ^ 1u, p.err)) { ok = false; break; }
                    ++use[h];
                    tc_fence_after();
                    const uint32_t b_base = smem_u32(sB + (hb == 0 ? 0u : b0_bytes));
                    const uint32_t b_half = (hb == 0 ? b0_bytes : b1_bytes) / 2;
                    const uint32_t d = tbase + (uint32_t)(h * kSlotCols);
                    const uint32_t idesc = hb == 0 ? idesc0 : idesc1;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t koff = (uint32_t)((kk & 3) * 32);
                        const uint64_t ad = sw128_kmajor_desc(a_base + (kk >> 2) * kAHalfBytes + koff);
                        const uint64_t bd = sw128_kmajor_desc(b_base + (kk >> 2) * b_half + koff);
                        umma_bf16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&bars->t_full[h]);
                }
                if (!ok) { *abort_flag = 1; break; }
                umma_commit(&bars->a_empty[s]);
            }
            // Every issued MMA must finish before the tensor memory is released.
            umma_commit(&bars->done);
            mbar_wait(&bars->done, 0, p.err);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // warp w: TMEM lane quadrant w % 4 (rows), column quarter w / 4 of each slot
        const int quad = warp & 3;
        const int qtr = warp >> 2;
        const int row = quad * 32 + lane;
        const uint32_t lane_addr = tbase + ((uint32_t)(quad * 32) << 16);
        uint32_t use[2] = {0, 0};
        int64_t i = 0;
        for (int64_t f = f0; f < f1; ++f, ++i) {
            const int32_t u = (int32_t)(f / p.T);
            const int32_t t = (int32_t)(f % p.T);
            float best = -INFINITY;
            int32_t bidx = 0;
            const int nuse = p.nslots == 1 ? 1 : 2;
            bool ok = true;
            for (int k = 0; k < nuse && ok; ++k) {
                const int h = p.nslots == 1 ? (int)(i & 1) : k;
                const int hb = p.nslots == 1 ? 0 : h;
                const int valid = hb == 0 ? p.valid0 : p.valid1;
                if (*abort_flag || !mbar_wait(&bars->t_full[h], use[h] & 1u, p.err)) {
                    ok = false;
                    break;
                }
                ++use[h];
                tc_fence_after();
                float v[2][32];
                const int col0 = qtr * 64;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
                    if (col0 + cc * 32 < valid)
                        tmem_ld32(lane_addr + (uint32_t)(h * kSlotCols + col0 + cc * 32), v[cc]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->t_empty[h]);
                const int cbase = p.c_lo + hb * kSlotCols + col0;
                // the maximum of each 32-column block, then one first-index search in the
                // first block that holds the slot's maximum (if it beats the running best)
                float mxb[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c0 = col0 + cc * 32;
                    if (c0 >= valid) continue;  // uniform across the warp
                    if (c0 + 32 > valid) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c0 + j >= valid) v[cc][j] = -INFINITY;
                    }
                    mxb[cc] = max32(v[cc]);
                }
                const float mx = fmaxf(mxb[0], mxb[1]);
                if (mx > best) {  // ascending column order: ties keep the lower index
                    const bool in1 = !(mxb[0] == mx);
                    float t[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) t[j] = in1 ? v[1][j] : v[0][j];
                    best = mx;
                    bidx = cbase + (in1 ? 32 : 0) + first_index(t, mx);
                }
            }
            const int buf = (int)(i & 1);
            if (qtr > 0) {
                xval[(buf * 3 + qtr - 1) * kTileM + row] = best;
                xidx[(buf * 3 + qtr - 1) * kTileM + row] = bidx;
            }
            if (epi_bar_any(!ok || *abort_flag)) {
                *abort_flag = 1;
                break;
            }
            if (qtr == 0) {
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const float ov = xval[(buf * 3 + q) * kTileM + row];
                    const int32_t oi = xidx[(buf * 3 + q) * kTileM + row];
                    if (ov > best || (ov == best && oi < bidx)) {
                        best = ov;
                        bidx = oi;
                    }
                }
                const int64_t r = (int64_t)t * kTileM + row;
                if (r < p.m) {
                    if (p.merge) {
                        const float pv = p.best[(int64_t)u * p.best_ustride + r];
                        if (!(best > pv)) {  // earlier launches hold lower indices
                            best = pv;
                            bidx = p.assign[(int64_t)u * p.assign_ustride + r];
                        }
                    }
                    p.assign[(int64_t)u * p.assign_ustride + r] = bidx;
                    if (p.store_best) p.best[(int64_t)u * p.best_ustride + r] = best;
                    else if (p.counts)
                        atomicAdd(p.counts + ((int64_t)u * p.nch + r / kChunk) * p.C_all + bidx, 1);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kEpiWarps + 1) tmem_dealloc(tbase, 512);
}

}  // namespace

struct AssignPlanImpl {
    CUtensorMap map_a;
    std::vector<CUtensorMap> map_b0, map_b1;
    std::vector<AssignParams> params;
    std::vector<size_t> smem;
    int grid = 0;
};

int prepare_kmeans_assign(const KeysView& k, const uint16_t* mu_hat, int64_t muhat_ustride,
                          int32_t C, int32_t* assign, int64_t assign_ustride, float* best,
                          int64_t best_ustride, uint32_t* err, AssignPlan* out, int32_t* counts) {
    auto impl = std::make_shared<AssignPlanImpl>();
    out->impl = impl;
    if (k.m <= 0 || k.U <= 0) return CKV_OK;
    int rc = encode_bf16_3d(&impl->map_a, k.base, kD, (uint64_t)k.n_rows, (uint64_t)k.U, kD * 2,
                            (uint64_t)k.n_rows * kD * 2, 64, kTileM);
    if (rc != CKV_OK) return rc;
    AssignParams p{};
    p.U = k.U;
    p.T = (int32_t)((k.m + kTileM - 1) / kTileM);
    p.m = k.m;
    p.row0 = (int32_t)k.row0;
    p.assign = assign;
    p.assign_ustride = assign_ustride;
    p.best = best;
    p.best_ustride = best_ustride;
    p.counts = counts;
    p.nch = (int32_t)n_chunks(k.m);
    p.C_all = C;
    p.err = err;
    const int nchunks = (C + 2 * kSlotCols - 1) / (2 * kSlotCols);
    const int sms = num_sms_of_current_device();
    const int64_t total = (int64_t)p.U * p.T;
    impl->grid = (int)(total < sms ? total : sms);
    constexpr size_t kSmemLimit = 232448;  // 227 KB opt-in per block
    for (int ch = 0; ch < nchunks; ++ch) {
        p.c_lo = ch * 2 * kSlotCols;
        const int cnt = C - p.c_lo < 2 * kSlotCols ? C - p.c_lo : 2 * kSlotCols;
        p.nslots = cnt > kSlotCols ? 2 : 1;
        p.valid0 = cnt < kSlotCols ? cnt : kSlotCols;
        p.valid1 = cnt - p.valid0;
        p.n0 = (p.valid0 + 15) / 16 * 16;
        p.n1 = (p.valid1 + 15) / 16 * 16;
        p.merge = ch > 0;
        p.store_best = ch + 1 < nchunks;
        // one tensor map per centroid slot, its box sized to the slot's rows
        CUtensorMap b0, b1;
        rc = encode_bf16_3d(&b0, mu_hat, kD, (uint64_t)C, (uint64_t)k.U, kD * 2,
                            (uint64_t)muhat_ustride * kD * 2, 64, (uint32_t)p.n0);
        if (rc != CKV_OK) return rc;
        rc = encode_bf16_3d(&b1, mu_hat, kD, (uint64_t)C, (uint64_t)k.U, kD * 2,
                            (uint64_t)muhat_ustride * kD * 2, 64,
                            (uint32_t)(p.nslots == 2 ? p.n1 : p.n0));
        if (rc != CKV_OK) return rc;
        const size_t fixed = 1024 + (size_t)(p.n0 + (p.nslots == 2 ? p.n1 : 0)) * kD * 2 +
                             12 * kTileM * 4 + sizeof(Bars) + 64;
        int nst = (int)((kSmemLimit - fixed) / kATileBytes);
        nst = nst > kMaxStages ? kMaxStages : nst;
        if (nst < 2) {
            set_error("assign: shared memory too small for two key stages");
            return CKV_EINVAL;
        }
        p.nst = nst;
        const size_t smem = fixed + (size_t)nst * kATileBytes;
        rc = ensure_smem((const void*)assign_tc_kernel, smem, "assign: set smem");
        if (rc != CKV_OK) return rc;
        impl->map_b0.push_back(b0);
        impl->map_b1.push_back(b1);
        impl->params.push_back(p);
        impl->smem.push_back(smem);
    }
    return CKV_OK;
}

int run_kmeans_assign(const AssignPlan& plan, cudaStream_t s) {
    const AssignPlanImpl* impl = plan.impl.get();
    if (!impl) return CKV_EINVAL;
    for (size_t ch = 0; ch < impl->params.size(); ++ch) {
        cudaError_t e = launch_pdl(assign_tc_kernel, dim3(impl->grid), dim3(kThreads), impl->smem[ch], s,
                                   impl->map_a, impl->map_b0[ch], impl->map_b1[ch], impl->params[ch]);
        if (e != cudaSuccess) return cuda_fail(e, "assign: launch");
    }
    return CKV_OK;
}

int launch_kmeans_assign(const KeysView& k, const uint16_t* mu_hat, int64_t muhat_ustride,
                         int32_t C, int32_t* assign, int64_t assign_ustride, float* best,
                         int64_t best_ustride, uint32_t* err, cudaStream_t s) {
    AssignPlan plan;
    const int rc = prepare_kmeans_assign(k, mu_hat, muhat_ustride, C, assign, assign_ustride, best,
                                         best_ustride, err, &plan);
    if (rc != CKV_OK) return rc;
    return run_kmeans_assign(plan, s);
}

}  // namespace ckv
