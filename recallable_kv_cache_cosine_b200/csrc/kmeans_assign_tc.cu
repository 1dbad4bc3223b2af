// Cosine K-means assignment on the 5th-generation tensor cores (sm_100a).
//
// The ClusterKV explainer ("大模型KV Cache压缩技术：ClusterKV的语义空间优化") computes the
// cosine distances of prefill clustering with a half-precision matmul (section 4.1):
//   assign[i] = argmax_c  k_i . mu_hat_c ,   mu_hat_c = bf16(mu_c / |mu_c|)
// (section 3.2; |k_i| does not depend on c, so this is the argmax of the cosine). Ties go
// to the lower c. The n x C score matrix is never written to memory.
//
// Design (one CTA per SM, persistent over the flattened (unit, 128-key tile) list):
//   warp 8      TMA producer: the unit's centroid block mu_hat (<= 512 rows, kept in shared
//               memory while the unit lasts), then the 128x128 bf16 key tiles through a
//               2-stage ring. All loads use the 128-byte swizzle and no multicast.
//   warp 9      allocates 512 TMEM columns. One thread issues tcgen05.mma (M=128, N<=256,
//               K=16, bf16 x bf16 -> fp32) into two 256-column accumulator slots. With
//               C <= 256, consecutive tiles alternate slots (double buffering). With
//               256 < C <= 512, every tile uses both slots.
//   warps 0..7  epilogue: warp w reads TMEM lanes 32*(w%4).. (its rows) and column half w/4
//               of each slot with tcgen05.ld, frees the slot, takes the running argmax, and
//               merges the two halves through shared memory.
// For C > 512 the host launches once per 512-centroid chunk. Each later launch merges into
// the running (best value, index) of the earlier ones, so ties still go to the lower c.
#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

constexpr int kTileM = 128;
constexpr int kSlotCols = 256;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr uint32_t kATileBytes = kTileM * kD * 2;       // 32 KB
constexpr uint32_t kAHalfBytes = kTileM * 64 * 2;       // 16 KB (one 64-wide K half)
constexpr uint32_t kBSlotBytes = kSlotCols * kD * 2;    // 64 KB
constexpr uint32_t kBHalfBytes = kSlotCols * 64 * 2;    // 32 KB

struct AssignParams {
    int32_t U;
    int32_t T;             // tiles per unit
    int64_t m;             // keys per unit
    int32_t row0;          // first key row inside each unit
    int32_t c_lo;          // first centroid of this launch
    int32_t nslots;        // 1 or 2
    int32_t valid0, valid1;  // centroids in slot 0 / 1
    int32_t n0, n1;          // MMA N of slot 0 / 1 (multiple of 16)
    int32_t merge;         // merge with the running best of earlier launches
    int32_t store_best;    // write the running best for later launches
    int32_t* assign;
    int64_t assign_ustride;
    float* best;
    int64_t best_ustride;
    uint32_t* err;
};

struct __align__(8) Bars {
    uint64_t a_full[2], a_empty[2], b_full, b_empty, t_full[2], t_empty[2], done;
};

// Barrier over the 8 epilogue warps that also ORs a per-thread flag, so that every epilogue
// warp takes the same abort decision after it.
CKV_DEV bool epi_bar_any(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred q, a;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred a, 1, 256, q;\n"
        " selp.u32 %0, 1, 0, a;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)flag)
        : "memory");
    return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap map_a,
                     const __grid_constant__ CUtensorMap map_b, const AssignParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sB = smem;                                       // nslots x 64 KB
    uint8_t* sA = sB + (size_t)p.nslots * kBSlotBytes;        // 2 x 32 KB
    float* xval = (float*)(sA + 2 * kATileBytes);             // [2][128]
    int32_t* xidx = (int32_t*)(xval + 2 * kTileM);            // [2][128]
    Bars* bars = (Bars*)(xidx + 2 * kTileM);
    uint32_t* tmem_slot = (uint32_t*)(bars + 1);
    volatile int32_t* abort_flag = (volatile int32_t*)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t total = (int64_t)p.U * p.T;
    const int64_t f0 = total * blockIdx.x / gridDim.x;
    const int64_t f1 = total * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->a_full[s], 1);
            mbar_init(&bars->a_empty[s], 1);
            mbar_init(&bars->t_full[s], 1);
            mbar_init(&bars->t_empty[s], kEpiWarps);
        }
        mbar_init(&bars->b_full, 1);
        mbar_init(&bars->b_empty, 1);
        mbar_init(&bars->done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&map_a);
            tma_prefetch_desc(&map_b);
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
                    mbar_arrive_expect_tx(&bars->b_full, (uint32_t)p.nslots * kBSlotBytes);
                    for (int h = 0; h < p.nslots; ++h)
                        for (int kh = 0; kh < 2; ++kh)
                            tma_load_3d(sB + h * kBSlotBytes + kh * kBHalfBytes, &map_b,
                                        &bars->b_full, kh * 64, p.c_lo + h * kSlotCols, u);
                    ++nb;
                    cur_u = u;
                }
                const int s = (int)(i & 1);
                if (!mbar_wait(&bars->a_empty[s], ((uint32_t)(i >> 1) & 1u) ^ 1u, p.err)) {
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
            for (int64_t j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j)
                mbar_wait(&bars->a_full[j & 1], (uint32_t)(j >> 1) & 1u, p.err);
            if (nb > 0) mbar_wait(&bars->b_full, (nb - 1) & 1, p.err);
        }
    } else if (warp == 9) {
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
                const int s = (int)(i & 1);
                if (!mbar_wait(&bars->a_full[s], (uint32_t)(i >> 1) & 1u, p.err)) {
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
                    const uint32_t b_base = smem_u32(sB + hb * kBSlotBytes);
                    const uint32_t d = tbase + (uint32_t)(h * kSlotCols);
                    const uint32_t idesc = hb == 0 ? idesc0 : idesc1;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t koff = (uint32_t)((kk & 3) * 32);
                        const uint64_t ad = sw128_kmajor_desc(a_base + (kk >> 2) * kAHalfBytes + koff);
                        const uint64_t bd = sw128_kmajor_desc(b_base + (kk >> 2) * kBHalfBytes + koff);
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
        const int quad = warp & 3;
        const int half = warp >> 2;
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
                float v[4][32];
                const int col0 = half * 128;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    if (col0 + cc * 32 < valid)
                        tmem_ld32(lane_addr + (uint32_t)(h * kSlotCols + col0 + cc * 32), v[cc]);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->t_empty[h]);
                const int cbase = p.c_lo + hb * kSlotCols + col0;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int c0 = col0 + cc * 32;
                    if (c0 >= valid) break;
                    if (c0 + 32 > valid) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (c0 + j >= valid) v[cc][j] = -INFINITY;
                    }
                    float mx = v[cc][0];
#pragma unroll
                    for (int j = 1; j < 32; ++j) mx = fmaxf(mx, v[cc][j]);
                    if (mx > best) {
                        int jj = 31;
#pragma unroll
                        for (int j = 31; j >= 0; --j)
                            if (v[cc][j] == mx) jj = j;
                        best = mx;
                        bidx = cbase + cc * 32 + jj;
                    }
                }
            }
            const int buf = (int)(i & 1);
            if (half == 1) {
                xval[buf * kTileM + row] = best;
                xidx[buf * kTileM + row] = bidx;
            }
            if (epi_bar_any(!ok || *abort_flag)) {
                *abort_flag = 1;
                break;
            }
            if (half == 0) {
                const float ov = xval[buf * kTileM + row];
                const int32_t oi = xidx[buf * kTileM + row];
                if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
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
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tbase, 512);
}

}  // namespace

int launch_kmeans_assign(const KeysView& k, const uint16_t* mu_hat, int64_t muhat_ustride,
                         int32_t C, int32_t* assign, int64_t assign_ustride, float* best,
                         int64_t best_ustride, uint32_t* err, cudaStream_t s) {
    if (k.m <= 0 || k.U <= 0) return CKV_OK;
    CUtensorMap map_a, map_b;
    int rc = encode_bf16_3d(&map_a, k.base, kD, (uint64_t)k.n_rows, (uint64_t)k.U, kD * 2,
                            (uint64_t)k.n_rows * kD * 2, 64, kTileM);
    if (rc != CKV_OK) return rc;
    rc = encode_bf16_3d(&map_b, mu_hat, kD, (uint64_t)C, (uint64_t)k.U, kD * 2,
                        (uint64_t)muhat_ustride * kD * 2, 64, kSlotCols);
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
    p.err = err;
    const int nchunks = (C + 2 * kSlotCols - 1) / (2 * kSlotCols);
    const int sms = num_sms_of_current_device();
    const int64_t total = (int64_t)p.U * p.T;
    const int grid = (int)(total < sms ? total : sms);
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
        const size_t smem = 1024 + (size_t)p.nslots * kBSlotBytes + 2 * kATileBytes +
                            4 * kTileM * 4 + sizeof(Bars) + 64;
        cudaError_t e = cudaFuncSetAttribute(assign_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "assign: set smem");
        assign_tc_kernel<<<grid, kThreads, smem, s>>>(map_a, map_b, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "assign: launch");
    }
    return CKV_OK;
}

}  // namespace ckv
