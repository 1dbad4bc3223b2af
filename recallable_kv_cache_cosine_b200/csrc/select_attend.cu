// Fused ClusterKV decode step: centroid scoring, budgeted cluster selection, gather and
// sparse GQA flash-decode, in one launch (sm_100a).
//
// Page: "大模型KV Cache压缩技术：ClusterKV的语义空间优化" (ClusterKV explainer).
//  - section 3.3 (select_clusters): score every cluster by q . centroid; visit clusters by
//    descending score; take whole clusters while they fit the budget; the first cluster that
//    does not fit is filled with its top-`remaining` tokens by q . k; stop;
//  - section 3.1: attention softmax(q K^T / sqrt(d)) V over the recalled tokens;
//  - section 4.1: each cluster's KV is stored contiguously, so a whole selected cluster is
//    one contiguous run of rows.
// Readings: one selection per KV head with qbar = sum of its G query heads; ties go to the
// lower cluster index and the lower token id; the 16 sinks and the pending tokens are always
// attended and counted against the budget.
//
// One unit (sequence b, KV head h) is served by a thread-block cluster of S CTAs. The launch
// is split around the programmatic-dependent-launch wait:
//   0. before the wait, while the previous kernel of the stream may still run, each CTA
//      bulk-copies its slice of the fp32 centroids into shared memory, loads the cluster
//      boundaries and prefetches the queries and the sink / pending rows into L2. The store
//      is only written by this library's own kernels, and the last kernel of every call that
//      writes it signals its dependents only when it ends, so these reads see the finished
//      store. The queries, the sink / pending rows and every output are touched only after
//      the wait;
//   1. qbar = sum of the group's queries; each CTA scores its slice (a warp per centroid,
//      eight in flight, their lane sums reduced together) and stores the scores into every
//      CTA of the cluster by asynchronous remote stores (st.async) that count their bytes on
//      the receiver's mbarrier; each CTA goes on once its own copy is complete;
//   2. every CTA computes the same selection on its own. The walk in descending
//      (score, -index) order stops at the first cluster whose inclusive token count exceeds
//      the remaining budget R: the cut, a size-weighted quantile of the scores. The scores are
//      mapped monotonically onto 256 linear buckets between the smallest and the largest;
//      a size-weighted histogram gives the cut's bucket b*. The clusters of b* and above (a
//      dozen or two) are compacted and ranked exactly among themselves in one pass, which
//      gives each one's walk rank and prefix: the whole clusters in walk order, and the cut;
//   3. the selected rows form one index space: sinks, pending (in append order, from the
//      two-window pending ring), whole clusters in walk order, then the partial tokens of the cut
//      cluster in store order. With a partial fill and S > 1, CTA S-1 takes the partial
//      tokens: it bulk-copies the cut cluster's K and V rows (started during the selection
//      when the histogram isolates the cut), ranks the tokens by qbar . k there and attends
//      the top ones in place; it also takes the last whole rows, up to an even share of the
//      work less the cut cluster it loaded. The other CTAs split the rest evenly;
//   4. rows reach a shared-memory ring in runs: each run of consecutive store rows (the
//      sinks, the pending rows, the selected part of a whole cluster) by one bulk copy
//      (cp.async.bulk) for K and one for V, completing on the chunk's mbarrier. Ring rows are
//      store rows as they are; the store keeps chunk c of row r at c ^ (r & 7), so the 8 rows
//      of a matrix load fall on distinct banks. Each warp runs flash-decode on 16-row tiles with
//      tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulate): S^T = K Q^T with the
//      rows as M and the G query heads as N, an online softmax per head, then O^T += V^T P
//      with P split into bf16 high and low parts;
//   5. the warp partials (max, sum, accumulator) are merged per CTA; the other CTAs store
//      theirs into CTA 0 (st.async, counted on CTA 0's mbarrier), which merges them and
//      writes the fp32 output.
// Every loop that holds a warp-synchronous operation (shuffle, ballot, reduce) starts at a
// warp- or CTA-uniform value and steps by a uniform stride, so all 32 lanes run every
// iteration. Bounded waits that give up set the device error word; the CTA then skips its
// arithmetic but still takes part in every cluster barrier, so no CTA of the cluster hangs.
// A compile-time flag instantiates the kernel for one selection per query head (G = 1 over
// (sequence, query head) units). Another instantiates the mixed-precision decode of the
// explainer's outlook (section 7, lower precision for far clusters): the selection is the
// same, but the rows of clusters at walk rank >= n_near arrive as fp8 e4m3 codes with one fp32
// scale per row. Their codes are bulk-copied into the upper half of their ring row, converted
// exactly to bf16 (e4m3 values are bf16 values) by one warp per row, and the row's scales
// multiply its scores (K) and its softmax weights in the P V product (V).
#include <cuda_fp8.h>
#include <float.h>

#include <map>
#include <mutex>
#include <tuple>

#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

constexpr int kNT = 256;          // threads per CTA
constexpr int kWarps = kNT / 32;
constexpr int kPartCap = 4096;    // cut-cluster tokens ranked in shared memory (outside the ring path)
constexpr float kLog2e = 1.4426950408889634f;
// Ring rows are stored rows copied as they are (256 bytes, chunks in stored order): a run of
// consecutive store rows lands in consecutive ring rows by one bulk copy, and the chunk key of
// each ring row (its store row & 7) spreads the 8 rows a matrix load reads at one logical
// 16-byte column over 8 distinct groups of 4 banks.
constexpr int kPitch = 2 * kD;
constexpr int kRowBytes = 2 * kPitch;  // one K row and one V row
constexpr int kCombStride = 132;       // accumulator[128], max, sum, 2 pad (16-byte rows)

// wbuf slots
constexpr int kWRank = 43;    // the cut's walk rank (the number of whole clusters)
constexpr int kWCut = 41;     // the cut cluster
constexpr int kWPre = 42;     // tokens of bucket b* ranked before the cut
constexpr int kWCopy = 45;    // the cut cluster's bulk copies were issued
constexpr int kWBad = 46;     // a bounded wait of this CTA gave up
constexpr int kWCnt2 = 47;    // candidates found in the bucket of walk rank n_near - 1
constexpr int kWNear = 64;    // [2] the walk key of rank n_near - 1 (two halves)
constexpr int kWList = 66;    // [8] candidates compacted by each warp
constexpr int32_t kFarBit = 0x40000000;  // rsrc flag: a store row read from the fp8 copy

CKV_DEV uint32_t orderable(float f) {
    f = f + 0.0f;  // -0 -> +0
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
CKV_DEV float from_orderable(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
// Walk order key of cluster c: larger = visited earlier (score descending, index ascending).
CKV_DEV uint64_t walk_key(float score, int c) {
    return ((uint64_t)orderable(score) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)c);
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) into this CTA's
// shared memory, completing on the mbarrier at shared address `bar`.
CKV_DEV void bulk_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
CKV_DEV void sts_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}
// Two e4m3 codes (low byte first) -> two bf16 in one word, exactly (every e4m3 value,
// subnormals included, is a bf16 value).
CKV_DEV uint32_t e4m3x2_to_bf16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    const float lo = __half2float(__half(__half_raw{h.x}));
    const float hi = __half2float(__half(__half_raw{h.y}));
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}
// The fp8 copy's value of four bf16 elements held by each lane of a warp (one 128-element
// row): scale = max|x| / 448, code = e4m3(x / scale) (ties to even, saturating), returned
// as the codes' bf16 values; *scale_out = scale. The same arithmetic as the stored copy.
CKV_DEV uint2 fp8_row_values(uint2 w, float* scale_out) {
    const float x0 = bf16_lo(w.x), x1 = bf16_hi(w.x), x2 = bf16_lo(w.y), x3 = bf16_hi(w.y);
    float mx = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float scale = __fdiv_rn(mx, 448.0f);
    *scale_out = scale;
    if (!(scale > 0.f)) return make_uint2(0u, 0u);
    const __nv_fp8x2_storage_t c01 = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(x0, scale), __fdiv_rn(x1, scale)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t c23 = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(x2, scale), __fdiv_rn(x3, scale)), __NV_SATFINITE, __NV_E4M3);
    return make_uint2(e4m3x2_to_bf16x2(c01), e4m3x2_to_bf16x2(c23));
}
CKV_DEV void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}
CKV_DEV void ldsm_x4_trans(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}
// D += A B, m16n8k16, A 16x16 row-major bf16, B 16x8 column-major bf16, D fp32.
CKV_DEV void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                            uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// floor(total * k / parts) in 32-bit arithmetic when the product fits.
CKV_DEV int32_t split_point(int32_t total, uint32_t k, int parts) {
    if ((uint32_t)total < (1u << 27)) return (int32_t)((uint32_t)total * k / (uint32_t)parts);
    return (int32_t)((int64_t)total * k / parts);
}
CKV_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

CKV_DEV uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// qbar . k over one 64-dimension half (`half`) of two K rows, with all 16 loads in flight; a
// negative row index gives 0. Dimensions in ascending order, one fmaf chain per row.
CKV_DEV void half_row_dot2(const uint16_t* kp, int32_t row0, int32_t ia, int32_t ib, int half,
                           const float* qbar, float* sa, float* sb) {
    // kp[i] is store row row0 + i: logical chunk 8 half + t of it is stored at 8 half + (t ^ key)
    uint4 w[2][8];
    const int ka = (row0 + ia) & 7, kb = (row0 + ib) & 7;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        w[0][t] = ia >= 0 ? ldg_nc_v4(kp + (int64_t)ia * kD + 64 * half + 8 * (t ^ ka)) : make_uint4(0u, 0u, 0u, 0u);
        w[1][t] = ib >= 0 ? ldg_nc_v4(kp + (int64_t)ib * kD + 64 * half + 8 * (t ^ kb)) : make_uint4(0u, 0u, 0u, 0u);
    }
    const float4* q4 = reinterpret_cast<const float4*>(qbar + 64 * half);
    float s[2] = {0.f, 0.f};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const float4 qa = q4[2 * t], qb = q4[2 * t + 1];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            s[r] = fmaf(qa.x, bf16_lo(w[r][t].x), s[r]);
            s[r] = fmaf(qa.y, bf16_hi(w[r][t].x), s[r]);
            s[r] = fmaf(qa.z, bf16_lo(w[r][t].y), s[r]);
            s[r] = fmaf(qa.w, bf16_hi(w[r][t].y), s[r]);
            s[r] = fmaf(qb.x, bf16_lo(w[r][t].z), s[r]);
            s[r] = fmaf(qb.y, bf16_hi(w[r][t].z), s[r]);
            s[r] = fmaf(qb.z, bf16_lo(w[r][t].w), s[r]);
            s[r] = fmaf(qb.w, bf16_hi(w[r][t].w), s[r]);
        }
    }
    *sa = s[0];
    *sb = s[1];
}

// Exclusive block scan of one int per thread: x = this thread's exclusive prefix, y = the
// block total. Not inlined: it is called from several places, and one copy of its code
// keeps the kernel's instruction footprint smaller.
__device__ __noinline__ int2 block_excl_scan(int32_t v, int32_t* wscan) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wscan[warp] = incl;
    __syncthreads();
    int32_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int32_t x = wscan[w];
        if (w < warp) before += x;
        total += x;
    }
    __syncthreads();
    return make_int2(before + incl - v, total);
}

// The same scan on two ints at once: x / y = this thread's exclusive prefixes of a / b,
// z / w = the block totals.
__device__ __noinline__ int4 block_excl_scan2(int32_t a, int32_t b, int32_t* wscan) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t ya = __shfl_up_sync(0xffffffffu, ia, o);
        const int32_t yb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
            ia += ya;
            ib += yb;
        }
    }
    if (lane == 31) {
        wscan[warp] = ia;
        wscan[kWarps + warp] = ib;
    }
    __syncthreads();
    int32_t ba = 0, bb = 0, ta = 0, tb = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int32_t xa = wscan[w], xb = wscan[kWarps + w];
        if (w < warp) {
            ba += xa;
            bb += xb;
        }
        ta += xa;
        tb += xb;
    }
    __syncthreads();
    return make_int4(ba + ia - a, bb + ib - b, ta, tb);
}


// Warp 0 of a radix pass: bins hold weights in descending digit order; find the digit whose
// bin contains the position `need` (0-based, counting weight from the top), i.e. the first
// bin whose inclusive cumulative weight exceeds `need`. Writes the digit and the weight
// above it. `first_exceeding` = false finds the bin of the need-th key (1-based) instead.
CKV_DEV void radix_pick_bin(const int32_t* hist, int32_t need, bool first_exceeding, int32_t* out) {
    const int lane = threadIdx.x & 31;
    int32_t cnt[8], tot = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        cnt[e] = hist[255 - 8 * lane - e];
        tot += cnt[e];
    }
    int32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    int32_t above = incl - tot;
    const bool mine = first_exceeding ? (above <= need && need < incl) : (above < need && need <= incl);
    if (mine) {
        for (int e = 0; e < 8; ++e) {
            const bool hit = first_exceeding ? (need < above + cnt[e]) : (need <= above + cnt[e]);
            if (hit) {
                out[0] = 255 - 8 * lane - e;
                out[1] = above;
                break;
            }
            above += cnt[e];
        }
    }
}

// The bucket (of 256, scanned from the top) whose inclusive cumulative weight first exceeds
// `need`, and the weight of the buckets above it, computed by a whole warp; every lane
// returns both. The caller guarantees that the total weight exceeds `need`.
CKV_DEV int cut_bucket_warp(const int32_t* hist, int32_t need, int32_t* above_out) {
    const int lane = threadIdx.x & 31;
    int32_t cnt[8], tot = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        cnt[e] = hist[255 - 8 * lane - e];
        tot += cnt[e];
    }
    int32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    int32_t above = incl - tot;
    int bin = 255;
    int32_t ab = 0;
    const bool mine = above <= need && need < incl;
    if (mine) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (need < above + cnt[e]) {
                bin = 255 - 8 * lane - e;
                ab = above;
                break;
            }
            above += cnt[e];
        }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, mine);
    const int src = who ? __ffs(who) - 1 : 0;
    *above_out = __shfl_sync(0xffffffffu, ab, src);
    return __shfl_sync(0xffffffffu, bin, src);
}

// Arguments of partial_rows (below), the partial tokens of a cut cluster that is not held in
// the ring (a large cluster, or a CTA that is not the dedicated one). Not inlined: a cold path.
struct PartialArgs {
    const uint16_t* kp;  // the cut cluster's first K row
    uint32_t* gkeys;     // global key scratch of the unit (cuts of more than kNT tokens)
    const float* qbar;   // shared [128]
    uint32_t* pkey;      // shared [kPartCap + 4]
    int32_t* hist;       // shared [256]
    int32_t* wbuf;       // shared scan / pick scratch
    int32_t* prow;       // shared: this CTA's partial rows
    int32_t crow, csz, r_part, p_lo, p_hi;
    int32_t rank, S;
};
// The cut cluster's partial rows of this CTA: the top r_part tokens by qbar . k (ties: lower
// index), listed at selection positions [p_lo, p_hi) of the partial fill. A cut of more than
// kNT tokens is scored by every CTA of the cluster (an even share each) into the unit's global
// key scratch, then read back after a cluster barrier (into shared memory when it fits);
// every CTA of the cluster must call this then.
__device__ __noinline__ void partial_rows(const PartialArgs& P) {
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool coop = P.csz > kNT;
    const bool in_smem = P.csz <= kPartCap;
    auto score_keys = [&](int32_t k0, int32_t k1, uint32_t* dst) {
        // two threads per row, two rows per thread pair: one memory round trip per 256 rows
        for (int32_t i0 = k0; i0 < k1; i0 += kNT) {  // CTA-uniform trip count
            const int32_t ia = i0 + (tid >> 1), ib = ia + kNT / 2;
            const int half = tid & 1;
            float sa, sb;
            half_row_dot2(P.kp, P.crow, ia < k1 ? ia : -1, ib < k1 ? ib : -1, half, P.qbar, &sa, &sb);
            sa += __shfl_xor_sync(0xffffffffu, sa, 1);
            sb += __shfl_xor_sync(0xffffffffu, sb, 1);
            if (half == 0) {
                if (ia < k1) dst[ia] = orderable(sa);
                if (ib < k1) dst[ib] = orderable(sb);
            }
        }
    };
    if (coop) {
        const int32_t k0 = (int32_t)((int64_t)P.csz * P.rank / P.S);
        const int32_t k1 = (int32_t)((int64_t)P.csz * (P.rank + 1) / P.S);
        score_keys(k0, k1, P.gkeys);
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    if (P.p_hi <= P.p_lo) return;
    if (coop && in_smem) {
        for (int i = tid; i < P.csz; i += kNT) P.pkey[i] = __ldcg(P.gkeys + i);
    } else if (!coop) {
        score_keys(0, P.csz, P.pkey);
    }
    if (in_smem && tid < 4) P.pkey[P.csz + tid] = 0u;  // pad: never outranks a key
    auto key_at = [&](int i) -> uint32_t { return in_smem ? P.pkey[i] : __ldcg(P.gkeys + i); };
    __syncthreads();
    if (P.csz <= kNT) {
        // comparison rank (ties: lower index), tpe threads per token, 4 keys per load
        const int tpe = P.csz <= 32 ? 8 : (P.csz <= 64 ? 4 : (P.csz <= 128 ? 2 : 1));
        const int e = tid / tpe, sub = tid % tpe;
        int32_t rk = 0;
        if (e < P.csz) {
            const uint32_t ke = P.pkey[e];
            const uint4* k4 = reinterpret_cast<const uint4*>(P.pkey);
            const int n4 = (P.csz + 3) >> 2;
            for (int j4 = sub; j4 < n4; j4 += tpe) {
                const uint4 v = k4[j4];
                const int j = 4 * j4;
                rk += (v.x > ke) || (v.x == ke && j < e);
                rk += (v.y > ke) || (v.y == ke && j + 1 < e);
                rk += (v.z > ke) || (v.z == ke && j + 2 < e);
                rk += (v.w > ke) || (v.w == ke && j + 3 < e);
            }
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
            const int32_t y = __shfl_xor_sync(0xffffffffu, rk, o);
            if (o < tpe) rk += y;
        }
        const int32_t sel = (e < P.csz && sub == 0 && rk < P.r_part) ? 1 : 0;
        const int32_t pos = block_excl_scan(sel, P.wbuf).x;
        if (sel && pos >= P.p_lo && pos < P.p_hi) P.prow[pos - P.p_lo] = P.crow + e;
    } else {
        // radix select over 4 digits of 8 bits, most significant first: the threshold key
        // theta and `pneed` = how many keys equal to theta are taken (the lowest-index ones),
        // so that exactly r_part tokens are selected.
        uint32_t prefix = 0, mask = 0;
        int32_t pneed = P.r_part;
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            P.hist[tid] = 0;
            __syncthreads();
            for (int i = tid; i < P.csz; i += kNT) {
                const uint32_t k = key_at(i);
                if ((k & mask) == prefix) atomicAdd(&P.hist[(k >> shift) & 255u], 1);
            }
            __syncthreads();
            if (warp == 0) radix_pick_bin(P.hist, pneed, false, P.wbuf + 32);
            __syncthreads();
            pneed -= P.wbuf[33];
            prefix |= (uint32_t)P.wbuf[32] << shift;
            mask |= 255u << shift;
        }
        const uint32_t theta = prefix;
        // a contiguous run of keys per thread, in index order: the keys equal to theta before
        // the run (one scan), then the selected keys before the run (another scan)
        const int per = (P.csz + kNT - 1) / kNT;
        const int i0 = tid * per;
        const int i1 = i0 + per < P.csz ? i0 + per : P.csz;
        int32_t neq = 0;
        for (int i = i0; i < i1; ++i) neq += key_at(i) == theta ? 1 : 0;
        const int32_t eq0 = block_excl_scan(neq, P.wbuf).x;
        int32_t nsel = 0, eq = eq0;
        for (int i = i0; i < i1; ++i) {
            const uint32_t k = key_at(i);
            if (k > theta) {
                ++nsel;
            } else if (k == theta) {
                nsel += eq < pneed ? 1 : 0;
                ++eq;
            }
        }
        int32_t pos = block_excl_scan(nsel, P.wbuf).x;
        eq = eq0;
        for (int i = i0; i < i1; ++i) {
            const uint32_t k = key_at(i);
            bool sel = k > theta;
            if (k == theta) {
                sel = eq < pneed;
                ++eq;
            }
            if (sel) {
                if (pos >= P.p_lo && pos < P.p_hi) P.prow[pos - P.p_lo] = P.crow + i;
                ++pos;
            }
        }
    }
    __syncthreads();
}

// Shared-memory layout, computed identically on the host (launch size) and the device.
struct Layout {
    uint32_t ring, qbar, qh, score, off, spre, cand, clist, bkt, hist, hcnt, hnear, rkey, prow,
        rsrc, rks, rvs, key8, wbuf, scl, ccomb, pbuf, bars, total;
};
// The ring also holds, before any row arrives, the centroid slice (up to ring / 512 rows of
// fp32 centroids per chunk) and the cut cluster's keys; after the last row, the warp partials.
__host__ __device__ inline uint32_t ring_bytes(int G, int RB) {
    uint32_t r = (uint32_t)RB * kRowBytes;
    const uint32_t w = 4u * kWarps * G * kCombStride;
    const uint32_t k = 4u * (kPartCap + 4);
    if (w > r) r = w;
    if (k > r) r = k;
    return r;
}
__host__ __device__ inline Layout make_layout(int G, int S, int C, int RB, int prow_cap, bool mixed) {
    Layout L{};
    uint32_t p = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t r = p;
        p += (bytes + 127u) & ~127u;
        return r;
    };
    L.ring = take(ring_bytes(G, RB));
    L.qbar = take(4u * kD);
    L.qh = take(2u * G * kD);
    L.score = take(4u * C);
    L.off = take(4u * (C + 1));
    L.spre = take(4u * (C + 1));
    L.cand = take(4u * C);
    L.bkt = take((uint32_t)C);
    L.hist = take(4u * 256);
    L.hcnt = take(4u * 256);
    L.hnear = take(4u * 256);
    L.rkey = take(4u * (RB + 4));
    L.prow = take(4u * prow_cap);
    L.rsrc = take(mixed ? 4u * RB : 0u);  // far-row sources and scales: mixed precision only
    L.rks = take(mixed ? 4u * RB : 0u);
    L.rvs = take(mixed ? 4u * RB : 0u);
    L.key8 = take((uint32_t)RB);  // per ring row: the chunk key of its store row
    L.wbuf = take(4u * 128);
    L.scl = take(4u * ((kWarps + S) * G + 2 * G));
    L.ccomb = take(4u * S * G * kCombStride);
    L.pbuf = take(2u * kWarps * 256);
    // the warps' candidate lists (walk keys) live in pbuf, which only the attention uses, when
    // they fit (C <= 512)
    const uint32_t nlist = 256u * (uint32_t)((C + 255) / 256);
    L.clist = 8u * nlist <= 2u * kWarps * 256 ? L.pbuf : take(8u * nlist);
    L.bars = take(8u * 6);
    L.total = p;
    return L;
}

struct Params {
    int32_t S;         // CTAs per unit (thread-block cluster size)
    int32_t RB;        // ring rows
    int32_t prow_cap;  // partial rows one CTA may own
    int32_t hold;      // 1: the CTAs of a cluster leave together, when CTA 0 is done
};

// kPerHead: one selection per query head. The kernel then runs with G = 1 over virtual
// units (b, query head): virtual unit v reads the store of KV unit v / a.qsplit and its own
// query, output and selection rows. kMixed: rows of clusters at walk rank >= a.n_near are
// read from the fp8 copy.
template <int G, bool kPerHead, bool kMixed>
__global__ void __launch_bounds__(kNT, 2) select_attend_kernel(const DecodeArgs a, const Params P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int C = a.C;
    const int S = P.S, RB = P.RB;
    const uint32_t rank = cluster_ctarank();
    const int unit = blockIdx.x / S;
    const int su = kPerHead ? unit / a.qsplit : unit;  // the store's unit
    const int b = unit / a.Hkv, h = unit % a.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const Layout Ly = make_layout(G, S, C, RB, P.prow_cap, kMixed);
    const int cch = (int)(ring_bytes(G, RB) / (kD * 4));  // centroid rows per slice chunk
    uint8_t* const base = smem_raw;
    float* const s_qbar = (float*)(base + Ly.qbar);
    uint16_t* const s_qh = (uint16_t*)(base + Ly.qh);
    float* const s_score = (float*)(base + Ly.score);
    int32_t* const s_off = (int32_t*)(base + Ly.off);
    int32_t* const s_spre = (int32_t*)(base + Ly.spre);
    int32_t* const s_cand = (int32_t*)(base + Ly.cand);
    uint64_t* const s_clist = (uint64_t*)(base + Ly.clist);  // candidates' walk keys (warp lists)
    uint8_t* const s_bkt = base + Ly.bkt;  // every cluster's score bucket
    int32_t* const s_hist = (int32_t*)(base + Ly.hist);
    int32_t* const s_hcnt = (int32_t*)(base + Ly.hcnt);
    int32_t* const s_hnear = (int32_t*)(base + Ly.hnear);
    float* const s_rks = (float*)(base + Ly.rks);  // per ring row: K scale (1 for bf16 rows)
    float* const s_rvs = (float*)(base + Ly.rvs);  // per ring row: V scale
    uint32_t* const s_rkey = (uint32_t*)(base + Ly.rkey);
    int32_t* const s_prow = (int32_t*)(base + Ly.prow);
    int32_t* const s_rsrc = (int32_t*)(base + Ly.rsrc);
    uint8_t* const s_key8 = base + Ly.key8;
    int32_t* const s_wbuf = (int32_t*)(base + Ly.wbuf);
    float* const s_scl = (float*)(base + Ly.scl);
    float* const s_ccomb = (float*)(base + Ly.ccomb);
    uint16_t* const s_pbuf = (uint16_t*)(base + Ly.pbuf);
    uint64_t* const cbar = (uint64_t*)(base + Ly.bars);      // centroid slice
    uint64_t* const fbar = cbar + 1;                         // cut cluster rows (a warp's arrival each)
    uint64_t* const rbar = cbar + 2;                         // [2] ring chunk slots (a warp's arrival each)
    uint64_t* const xbar = cbar + 4;                         // the other slices' scores and keys
    uint64_t* const obar = cbar + 5;                         // the other CTAs' partials (CTA 0)
    float* const s_cent = (float*)(base + Ly.ring);          // centroid slice (aliases the ring)
    float* const s_wcomb = (float*)(base + Ly.ring);         // warp partials (after the rows)
    uint32_t* const s_pkey = (uint32_t*)(base + Ly.ring);    // cut keys (before the rows)
    const uint32_t ringK = smem_u32(base + Ly.ring);
    const uint32_t ringV = ringK + (uint32_t)RB * kPitch;

    const int64_t kp_base = (int64_t)su * a.kp_ustride;
    const int64_t sp_base = (int64_t)su * a.sp_ustride;
    const int32_t* off_g = a.offsets + (int64_t)su * a.off_ustride;
    const float* mu = a.mu + (int64_t)su * a.mu_ustride * kD;
    const int c_begin = C * (int)rank / S;  // C <= 4096, S <= 16: no overflow
    const int c_end = C * ((int)rank + 1) / S;
    const int nc = c_end - c_begin;
    const uint16_t* qsrc = a.q + ((int64_t)b * a.Hkv * G + (int64_t)h * G) * kD;

    // ---------------------------------------------------------------- phase 0: the store
    // (before the dependency wait; see the header comment for why the store may be read here)
    pdl_launch_dependents();
    if (tid == 0) {
        mbar_init(cbar, 1);
        mbar_init(fbar, 1);
        mbar_init(rbar, kWarps);  // a byte-count arrival per warp
        mbar_init(rbar + 1, kWarps);
        mbar_init(xbar, 1);
        mbar_init(obar, 1);
        fence_mbar_init();
        // bytes the other CTAs store here: their slices' scores and two keys each; into CTA 0,
        // their partials
        const uint32_t bx = 4u * (uint32_t)(C - nc) + 8u * (uint32_t)(S - 1);
        if (bx) mbar_arrive_expect_tx(xbar, bx);
        else mbar_arrive(xbar);
        const uint32_t bo = rank == 0 ? 4u * (uint32_t)((S - 1) * G * kCombStride) : 0u;
        if (bo) mbar_arrive_expect_tx(obar, bo);
        else mbar_arrive(obar);
        s_wbuf[kWCopy] = 0;
        s_wbuf[kWBad] = 0;
    }
    __syncthreads();
    cluster_arrive_relaxed();  // this CTA runs and its mbarriers are set: others may store here
    if (tid == 0 && nc > 0) {  // the slice's first chunk
        const uint32_t bytes = (uint32_t)min(nc, cch) * kD * 4;
        mbar_arrive_expect_tx(cbar, bytes);
        bulk_load(s_cent, mu + (int64_t)c_begin * kD, bytes, cbar);
    }
    if (tid < 2 * G) prefetch_l2(qsrc + tid * 64);  // the queries, one 128-byte line each
    if (rank == 0 && tid == 32) {  // sinks, then the pending rows (up to two runs of the ring)
        const int32_t run1 = min(a.pending, a.pring - a.pstart);
        const int64_t r0[3] = {0, a.n_sink + a.pstart, a.n_sink};
        const int32_t nr[3] = {a.n_sink, run1, a.pending - run1};
        for (int k = 0; k < 3; ++k)
            if (nr[k] > 0) {
                prefetch_l2_bulk(a.spk + (sp_base + r0[k]) * kD, (uint32_t)nr[k] * kD * 2);
                prefetch_l2_bulk(a.spv + (sp_base + r0[k]) * kD, (uint32_t)nr[k] * kD * 2);
            }
    }
    for (int i = tid; i <= C; i += kNT) s_off[i] = off_g[i];
    s_hist[tid] = 0;
    s_hcnt[tid] = 0;
    s_hnear[tid] = 0;
    if (tid == 0) s_wbuf[kWCnt2] = 0;
    pdl_wait();

    // ---------------------------------------------------------------- phase 1: scores
    const int32_t pend = a.pending;
    const int32_t R = a.budget - a.n_sink - pend;  // >= 0 (host-checked)
    if (tid < kD) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const uint16_t raw = qsrc[g * kD + tid];
            s += __uint_as_float((uint32_t)raw << 16);
            s_qh[g * kD + tid] = raw;
        }
        s_qbar[tid] = s;
    }
    __syncthreads();
    bool ok = true;
    auto size_of = [&](int c) { return s_off[c + 1] - s_off[c]; };
    // One arrival per warp on a chunk mbarrier, announcing the bytes its lanes copy (before
    // any of those copies is issued, so the transaction count never goes below zero).
    auto warp_arrive = [&](uint64_t* bar, uint32_t bytes) {
        const uint32_t total = __reduce_add_sync(0xffffffffu, bytes);
        if (lane == 0) {
            if (total) mbar_arrive_expect_tx(bar, total);
            else mbar_arrive(bar);
        }
        __syncwarp();
    };
    // The slice's scores are stored into every CTA's shared memory, and so are the slice's
    // smallest and largest order keys (over the clusters with tokens; over every cluster in
    // the mixed-precision instantiation, whose rank counts empty clusters too): asynchronous
    // stores that count their bytes on the receiver's mbarrier xbar, so that each CTA goes on
    // once its own copy is complete. The remote stores wait for the arrival every CTA made
    // once it started.
    uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
    cluster_wait_acquire();
    {
        const float4 qv = reinterpret_cast<const float4*>(s_qbar)[lane];
        // The slice in chunks of at most cch centroids (one chunk unless C / S exceeds the
        // ring); a warp per centroid (lane: dims 4 lane .. 4 lane + 3, a conflict-free 512-byte
        // row), eight centroids per warp in flight. The eight lane sums are reduced together:
        // each exchange step halves the values a lane keeps (xor 16: four, xor 8: two, xor 4:
        // one), then xor 2 and 1 finish the sum, so lane l ends with the full score of the
        // warp's centroid number l >> 2 (9 shuffles for 8 scores).
        for (int done = 0, chunk_no = 0; done < nc; ++chunk_no) {
            const int n1 = min(nc - done, cch);
            ok = ok && mbar_wait(cbar, (uint32_t)(chunk_no & 1), a.err);
            for (int j0 = warp; j0 < n1; j0 += 8 * kWarps) {
                float p[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int j = j0 + k * kWarps;
                    p[k] = 0.f;
                    if (ok && j < n1) {
                        const float4 mv = reinterpret_cast<const float4*>(s_cent + (size_t)j * kD)[lane];
                        p[k] = fmaf(qv.w, mv.w, fmaf(qv.z, mv.z, fmaf(qv.y, mv.y, qv.x * mv.x)));
                    }
                }
                const bool hA = (lane & 16) != 0, hB = (lane & 8) != 0, hC = (lane & 4) != 0;
                float q[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)  // q[i]: centroid 4 hA + i
                    q[i] = (hA ? p[4 + i] : p[i]) + __shfl_xor_sync(0xffffffffu, hA ? p[i] : p[4 + i], 16);
                const float r0 = (hB ? q[2] : q[0]) + __shfl_xor_sync(0xffffffffu, hB ? q[0] : q[2], 8);
                const float r1 = (hB ? q[3] : q[1]) + __shfl_xor_sync(0xffffffffu, hB ? q[1] : q[3], 8);
                float v = (hC ? r1 : r0) + __shfl_xor_sync(0xffffffffu, hC ? r0 : r1, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                const int j = j0 + (lane >> 2) * kWarps;  // lanes 4 k store centroid k's score
                if ((lane & 3) == 0 && j < n1) {
                    const int c = c_begin + done + j;
                    s_score[c] = v;
                    if (kMixed || size_of(c) > 0) {
                        const uint32_t key = orderable(v);
                        kmn = min(kmn, key);
                        kmx = max(kmx, key);
                    }
                }
            }
            done += n1;
            if (done < nc) {  // the next chunk, once every warp is done with this one
                __syncthreads();
                if (tid == 0) {
                    fence_proxy_async();
                    const uint32_t bytes = (uint32_t)min(nc - done, cch) * kD * 4;
                    mbar_arrive_expect_tx(cbar, bytes);
                    bulk_load(s_cent, mu + (int64_t)(c_begin + done) * kD, bytes, cbar);
                }
            }
        }
    }
    {
        kmn = __reduce_min_sync(0xffffffffu, kmn);
        kmx = __reduce_max_sync(0xffffffffu, kmx);
        uint32_t* kb = reinterpret_cast<uint32_t*>(s_wbuf + 48);  // [8] minima, [8] maxima
        if (lane == 0) {
            kb[warp] = kmn;
            kb[8 + warp] = kmx;
        }
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                kmn = min(kmn, kb[w]);
                kmx = max(kmx, kb[8 + w]);
            }
            s_wbuf[80] = (int32_t)kmn;  // this CTA's slice
            s_wbuf[81] = (int32_t)kmx;
        }
        __syncthreads();
        if (tid < S) {  // this slice's smallest and largest keys into every CTA
            int32_t* dst = &s_wbuf[96 + 2 * rank];
            if (tid == (int)rank) {
                dst[0] = s_wbuf[80];
                dst[1] = s_wbuf[81];
            } else {
                st_async_v2_u32(map_shared_rank(smem_u32(dst), (uint32_t)tid), (uint32_t)s_wbuf[80],
                                (uint32_t)s_wbuf[81], map_shared_rank(smem_u32(xbar), (uint32_t)tid));
            }
        }
        // the slice's scores into every other CTA: 16-byte pieces over the 16-byte aligned
        // interior [a0, a1), single floats at the two ends
        const int a0 = min((c_begin + 3) & ~3, c_end), a1 = max(c_end & ~3, a0);
        const int nv = (a1 - a0) >> 2, nhead = a0 - c_begin, per = nv + nhead + (c_end - a1);
        for (int t = tid; t < (S - 1) * per; t += kNT) {
            const int k = t / per, i = t - k * per;
            const uint32_t r = (uint32_t)(k < (int)rank ? k : k + 1);  // every CTA but this one
            const uint32_t bar = map_shared_rank(smem_u32(xbar), r);
            if (i < nv) {
                const int c = a0 + 4 * i;
                const uint4 v = *reinterpret_cast<const uint4*>(&s_score[c]);
                st_async_v4_u32(map_shared_rank(smem_u32(&s_score[c]), r), v.x, v.y, v.z, v.w, bar);
            } else {
                const int e = i - nv;
                const int c = e < nhead ? c_begin + e : a1 + (e - nhead);
                st_async_f32(map_shared_rank(smem_u32(&s_score[c]), r), s_score[c], bar);
            }
        }
    }
    // every slice's scores and keys are here: warp 0 waits (the others sleep at the block
    // barrier, leaving the issue slots to a co-resident CTA), then each thread acquires the
    // completed phase itself
    if (warp == 0) ok = mbar_wait_cluster(xbar, 0, a.err) && ok;
    __syncthreads();
    if (warp != 0) ok = mbar_try_wait_cluster(xbar, 0) && ok;

    // ---------------------------------------------------------------- phase 2: selection
    const int32_t m_tot = s_off[C] - s_off[0];
    const bool has_cut = m_tot > R;  // otherwise every cluster is whole
    float smin = 0.f, inv = 0.f;
    int bstar = 0;
    int32_t w_above = 0;
    auto bucket = [&](float sc) {
        const float t = (sc + 0.0f - smin) * inv;
        return (int)fminf(fmaxf(t, 0.f), 255.f);
    };
    // mixed precision: the walk key of rank n_near - 1 separates near from far clusters
    const bool mid_near = kMixed && a.n_near > 0 && a.n_near < C;
    if (has_cut || mid_near) {
        // the smallest and largest score over the slices, then every cluster's bucket
        uint32_t gmn = 0xFFFFFFFFu, gmx = 0u;
        for (int r = 0; r < S; ++r) {
            gmn = min(gmn, (uint32_t)s_wbuf[96 + 2 * r]);
            gmx = max(gmx, (uint32_t)s_wbuf[97 + 2 * r]);
        }
        const float mn = from_orderable(gmn), mx = from_orderable(gmx);
        const float range = mx - mn;
        smin = mn;
        inv = range > 1e-30f ? 255.99f / range : 0.f;  // finite; 0 puts every score in bucket 0
        for (int c = tid; c < C; c += kNT) {
            const int bk = bucket(s_score[c]);
            s_bkt[c] = (uint8_t)bk;
            const int32_t w = size_of(c);
            if (has_cut && w > 0) {
                atomicAdd(&s_hist[bk], w);
                atomicAdd(&s_hcnt[bk], 1);
            }
        }
        __syncthreads();
    }
    if (has_cut) {
        // every warp finds the cut's bucket itself (no extra block barrier)
        bstar = cut_bucket_warp(s_hist, R, &w_above);
        // When b* holds a single cluster with tokens, that cluster is the cut: CTA S-1, which
        // fills the partial tokens, starts the bulk copies of its K and V rows (plain 256-byte
        // rows) now, while the whole clusters are still being ranked.
        if ((int)rank == S - 1 && S > 1 && s_hcnt[bstar] == 1) {
            for (int c = tid; c < C; c += kNT) {
                const int32_t w = size_of(c);
                if (w > 0 && w <= RB && w <= kNT && s_bkt[c] == bstar) {
                    fence_proxy_async();  // the ring's centroid reads come before the copies
                    const int64_t row = kp_base + s_off[c];
                    const uint32_t bytes = (uint32_t)w * kD * 2;
                    mbar_arrive_expect_tx(fbar, 2 * bytes);
                    bulk_load(base + Ly.ring, a.kp + row * kD, bytes, fbar);
                    bulk_load(base + Ly.ring + (size_t)RB * kPitch, a.vp + row * kD, bytes, fbar);
                    s_wbuf[kWCopy] = 1;
                }
            }
        }
    }
    // near(c): walk rank < n_near, i.e. walk key >= the key of rank n_near - 1. The count
    // histogram over the same buckets gives the bucket of that rank; its clusters are ranked
    // exactly among themselves.
    uint64_t k_near = 0;
    if (mid_near) {
        for (int c = tid; c < C; c += kNT) atomicAdd(&s_hnear[s_bkt[c]], 1);
        __syncthreads();
        int32_t n_above = 0;
        const int bn = cut_bucket_warp(s_hnear, a.n_near - 1, &n_above);
        int32_t* cand2 = s_spre;  // free until the whole-size scan below
        for (int c0 = 0; c0 < C; c0 += kNT) {
            const int c = c0 + tid;
            const bool in_b = c < C && s_bkt[c] == bn;
            const uint32_t bal = __ballot_sync(0xffffffffu, in_b);
            int32_t pos0 = 0;
            if (lane == 0 && bal) pos0 = atomicAdd(&s_wbuf[kWCnt2], __popc(bal));
            pos0 = __shfl_sync(0xffffffffu, pos0, 0);
            if (in_b) cand2[pos0 + __popc(bal & ((1u << lane) - 1u))] = c;
        }
        __syncthreads();
        const int32_t n_bn = s_wbuf[kWCnt2];
        for (int i = tid; i < n_bn; i += kNT) {
            const int ci = cand2[i];
            const uint64_t ki = walk_key(s_score[ci], ci);
            int32_t rk = n_above;
            for (int j = 0; j < n_bn; ++j) {
                const int cj = cand2[j];
                rk += walk_key(s_score[cj], cj) > ki ? 1 : 0;
            }
            if (rk == a.n_near - 1) {  // exactly one cluster has this rank
                s_wbuf[kWNear] = (int32_t)(uint32_t)(ki >> 32);
                s_wbuf[kWNear + 1] = (int32_t)(uint32_t)ki;
            }
        }
        __syncthreads();
        k_near = ((uint64_t)(uint32_t)s_wbuf[kWNear] << 32) | (uint64_t)(uint32_t)s_wbuf[kWNear + 1];
    }
    auto is_far = [&](int c) -> bool {
        if (!kMixed || a.n_near >= C) return false;
        if (a.n_near <= 0) return true;
        return walk_key(s_score[c], c) < k_near;
    };
    // Whole clusters, laid out in walk order. With a cut, the candidates are the clusters with
    // tokens in buckets >= b* (a dozen or two): each warp compacts the ones it visits into its
    // own list, and 8 threads per candidate count the candidates before it in walk order and
    // their tokens. A candidate whose prefix plus size fits R is whole at that rank; the one
    // whose prefix fits and whose prefix plus size does not is the cut (its rank is the number
    // of whole clusters). Without a cut every cluster with tokens is whole; they are listed in
    // cluster-index order by one block scan. wl_pre[k] = the selection position (past the
    // sinks and pending rows) of the k-th whole cluster's first row, wl_off[k] = its first
    // store row (kFarBit set when it is attended from the fp8 copy).
    int32_t* const wl_pre = s_spre;  // [n_whole + 1]
    int32_t* const wl_off = s_cand;  // [n_whole]
    int32_t n_whole;
    int32_t cut_c = -1, W_cut = 0;
    if (has_cut) {
        const int cap = 32 * ((C + kNT - 1) / kNT);  // one list of cap entries per warp
        int32_t n_mine = 0;
        for (int c0 = 0; c0 < C; c0 += kNT) {  // CTA-uniform trip count
            const int c = c0 + tid;
            const bool cand = c < C && size_of(c) > 0 && s_bkt[c] >= bstar;
            const uint32_t bal = __ballot_sync(0xffffffffu, cand);
            if (cand) s_clist[warp * cap + n_mine + __popc(bal & ((1u << lane) - 1u))] = walk_key(s_score[c], c);
            n_mine += __popc(bal);
        }
        if (lane == 0) s_wbuf[kWList + warp] = n_mine;
        __syncthreads();
        int32_t pref[kWarps + 1];  // list starts in the flat candidate order
        pref[0] = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) pref[w + 1] = pref[w] + s_wbuf[kWList + w];
        const int32_t n_cand = pref[kWarps];
        auto slot_of = [&](int f) {  // flat candidate index -> slot in the warp lists
            int slot = f;
#pragma unroll
            for (int v = 1; v < kWarps; ++v)
                if (f >= pref[v]) slot = f - pref[v] + v * cap;
            return slot;
        };
        for (int i0 = 0; i0 < n_cand; i0 += kNT / 8) {  // CTA-uniform trip count
            const int i = i0 + (tid >> 3), sub = tid & 7;
            const uint64_t ki = i < n_cand ? s_clist[slot_of(i)] : ~0ull;
            const int ci = (int)(0xFFFFFFFFu - (uint32_t)(ki & 0xFFFFFFFFull));
            int32_t rk = 0, pre = 0;
            for (int j = sub; j < n_cand; j += 8) {
                const uint64_t kj = s_clist[slot_of(j)];
                if (kj > ki) {
                    ++rk;
                    pre += size_of((int)(0xFFFFFFFFu - (uint32_t)(kj & 0xFFFFFFFFull)));
                }
            }
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) {
                rk += __shfl_xor_sync(0xffffffffu, rk, o);
                pre += __shfl_xor_sync(0xffffffffu, pre, o);
            }
            if (i < n_cand && sub == 0) {
                const int c = ci;
                if (pre + size_of(c) <= R) {  // whole
                    wl_pre[rk] = pre;
                    wl_off[rk] = s_off[c] | ((kMixed && is_far(c)) ? kFarBit : 0);
                } else if (pre <= R) {  // the cut
                    s_wbuf[kWCut] = c;
                    s_wbuf[kWPre] = pre;
                    s_wbuf[kWRank] = rk;
                }
            }
        }
        __syncthreads();
        cut_c = s_wbuf[kWCut];
        W_cut = s_wbuf[kWPre];
        n_whole = s_wbuf[kWRank];
        if (tid == 0) wl_pre[n_whole] = W_cut;
    } else {
        const int per = (C + kNT - 1) / kNT;
        const int c0 = tid * per;
        int32_t lsz = 0, lcnt = 0;
        for (int j = 0; j < per; ++j)
            if (c0 + j < C) {
                const int32_t w = size_of(c0 + j);
                lsz += w;
                lcnt += w > 0 ? 1 : 0;
            }
        const int4 sc = block_excl_scan2(lsz, lcnt, s_wbuf);
        int32_t run = sc.x, k = sc.y;
        for (int j = 0; j < per; ++j)
            if (c0 + j < C) {
                const int c = c0 + j;
                const int32_t w = size_of(c);
                if (w > 0) {
                    wl_pre[k] = run;
                    wl_off[k] = s_off[c] | ((kMixed && is_far(c)) ? kFarBit : 0);
                    ++k;
                    run += w;
                }
            }
        n_whole = sc.w;
        if (tid == 0) wl_pre[sc.w] = sc.z;
    }
    __syncthreads();

    // Index-space quantities are below the budget (int32).
    const int32_t W = has_cut ? W_cut : m_tot;  // tokens in whole clusters
    const int32_t r_part = has_cut ? R - W : 0;
    const int32_t csz = has_cut ? size_of(cut_c) : 0;
    const int32_t crow = has_cut ? s_off[cut_c] : 0;
    const int32_t base_w = a.n_sink + pend;
    const int32_t base_p = base_w + W;
    const int32_t T = base_p + r_part;
    // Work split of the selection index space [0, T). With a partial fill, CTA S-1 takes
    // the partial tokens (it also loads and ranks the cut cluster) and the last x whole
    // positions, x = an even share T / S less the cut cluster's rows and a fixed allowance
    // for the ranking (64 rows), at least 0; the other CTAs split the rest.
    const bool dedicated = r_part > 0 && S > 1 && r_part <= P.prow_cap;
    int32_t lo, hi;
    if (dedicated) {
        int32_t x = T / S - csz - 64;
        x = x < 0 ? 0 : (x > base_p ? base_p : x);
        if ((int)rank == S - 1) {
            lo = base_p - x;
            hi = T;
        } else {
            lo = split_point(base_p - x, rank, S - 1);
            hi = split_point(base_p - x, rank + 1, S - 1);
        }
    } else {
        lo = split_point(T, rank, S);
        hi = split_point(T, rank + 1, S);
    }
    const int32_t p_lo = lo > base_p ? lo - base_p : 0;
    const int32_t p_hi = hi > base_p ? hi - base_p : 0;
    const bool coop_cut = csz > kNT;  // scored by every CTA of the cluster (see partial_rows)
    const bool resident = dedicated && (int)rank == S - 1 && csz <= RB && csz <= kNT;
    const bool cut_far = kMixed && has_cut && is_far(cut_c);
    int32_t* sel_out = a.sel_idx ? a.sel_idx + (int64_t)unit * a.budget : nullptr;
    const int32_t* ids = a.ids + kp_base;

    // ---------------------------------------------------------------- phase 3/4: rows
    // A far row (kMixed) arrives as its 128 fp8 codes in the upper half of its ring row, its
    // two scales in rks / rvs; convert_far turns the codes into the bf16 row. rsrc[p] names
    // the source of ring row p (kMixed only): a store row (kFarBit when far) or -1.
    // Far rows of ring rows [p0, p0 + n): one warp per row; lanes 0-7 hold the K code chunks,
    // lanes 8-15 the V code chunks (16 codes each), all read before any bf16 chunk is written.
    auto convert_far = [&](int p0, int n) {
        for (int p = p0 + warp; p < p0 + n; p += kWarps) {  // warp-uniform trip count
            const int32_t r = s_rsrc[p];
            if (r < 0 || (r & kFarBit) == 0) continue;  // uniform across the warp
            const int jj = lane & 7;
            const uint32_t rb = (lane < 8 ? ringK : ringV) + (uint32_t)p * kPitch;
            uint4 c = make_uint4(0u, 0u, 0u, 0u);
            if (lane < 16) c = lds_v4(rb + 128u + (uint32_t)jj * 16u);
            __syncwarp();
            if (lane < 16) {
                const uint4 lo = make_uint4(e4m3x2_to_bf16x2(c.x & 0xFFFFu), e4m3x2_to_bf16x2(c.x >> 16),
                                            e4m3x2_to_bf16x2(c.y & 0xFFFFu), e4m3x2_to_bf16x2(c.y >> 16));
                const uint4 hi = make_uint4(e4m3x2_to_bf16x2(c.z & 0xFFFFu), e4m3x2_to_bf16x2(c.z >> 16),
                                            e4m3x2_to_bf16x2(c.w & 0xFFFFu), e4m3x2_to_bf16x2(c.w >> 16));
                sts_v4(rb + (uint32_t)(2 * jj) * 16u, lo);
                sts_v4(rb + (uint32_t)(2 * jj + 1) * 16u, hi);
            }
            __syncwarp();
        }
    };

    if (!ok) s_wbuf[kWBad] = 1;
    // Streamed positions [lo, s_hi): the resident cut cluster's partial tokens are attended
    // from the rows already in the ring, before the stream reuses it.
    const int32_t s_hi = resident ? (hi < base_p ? hi : base_p) : hi;
    const int32_t n_rows = s_hi - lo;
    const int chunk = n_rows <= RB ? RB : RB / 2;  // <= RB <= kNT: one position per thread
    const int n_chunks = (n_rows + chunk - 1) / chunk;
    // Chunk ch: selection positions [lo + ch * chunk, ...) into ring slot ch & 1. Thread t
    // resolves position c0 + t (a sink or pending row, a whole cluster's row found by binary
    // search over the compact list, or a partial row) and records its ring row's chunk key.
    // Rows come in runs that are consecutive in the store (the sinks, the pending rows up to the
    // ring's end, the selected part of a whole cluster): the thread at a run's first position in
    // the chunk copies the run's K rows and its V rows with one bulk copy each. A partial row,
    // or a far row of the fp8 copy, is a run of its own. Each warp announces its lanes' bytes
    // on the slot's mbarrier before any of them issues a copy.
    auto issue = [&](int ch) {  // every thread
        const int32_t c0 = lo + ch * chunk;
        const int32_t c1 = (c0 + chunk < s_hi) ? c0 + chunk : s_hi;
        const int p = (n_chunks == 1 ? 0 : (ch & 1) * chunk) + tid;
        const uint32_t bar = smem_u32(rbar + (ch & 1));
        const int32_t idx = c0 + tid;
        fence_proxy_async();  // this CTA's earlier accesses of the ring come before the copies
        int32_t r = 0;               // >= 0: store row (| kFarBit when far); < 0: -1 - sink / pending row
        bool starts = true;          // a run starts at idx
        int32_t run_end = idx + 1;   // the end of that run in this chunk
        if (idx >= c1) {
            starts = false;
        } else if (idx < a.n_sink) {  // a sink
            r = -1 - idx;
            starts = idx == c0 || idx == 0;
            run_end = min(c1, a.n_sink);
        } else if (idx < base_w) {  // pending token i, at ring row q of the pending rows
            const int32_t i = idx - a.n_sink, q = (a.pstart + i) % a.pring;
            r = -1 - (a.n_sink + q);
            starts = idx == c0 || i == 0 || q == 0;
            run_end = min(min(c1, base_w), idx + (a.pring - q));
        } else if (idx < base_p) {
            const int32_t x = idx - base_w;
            int k0 = 0, khi = n_whole - 1;  // the whole cluster holding x: last wl_pre <= x
            while (k0 < khi) {
                const int mid = (k0 + khi + 1) >> 1;
                if (wl_pre[mid] <= x) k0 = mid; else khi = mid - 1;
            }
            const int32_t o = wl_off[k0];
            r = (o & ~kFarBit) + (x - wl_pre[k0]);
            if (kMixed && (o & kFarBit)) r |= kFarBit;
            starts = idx == c0 || x == wl_pre[k0];
            run_end = min(c1, base_w + wl_pre[k0 + 1]);
        } else {
            r = s_prow[idx - base_p - p_lo];
            if (kMixed && cut_far) r |= kFarBit;
        }
        const bool far = kMixed && r >= 0 && (r & kFarBit) != 0;
        const bool issues = idx < c1 && (starts || far);
        const int32_t len = far ? 1 : run_end - idx;
        // bulk-copied bytes: the run's K and V rows (bf16), or the row's two code rows (fp8)
        warp_arrive(rbar + (ch & 1), !issues ? 0u : (far ? 2u * kD : (uint32_t)len * kD * 4u));
        const uint32_t dk = ringK + (uint32_t)p * kPitch, dv = ringV + (uint32_t)p * kPitch;
        if (issues) {
            if (far) {
                const int64_t row = kp_base + (r & ~kFarBit);
                bulk_row(dk + 128u, a.kp8 + row * kD, kD, bar);
                bulk_row(dv + 128u, a.vp8 + row * kD, kD, bar);
                s_rks[p] = a.ks8[row];
                s_rvs[p] = a.vs8[row];
            } else {
                const int64_t rk = r >= 0 ? kp_base + r : sp_base + (-1 - r);
                bulk_row(dk, (r >= 0 ? a.kp : a.spk) + rk * kD, (uint32_t)len * kD * 2u, bar);
                bulk_row(dv, (r >= 0 ? a.vp : a.spv) + rk * kD, (uint32_t)len * kD * 2u, bar);
            }
        }
        if (idx >= c1) return;
        s_key8[p] = (uint8_t)((r >= 0 ? (r & ~kFarBit) : -1 - r) & 7);
        if (kMixed) {
            s_rsrc[p] = r;
            if (!far) {
                s_rks[p] = 1.f;
                s_rvs[p] = 1.f;
            }
        }
        if (sel_out)
            sel_out[idx] = r >= 0 ? ids[r & ~kFarBit] : (idx < a.n_sink ? idx : (int32_t)(a.m + idx));
    };

    if (resident) {
        // ---- the cut cluster in shared memory as plain 256-byte rows (K at the ring's start,
        // V at the V half): two bulk copies, issued during the selection when the histogram
        // isolated the cut, else now
        if (tid == 0 && s_wbuf[kWCopy] == 0) {
            fence_proxy_async();  // the ring's earlier shared-memory reads come before the copies
            const uint32_t bytes = (uint32_t)csz * kD * 2;
            mbar_arrive_expect_tx(fbar, 2 * bytes);
            bulk_load(base + Ly.ring, a.kp + (kp_base + crow) * kD, bytes, fbar);
            bulk_load(base + Ly.ring + (size_t)RB * kPitch, a.vp + (kp_base + crow) * kD, bytes, fbar);
        }
        for (int e = tid; e < csz; e += kNT) s_key8[e] = (uint8_t)((crow + e) & 7);
        const bool got = __syncthreads_and(mbar_wait(fbar, 0, a.err) ? 1 : 0) != 0;
        if (!got) s_wbuf[kWBad] = 1;
        // qbar . k, a half-warp per row (16-byte reads covering one 256-byte row; lane l16 reads
        // the stored chunk that holds logical chunk l16), 8 rows per half-warp in flight
        const int hw = tid >> 4, l16 = tid & 15;
        const float4 qa = reinterpret_cast<const float4*>(s_qbar)[l16 * 2];
        const float4 qb4 = reinterpret_cast<const float4*>(s_qbar)[l16 * 2 + 1];
        for (int r0 = 0; r0 < csz; r0 += 8 * (kNT / 16)) {  // CTA-uniform trip count
            float sk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int e = r0 + hw + k * (kNT / 16);
                sk[k] = 0.f;
                if (got && e < csz) {
                    const uint4 w = lds_v4(ringK + (uint32_t)e * 256u + ((uint32_t)swz(crow + e, l16) << 4));
                    float t = qa.x * bf16_lo(w.x);
                    t = fmaf(qa.y, bf16_hi(w.x), t);
                    t = fmaf(qa.z, bf16_lo(w.y), t);
                    t = fmaf(qa.w, bf16_hi(w.y), t);
                    t = fmaf(qb4.x, bf16_lo(w.z), t);
                    t = fmaf(qb4.y, bf16_hi(w.z), t);
                    t = fmaf(qb4.z, bf16_lo(w.w), t);
                    sk[k] = fmaf(qb4.w, bf16_hi(w.w), t);
                }
            }
            __syncwarp();  // all 8 rows' products first, then the reductions
#pragma unroll
            for (int o = 8; o > 0; o >>= 1)
#pragma unroll
                for (int k = 0; k < 8; ++k) sk[k] += __shfl_xor_sync(0xffffffffu, sk[k], o);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int e = r0 + hw + k * (kNT / 16);
                if (e < csz && l16 == 0) s_rkey[e] = orderable(sk[k]);
            }
        }
        if (tid < 4) s_rkey[csz + tid] = 0u;  // pad: never outranks a key
        __syncthreads();
        // comparison rank (ties: lower index), tpe threads per token, 4 keys per load
        const int tpe = csz <= 32 ? 8 : (csz <= 64 ? 4 : (csz <= 128 ? 2 : 1));
        const int e = tid / tpe, sub = tid % tpe;
        int32_t rk = 0;
        if (e < csz) {
            const uint32_t ke = s_rkey[e];
            const uint4* k4 = reinterpret_cast<const uint4*>(s_rkey);
            const int n4 = (csz + 3) >> 2;
            for (int j4 = sub; j4 < n4; j4 += tpe) {
                const uint4 v = k4[j4];
                const int j = 4 * j4;
                rk += (v.x > ke) || (v.x == ke && j < e);
                rk += (v.y > ke) || (v.y == ke && j + 1 < e);
                rk += (v.z > ke) || (v.z == ke && j + 2 < e);
                rk += (v.w > ke) || (v.w == ke && j + 3 < e);
            }
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
            const int32_t y = __shfl_xor_sync(0xffffffffu, rk, o);
            if (o < tpe) rk += y;
        }
        const int32_t sel = (e < csz && sub == 0 && rk < r_part) ? 1 : 0;
        const int32_t pos = block_excl_scan(sel, s_wbuf).x;
        if (sel) {
            s_prow[pos] = e;
            if (sel_out) sel_out[base_p + pos] = ids[crow + e];
        }
        __syncthreads();
        if (kMixed) {
            // the selected rows of a far cut cluster take their fp8 copy's values in place;
            // a near one keeps its bf16 rows (scale 1)
            for (int t = warp; t < r_part; t += kWarps) {  // warp-uniform trip count
                const int er = s_prow[t];
                if (cut_far) {
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        uint2* row = reinterpret_cast<uint2*>(base + Ly.ring + (size_t)part * RB * kPitch +
                                                              (size_t)er * 256);
                        float sc;
                        const uint2 v = fp8_row_values(row[lane], &sc);
                        __syncwarp();
                        row[lane] = v;
                        if (lane == 0) (part ? s_rvs : s_rks)[er] = sc;
                    }
                } else if (lane == 0) {
                    s_rks[er] = 1.f;
                    s_rvs[er] = 1.f;
                }
            }
            __syncthreads();
        }
    } else {
        if (s_wbuf[kWCopy] != 0) {  // cut copies land before the ring is reused
            const bool got = __syncthreads_and(mbar_wait(fbar, 0, a.err) ? 1 : 0) != 0;
            if (!got) {
                s_wbuf[kWBad] = 1;
                mbar_wait(fbar, 0, a.err);  // one more bounded wait for the copies in flight
            }
        }
        // partial tokens of this CTA's share outside the ring path: rows into prow (every CTA
        // of the cluster takes part when the keys go through the global scratch)
        if (r_part > 0 && (coop_cut || p_hi > p_lo)) {
            PartialArgs pa;
            pa.kp = a.kp + (kp_base + crow) * kD;
            pa.gkeys = a.part_scratch ? reinterpret_cast<uint32_t*>(a.part_scratch) +
                                            (int64_t)unit * a.part_ustride
                                      : nullptr;
            pa.qbar = s_qbar;
            pa.pkey = s_pkey;
            pa.hist = s_hist;
            pa.wbuf = s_wbuf;
            pa.prow = s_prow;
            pa.crow = crow;
            pa.csz = csz;
            pa.r_part = r_part;
            pa.p_lo = p_lo;
            pa.p_hi = p_hi;
            pa.rank = (int32_t)rank;
            pa.S = S;
            partial_rows(pa);
        }
    }
    // Attention on tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate), per warp over
    // 16-row tiles of the ring: S^T = K Q^T with the kv rows as M and the G heads as N (<= 8),
    // then O^T += V^T P with the head dimension as M. P is split into bf16 high and low parts
    // (two MMAs) so that the product keeps about 16 bits of the softmax weight.
    const int g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3;
    uint32_t qb[8][2];  // Q^T fragments: Q[head g8][16 s + 2 t4 ...], unscaled bf16
#pragma unroll
    for (int s8 = 0; s8 < 8; ++s8) {
        qb[s8][0] = g8 < G ? *reinterpret_cast<const uint32_t*>(s_qh + g8 * kD + 16 * s8 + 2 * t4) : 0u;
        qb[s8][1] = g8 < G ? *reinterpret_cast<const uint32_t*>(s_qh + g8 * kD + 16 * s8 + 2 * t4 + 8) : 0u;
    }
    float oacc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
    float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};  // heads 2 t4, 2 t4 + 1
    uint16_t* pw = s_pbuf + warp * 256;  // [2][8 heads][16 rows] bf16 (high, low)
    const float qscale = kLog2e * rsqrtf((float)kD);
    // rows: ring row of tile row t is pos[t] (pos != nullptr) or p0 + t
    auto attend = [&](int p0, int n, const int32_t* pos) {
        // logical 16-byte chunk j of ring row p (a 256-byte store row), whose chunk key is key
        auto addr = [&](uint32_t rbase, int p, int key, int j) {
            return rbase + (uint32_t)p * kPitch + ((uint32_t)(j ^ key) << 4);
        };
        const int n_tiles = (n + 15) >> 4;
        for (int tile = warp; tile < n_tiles; tile += kWarps) {
            const int r0 = tile * 16;
            int tk = r0 + (mi & 1) * 8 + (lane & 7);  // K tile row this lane addresses
            int tv = r0 + (mi >> 1) * 8 + (lane & 7); // V tile row this lane addresses
            if (tk >= n) tk = r0;                     // a valid row; masked below
            if (tv >= n) tv = r0;
            const int pk = pos ? pos[tk] : p0 + tk;
            const int pv = pos ? pos[tv] : p0 + tv;
            const int kk = s_key8[pk], kv = s_key8[pv];
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(addr(ringK, pk, kk, 2 * s8 + (mi >> 1)), a0, a1, a2, a3);
                mma_bf16_16816((s8 & 1) ? sb : sa, a0, a1, a2, a3, qb[s8][0], qb[s8][1]);
            }
            // S^T: [0], [1] = row g8, heads 2 t4, 2 t4 + 1; [2], [3] = row g8 + 8
            const bool v0 = r0 + g8 < n, v1 = r0 + g8 + 8 < n;
            // per-row scales of the fp8 copy (1 for bf16 rows)
            float ksa = 1.f, ksb = 1.f, vsa = 1.f, vsb = 1.f;
            if (kMixed) {
                const int ta = v0 ? r0 + g8 : r0, tb = v1 ? r0 + g8 + 8 : r0;
                const int pa = pos ? pos[ta] : p0 + ta, pb = pos ? pos[tb] : p0 + tb;
                ksa = s_rks[pa];
                ksb = s_rks[pb];
                vsa = s_rvs[pa];
                vsb = s_rvs[pb];
            }
            float pr[4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float z0 = v0 ? ((sa[hh] + sb[hh]) * ksa) * qscale : -INFINITY;
                const float z1 = v1 ? ((sa[2 + hh] + sb[2 + hh]) * ksb) * qscale : -INFINITY;
                float mx = fmaxf(z0, z1);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float mn = fmaxf(m2[hh], mx);  // finite: row g8 = 0 of a tile is valid
                const float corr = m2[hh] == -INFINITY ? 0.f : exp2f(m2[hh] - mn);
                pr[hh] = v0 ? exp2f(z0 - mn) : 0.f;
                pr[2 + hh] = v1 ? exp2f(z1 - mn) : 0.f;
                l2[hh] = l2[hh] * corr + pr[hh] + pr[2 + hh];
                m2[hh] = mn;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    oacc[mt][hh] *= corr;
                    oacc[mt][2 + hh] *= corr;
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hd = 2 * t4 + (e & 1), rr = g8 + (e >> 1) * 8;
                const float pv_ = kMixed ? pr[e] * ((e & 2) ? vsb : vsa) : pr[e];  // weight of V
                const __nv_bfloat16 hi_ = __float2bfloat16_rn(pv_);
                const __nv_bfloat16 lo_ = __float2bfloat16_rn(pv_ - __bfloat162float(hi_));
                pw[hd * 16 + rr] = __bfloat16_as_ushort(hi_);
                pw[128 + hd * 16 + rr] = __bfloat16_as_ushort(lo_);
            }
            __syncwarp();
            // P fragments (k = tile rows, n = heads): [r = 2 t4 (+8) ...][h = g8]
            const uint32_t ph0 = *reinterpret_cast<const uint32_t*>(pw + g8 * 16 + 2 * t4);
            const uint32_t ph1 = *reinterpret_cast<const uint32_t*>(pw + g8 * 16 + 2 * t4 + 8);
            const uint32_t pl0 = *reinterpret_cast<const uint32_t*>(pw + 128 + g8 * 16 + 2 * t4);
            const uint32_t pl1 = *reinterpret_cast<const uint32_t*>(pw + 128 + g8 * 16 + 2 * t4 + 8);
            __syncwarp();
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4_trans(addr(ringV, pv, kv, 2 * mt + (mi & 1)), a0, a1, a2, a3);
                mma_bf16_16816(oacc[mt], a0, a1, a2, a3, ph0, ph1);
                mma_bf16_16816(oacc[mt], a0, a1, a2, a3, pl0, pl1);
            }
        }
    };

    // ---- attention, chunk by chunk: the resident cut cluster first (its selected rows listed
    // in prow), as chunk -1; then the streamed rows through the ring, two chunks in flight.
    // One call site for each of issue and attend keeps the code small.
    int next = 0;  // chunks issued
    for (int ch = resident ? -1 : 0; ch < n_chunks; ++ch) {  // CTA-uniform trip count
        int pb0 = 0, n = r_part;
        const int32_t* pos = s_prow;
        if (ch >= 0) {
            while (next < n_chunks && next <= ch + 1) {
                // the slot (or, after the resident chunk, the ring) is no longer read
                if (next >= 2 || (resident && next == 0)) __syncthreads();
                issue(next);
                ++next;
            }
            if (!mbar_wait(rbar + (ch & 1), (uint32_t)(ch >> 1) & 1u, a.err)) s_wbuf[kWBad] = 1;
            const int32_t c0 = lo + ch * chunk;
            n = (s_hi - c0) < chunk ? (s_hi - c0) : chunk;
            pb0 = n_chunks == 1 ? 0 : (ch & 1) * chunk;
            pos = nullptr;
            if (kMixed) {
                __syncthreads();  // rsrc and the scales of the chunk
                convert_far(pb0, n);
                __syncthreads();
            }
        }
        if (s_wbuf[kWBad] == 0) attend(pb0, n, pos);
    }

    // ---------------------------------------------------------------- phase 5: combine
    // per-warp state: l summed over the 8 row groups of the tiles
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], 4);
        l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], 8);
        l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], 16);
    }
    __syncthreads();  // the ring is no longer read: wcomb reuses it
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int hd = 2 * t4 + hh;
        if (hd < G) {
            float* w = s_wcomb + (warp * G + hd) * kCombStride;
            if (g8 == 0) {
                w[128] = m2[hh];
                w[129] = l2[hh];
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                w[16 * mt + g8] = oacc[mt][hh];
                w[16 * mt + g8 + 8] = oacc[mt][2 + hh];
            }
        }
    }
    __syncthreads();
    // per-head merge scales of the 8 warps, computed once
    float* wsc = s_scl;                     // [kWarps][G]
    float* rsc = s_scl + kWarps * G;        // [S][G]
    float* sums = s_scl + (kWarps + S) * G; // [G] max, [G] sum
    // thread (g, w) in groups of 8 lanes: warp w's state for head g
    static_assert(kWarps == 8, "the merge below maps one lane per warp in groups of 8");
    if (tid < 8 * G) {
        // lanes of this warp taking part: 8 per head, heads in order (groups stay aligned)
        const int active = min(32, 8 * G - 32 * warp);
        const uint32_t gmask = active >= 32 ? 0xffffffffu : ((1u << active) - 1u);
        const int g = tid >> 3, w = tid & 7;
        const float mw = s_wcomb[(w * G + g) * kCombStride + 128];
        float mx = mw;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, o));
        const float sc = mw == -INFINITY ? 0.f : exp2f(mw - mx);
        wsc[w * G + g] = sc;
        float l = s_wcomb[(w * G + g) * kCombStride + 129] * sc;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) l += __shfl_xor_sync(gmask, l, o);
        if (w == 0) {
            sums[g] = mx;
            sums[G + g] = l;
        }
    }
    __syncthreads();
    // warps -> CTA partial: CTA 0 keeps its own, the others store theirs into CTA 0's combine
    // buffer (16 bytes per asynchronous store, counted on CTA 0's mbarrier obar)
    {
        const uint32_t dst0 = map_shared_rank(smem_u32(s_ccomb), 0);
        const uint32_t bar0 = map_shared_rank(smem_u32(obar), 0);
        static_assert(kCombStride % 4 == 0, "partials move in 16-byte pieces");
        for (int t = tid; t < G * (kCombStride / 4); t += kNT) {
            const int g = t / (kCombStride / 4), e0 = 4 * (t % (kCombStride / 4));
            float v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = e0 + q;
                if (e == 128) {
                    v[q] = sums[g];
                } else if (e == 129) {
                    v[q] = sums[G + g];
                } else if (e > 129) {
                    v[q] = 0.f;
                } else {
                    float x = 0.f;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w)
                        x = fmaf(s_wcomb[(w * G + g) * kCombStride + e], wsc[w * G + g], x);
                    v[q] = x;
                }
            }
            const int off = (g * kCombStride + e0);  // rank 0's rows come first
            if (rank == 0)
                *reinterpret_cast<float4*>(s_ccomb + off) = make_float4(v[0], v[1], v[2], v[3]);
            else
                st_async_v4_u32(dst0 + (uint32_t)((rank * G * kCombStride + off) * 4), __float_as_uint(v[0]),
                                __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]), bar0);
        }
    }
    if (rank == 0) {
        // the others' partials (warp 0 waits, as for the scores); CTA 0's own
        if (warp == 0) (void)mbar_wait_cluster(obar, 0, a.err);
        __syncthreads();
        if (warp != 0) (void)mbar_try_wait_cluster(obar, 0);
        // thread (g, r) in groups of S lanes (S is a power of two <= 16)
        if (tid < S * G) {
            const int active = min(32, S * G - 32 * warp);
            const uint32_t gmask = active >= 32 ? 0xffffffffu : ((1u << active) - 1u);
            const int g = tid / S, r = tid % S;
            const float mr = s_ccomb[(r * G + g) * kCombStride + 128];
            float mx = mr;
            for (int o = S >> 1; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, o));
            const float sc = mr == -INFINITY ? 0.f : exp2f(mr - mx);
            rsc[r * G + g] = sc;
            float l = s_ccomb[(r * G + g) * kCombStride + 129] * sc;
            for (int o = S >> 1; o > 0; o >>= 1) l += __shfl_xor_sync(gmask, l, o);
            if (r == 0) sums[G + g] = 1.f / l;
        }
        __syncthreads();
        float* o = a.out + ((int64_t)b * a.Hkv * G + (int64_t)h * G) * kD;
        for (int t = tid; t < G * kD; t += kNT) {
            const int g = t / kD, d = t % kD;
            float num = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r)
                if (r < S) num = fmaf(s_ccomb[(r * G + g) * kCombStride + d], rsc[r * G + g], num);
            o[t] = num * sums[G + g];
        }
        if (a.sel_count && tid == 0) a.sel_count[unit] = (int32_t)T;
    }
    if (sel_out && rank == (uint32_t)(S - 1)) {
        for (int32_t i = T + tid; i < a.budget; i += kNT) sel_out[i] = -1;
    }
    if (P.hold) {  // the cluster's CTAs leave together
        cluster_arrive_relaxed();
        cluster_wait_acquire();
    }
}

// Rows of partial tokens one CTA may own: twice the even share of the budget. The dedicated
// partial CTA is used only when the partial fill fits it; otherwise the even split applies,
// whose share is at most budget / S + 1.
int32_t prow_capacity(int budget, int S) { return (int32_t)(2 * ((int64_t)budget / S) + 2); }

struct Plan {
    Params p{};
    size_t smem = 0;
};

// Clusters of S CTAs with `smem` bytes each that can be resident at once (0 when none). Raises
// the kernel's shared-memory limit and allows 16-CTA clusters as needed.
int max_active_clusters(void (*kern)(DecodeArgs, Params), int S, size_t smem, size_t* smem_set,
                        bool* nonportable_set, int* nclusters) {
    *nclusters = 0;
    if (smem > *smem_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "select_attend: set smem");
        *smem_set = smem;
    }
    if (S > 8 && !*nonportable_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return cuda_fail(e, "select_attend: non-portable cluster");
        *nonportable_set = true;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(S * 64));
    cfg.blockDim = dim3(kNT);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaOccupancyMaxActiveClusters(nclusters, kern, &cfg);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        *nclusters = 0;
    }
    return CKV_OK;
}

// Ring rows for a cluster of S CTAs: one CTA's even share of the budget (plus the cut
// cluster's usual size) in one chunk, at least 128 and at most 256 rows, in steps of 16.
int ring_rows(int S, int budget) {
    const int64_t share = (int64_t)budget / (S > 1 ? S - 1 : 1) + 2;
    int64_t rb = ((share + 15) / 16) * 16;
    if (rb < 128) rb = 128;  // also holds most cut clusters whole
    if (rb > 256) rb = 256;
    return (int)rb;
}

// One launch plan per (device, units, C, budget), found once. The cluster size S is the
// largest power of two <= 16 (and <= 64 / G, which bounds CTA 0's combine buffer) whose
// U * S CTAs take at most half of the SMs when the units are few (U * 16 <= SMs), so that the
// next launch's CTAs, started early by programmatic dependent launch, find SMs of their own;
// with more units, at most two CTAs per SM (then the layout must fit two per SM); with more
// units than that, S = 1. The ring takes one CTA's share of the budget, reduced in steps of
// 16 rows while the launch does not fit.
template <int G, bool kPerHead, bool kMixed>
int plan_for(const DecodeArgs& a, int num_sms, Plan* out) {
    static std::mutex mtx;
    static std::map<std::tuple<int, int, int, int>, Plan> cache;
    // kernel attributes are set per device: what has been set, by device
    static std::map<int, size_t> smem_set_by_dev;
    static std::map<int, bool> nonportable_set_by_dev;
    int dev = 0;
    cudaGetDevice(&dev);
    const int U = a.B * a.Hkv;
    const auto key = std::make_tuple(dev, U, a.C, a.budget);
    std::lock_guard<std::mutex> lock(mtx);
    size_t& smem_set = smem_set_by_dev[dev];
    bool& nonportable_set = nonportable_set_by_dev[dev];
    auto it = cache.find(key);
    if (it != cache.end()) {
        *out = it->second;
        return CKV_OK;
    }
    auto kern = select_attend_kernel<G, kPerHead, kMixed>;
    Plan best{};
    const int64_t sm_cap = (int64_t)U * 16 <= num_sms ? num_sms / 2 : 2 * (int64_t)num_sms;
    constexpr uint32_t kTwoPerSm = 113 * 1024;  // two CTAs share one SM's 228 KB
    for (int S = 16; S >= 1 && best.p.S == 0; S /= 2) {
        if (S > 1 && (S * G > 64 || (int64_t)U * S > sm_cap)) continue;
        for (int RB = ring_rows(S, a.budget); RB >= 64 && best.p.S == 0; RB -= 16) {
            const int pc = prow_capacity(a.budget, S);
            const Layout L = make_layout(G, S, a.C, RB, pc, kMixed);
            if (L.total > 227 * 1024) continue;
            // more CTAs than SMs: the launch is one wave only with two CTAs per SM
            if (S > 1 && (int64_t)U * S > num_sms && L.total > kTwoPerSm) continue;
            int nclusters = 0;
            const int rc = max_active_clusters(kern, S, L.total, &smem_set, &nonportable_set, &nclusters);
            if (rc != CKV_OK) return rc;
            if (nclusters <= 0) continue;
            // Two CTAs per SM: when CTAs leave ahead of their cluster's CTA 0, the next launch
            // places clusters into the gaps piecemeal, and then one of its clusters can wait for
            // room until a whole cluster of that launch ends (measured: 18 -> 26 us per launch
            // at 32 units, back to back). There the CTAs of a cluster leave together.
            const int32_t hold = (S > 1 && (int64_t)U * S > num_sms) ? 1 : 0;
            best.p = Params{S, RB, pc, hold};
            best.smem = L.total;
        }
    }
    if (best.p.S == 0) {
        set_error("select_and_attend: no launch shape fits (budget or C too large for shared memory)");
        return CKV_ECAPACITY;
    }
    cache[key] = best;
    *out = best;
    return CKV_OK;
}

template <int G, bool kPerHead = false, bool kMixed = false>
int launch_g(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    Plan plan;
    int rc = plan_for<G, kPerHead, kMixed>(a, num_sms, &plan);
    if (rc != CKV_OK) return rc;
    const int U = a.B * a.Hkv;
    const int S = plan.p.S;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(U * S));
    cfg.blockDim = dim3(kNT);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[3];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = (unsigned)S;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[1].val.programmaticStreamSerializationAllowed = 1;
    attrs[2].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;  // one CTA per SM
    attrs[2].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
    cfg.attrs = attrs;
    cfg.numAttrs = 3;
    cudaError_t e = cudaLaunchKernelEx(&cfg, select_attend_kernel<G, kPerHead, kMixed>, a, plan.p);
    if (e != cudaSuccess) return cuda_fail(e, "select_attend: launch");
    return CKV_OK;
}

}  // namespace

int launch_select_attend_per_head(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    if (a.G != 1) {
        set_error("select_and_attend_per_head: internal group size must be 1");
        return CKV_EINVAL;
    }
    return launch_g<1, true>(a, num_sms, s);
}

int launch_select_attend_mixed(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    switch (a.G) {
        case 1: return launch_g<1, false, true>(a, num_sms, s);
        case 2: return launch_g<2, false, true>(a, num_sms, s);
        case 3: return launch_g<3, false, true>(a, num_sms, s);
        case 4: return launch_g<4, false, true>(a, num_sms, s);
        case 5: return launch_g<5, false, true>(a, num_sms, s);
        case 6: return launch_g<6, false, true>(a, num_sms, s);
        case 7: return launch_g<7, false, true>(a, num_sms, s);
        case 8: return launch_g<8, false, true>(a, num_sms, s);
        default: set_error("select_and_attend_mixed: group size must be 1..8"); return CKV_EINVAL;
    }
}

int launch_select_attend(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    switch (a.G) {
        case 1: return launch_g<1>(a, num_sms, s);
        case 2: return launch_g<2>(a, num_sms, s);
        case 3: return launch_g<3>(a, num_sms, s);
        case 4: return launch_g<4>(a, num_sms, s);
        case 5: return launch_g<5>(a, num_sms, s);
        case 6: return launch_g<6>(a, num_sms, s);
        case 7: return launch_g<7>(a, num_sms, s);
        case 8: return launch_g<8>(a, num_sms, s);
        default: set_error("select_and_attend: group size must be 1..8"); return CKV_EINVAL;
    }
}

}  // namespace ckv
