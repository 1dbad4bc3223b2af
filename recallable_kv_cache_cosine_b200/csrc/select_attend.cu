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
// One unit (sequence b, KV head h) is served by a thread-block cluster of S CTAs:
//   1. each CTA scores a slice of the C centroids (fp32; a quarter-warp per centroid) and
//      broadcasts (score, size) to every CTA of the cluster through distributed shared memory;
//   2. each CTA ranks its slice against all C scores (8 threads per cluster). The rank and
//      the number of tokens ranked before each cluster give the whole clusters and the cut
//      cluster without a sort. The whole clusters' (prefix, first row) are broadcast,
//      indexed by rank;
//   3. the selected rows form one index space: sinks, pending, whole clusters by rank, then
//      the partial tokens of the cut cluster. With a partial fill and S > 1, CTA S-1 takes
//      exactly the partial tokens and ranks the cut cluster's tokens by qbar . k (comparison
//      rank for small clusters, radix select for large ones); the other CTAs split the rest;
//   4. half-warps stream their rows with 16-byte loads, 4 rows per group, and run one online
//      softmax update per group for the G query heads;
//   5. the CTA partials (max, sum, accumulator) are merged in CTA 0 through distributed
//      shared memory, which writes the fp32 output.
// The kernel triggers programmatic dependent launch at entry and prefetches its centroid
// slice into L2 before waiting on the previous grid.
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
constexpr int kRowChunk = 256;    // rows per gather chunk
constexpr int kPartCap = 4096;    // cut-cluster tokens ranked in shared memory
constexpr float kLog2e = 1.4426950408889634f;

struct CutInfo {
    int32_t c, prefix, rank, row, size;
};

CKV_DEV uint32_t orderable(float f) {
    f = f + 0.0f;  // -0 -> +0
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// qbar . k over one half (64 dims) of a 256-byte key row: 8 independent 16-byte loads, then
// fp32 FMAs in dimension order.
CKV_DEV float half_row_dot(const uint16_t* row, int half, const float* qbar) {
    uint4 w[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) w[t] = ldg_nc_v4(row + 64 * half + 8 * t);
    const float4* q4 = reinterpret_cast<const float4*>(qbar + 64 * half);
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const float4 qa = q4[2 * t], qb = q4[2 * t + 1];
        s = fmaf(qa.x, bf16_lo(w[t].x), s);
        s = fmaf(qa.y, bf16_hi(w[t].x), s);
        s = fmaf(qa.z, bf16_lo(w[t].y), s);
        s = fmaf(qa.w, bf16_hi(w[t].y), s);
        s = fmaf(qb.x, bf16_lo(w[t].z), s);
        s = fmaf(qb.y, bf16_hi(w[t].z), s);
        s = fmaf(qb.z, bf16_lo(w[t].w), s);
        s = fmaf(qb.w, bf16_hi(w[t].w), s);
    }
    return s;
}

// Exclusive block scan of one int per thread. `tot` receives the block total.
CKV_DEV int32_t block_excl_scan(int32_t v, int32_t* wbuf, int32_t* tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wbuf[warp] = incl;
    __syncthreads();
    int32_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int32_t x = wbuf[w];
        if (w < warp) before += x;
        total += x;
    }
    __syncthreads();
    *tot = total;
    return before + incl - v;
}

struct Smem {
    float* qg;        // [G][128], scaled by log2(e)/sqrt(128)
    float* qbar;      // [128]
    int2* scsz;       // [C] (score bits, size) of every cluster
    int32_t* crow;    // [C] first store row of the clusters this CTA scored
    int32_t* spre;    // [C + 1] prefix of the whole cluster of rank k
    int32_t* srow;    // [C + 1] first store row of the whole cluster of rank k
    uint32_t* pkey;   // [kPartCap] cut-cluster token keys
    int32_t* prow;    // [prow_cap] partial rows of this CTA's share
    int32_t* rows;    // [kRowChunk] row list of the current chunk
    int32_t* wbuf;    // [64] scan / misc scratch
    float* wcomb;     // [kWarps][G][130]
    float* scl;       // [(kWarps + S) * G] merge scales, then [2 * G] sums
    float* ccomb;     // [S][G][130] (filled in CTA 0)
    CutInfo* cut;
};

template <int G>
__global__ void __launch_bounds__(kNT, (G <= 4) ? 2 : 1)
    select_attend_kernel(const DecodeArgs a, int32_t S, int32_t prow_cap) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int C = a.C;
    const uint32_t rank = cluster_ctarank();
    const int unit = blockIdx.x / S;
    const int b = unit / a.Hkv, h = unit % a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    Smem sm;
    {
        uint8_t* p = smem_raw;
        auto take = [&](size_t bytes) {
            uint8_t* r = p;
            p += (bytes + 15) & ~(size_t)15;
            return r;
        };
        sm.qg = (float*)take(sizeof(float) * G * kD);
        sm.qbar = (float*)take(sizeof(float) * kD);
        sm.scsz = (int2*)take(sizeof(int2) * C);
        sm.crow = (int32_t*)take(sizeof(int32_t) * C);
        sm.spre = (int32_t*)take(sizeof(int32_t) * (C + 1));
        sm.srow = (int32_t*)take(sizeof(int32_t) * (C + 1));
        sm.pkey = (uint32_t*)take(sizeof(uint32_t) * kPartCap);
        sm.prow = (int32_t*)take(sizeof(int32_t) * prow_cap);
        sm.rows = (int32_t*)take(sizeof(int32_t) * kRowChunk);
        sm.wbuf = (int32_t*)take(sizeof(int32_t) * 64);
        sm.wcomb = (float*)take(sizeof(float) * kWarps * G * 130);
        sm.scl = (float*)take(sizeof(float) * ((kWarps + S) * G + 2 * G));
        sm.ccomb = (float*)take(sizeof(float) * S * G * 130);
        sm.cut = (CutInfo*)take(sizeof(CutInfo));
    }

    const int64_t kp_base = (int64_t)unit * a.kp_ustride;
    const int64_t sp_base = (int64_t)unit * a.sp_ustride;
    const int32_t* off = a.offsets + (int64_t)unit * a.off_ustride;
    const float* mu = a.mu + (int64_t)unit * a.mu_ustride * kD;
    const int c_begin = (int)((int64_t)C * rank / S);
    const int c_end = (int)((int64_t)C * (rank + 1) / S);

    // ---------------------------------------------------------------- phase 0
    pdl_launch_dependents();
    if (threadIdx.x == 0 && c_end > c_begin) {
        prefetch_l2_bulk(mu + (int64_t)c_begin * kD, (uint32_t)(c_end - c_begin) * kD * 4);
    }
    cluster_arrive_relaxed();
    pdl_wait();

    // ---------------------------------------------------------------- phase 1: scores
    // A quarter-warp (8 lanes) per centroid, 16 dimensions per lane: 32 centroids per CTA
    // per round. The first round's centroid and offset loads are issued before the query
    // loads, so both share one memory round trip.
    const int32_t pend = a.pending;
    const int32_t R = a.budget - a.n_sink - pend;  // >= 0 (host-checked)
    const int q8 = lane >> 3, l8 = lane & 7;
    constexpr int kPerRound = kWarps * 4;
    float4 mv[4];
    int32_t c_lo_row = 0, c_hi_row = 0;
    auto load_centroid = [&](int c) {
        if (c < c_end) {
            const float4* row = reinterpret_cast<const float4*>(mu + (int64_t)c * kD) + l8 * 4;
#pragma unroll
            for (int t = 0; t < 4; ++t) mv[t] = row[t];
            c_lo_row = off[c];
            c_hi_row = off[c + 1];
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) mv[t] = make_float4(0.f, 0.f, 0.f, 0.f);
            c_lo_row = c_hi_row = 0;
        }
    };
    load_centroid(c_begin + warp * 4 + q8);
    {
        const uint16_t* q = a.q + ((int64_t)b * a.Hkv * G + (int64_t)h * G) * kD;
        const float scale = kLog2e * rsqrtf((float)kD);
        for (int i = threadIdx.x; i < kD; i += kNT) {
            float s = 0.f;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float x = __uint_as_float((uint32_t)q[g * kD + i] << 16);
                s += x;
                sm.qg[g * kD + i] = x * scale;
            }
            sm.qbar[i] = s;
        }
    }
    if (threadIdx.x == 0) sm.cut->c = -1;
    __syncthreads();
    cluster_wait_acquire();  // every CTA of the cluster is running
    for (int r0 = 0; r0 < c_end - c_begin; r0 += kPerRound) {
        const int c = c_begin + r0 + warp * 4 + q8;
        if (r0 > 0) load_centroid(c);
        const float4* qb4 = reinterpret_cast<const float4*>(sm.qbar) + l8 * 4;
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float4 qv4 = qb4[t];
            s += qv4.x * mv[t].x + qv4.y * mv[t].y + qv4.z * mv[t].z + qv4.w * mv[t].w;
        }
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if (c < c_end) {
            if (l8 == 0) sm.crow[c] = c_lo_row;
            const uint32_t sz = (uint32_t)(c_hi_row - c_lo_row);
            for (int r = l8; r < S; r += 8) {
                const uint32_t dst = map_shared_rank(smem_u32(&sm.scsz[c]), r);
                asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(dst),
                             "r"(__float_as_uint(s)), "r"(sz)
                             : "memory");
            }
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();

    // ---------------------------------------------------------------- phase 2: ranks
    // 8 threads per cluster of this CTA's slice; each compares 1/8 of all C clusters.
    for (int c0 = c_begin; c0 < c_end; c0 += kNT / 8) {
        const int c = c0 + (threadIdx.x >> 3);
        const int sub = threadIdx.x & 7;
        float s = 0.f;
        int32_t size = 0;
        if (c < c_end) {
            const int2 me = sm.scsz[c];
            s = __int_as_float(me.x);
            size = me.y;
        }
        int32_t rk = 0, pre = 0;
#pragma unroll 4
        for (int j = sub; j < C; j += 8) {
            const int2 o = sm.scsz[j];
            const float t = __int_as_float(o.x);
            const bool before = (t > s) || (t == s && j < c);
            rk += before ? 1 : 0;
            pre += before ? o.y : 0;
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
            rk += __shfl_xor_sync(0xffffffffu, rk, o);
            pre += __shfl_xor_sync(0xffffffffu, pre, o);
        }
        if (c < c_end) {
            if (pre + size <= R) {  // whole cluster
                const int32_t row = sm.crow[c];
                for (int r = sub; r < S; r += 8) {
                    st_cluster_u32(map_shared_rank(smem_u32(&sm.spre[rk]), r), (uint32_t)pre);
                    st_cluster_u32(map_shared_rank(smem_u32(&sm.srow[rk]), r), (uint32_t)row);
                }
            } else if (pre <= R) {  // the cut cluster (R < pre + size)
                const int32_t row = sm.crow[c];
                for (int r = sub; r < S; r += 8) {
                    const uint32_t base = map_shared_rank(smem_u32(sm.cut), r);
                    st_cluster_u32(base + 0, (uint32_t)c);
                    st_cluster_u32(base + 4, (uint32_t)pre);
                    st_cluster_u32(base + 8, (uint32_t)rk);
                    st_cluster_u32(base + 12, (uint32_t)row);
                    st_cluster_u32(base + 16, (uint32_t)size);
                }
            }
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();

    const bool has_cut = sm.cut->c >= 0;
    const int32_t n_whole = has_cut ? sm.cut->rank : C;
    const int64_t W = has_cut ? (int64_t)sm.cut->prefix : a.m;
    const int32_t r_part = has_cut ? (int32_t)(R - W) : 0;
    const int64_t base_w = (int64_t)a.n_sink + pend;
    const int64_t base_p = base_w + W;
    const int64_t T = base_p + r_part;
    // Work split of the selection index space [0, T). With a partial fill, CTA S-1 takes
    // exactly the partial tokens (it also ranks them) and the other CTAs split the rest.
    int64_t lo, hi;
    if (r_part > 0 && S > 1 && r_part <= prow_cap) {
        if ((int)rank == S - 1) {
            lo = base_p;
            hi = T;
        } else {
            lo = base_p * rank / (S - 1);
            hi = base_p * (rank + 1) / (S - 1);
        }
    } else {
        lo = T * rank / S;
        hi = T * (rank + 1) / S;
    }

    // ---------------------------------------------------------------- phase 3: partial
    // This CTA's share of the partial tokens: positions [p_lo, p_hi) in store order.
    const int64_t p_lo = lo > base_p ? lo - base_p : 0;
    const int64_t p_hi = hi > base_p ? hi - base_p : 0;
    const int32_t csz = has_cut ? sm.cut->size : 0;
    const bool big_cut = csz > kPartCap;
    uint32_t* gkeys = a.part_scratch ? reinterpret_cast<uint32_t*>(a.part_scratch) +
                                           (int64_t)unit * a.part_ustride
                                     : nullptr;
    auto score_keys = [&](int64_t k0, int64_t k1, uint32_t* dst, int32_t crow) {
        // two threads per row, one memory round trip per pass
        for (int64_t i0 = k0; i0 < k1; i0 += kNT / 2) {
            const int64_t i = i0 + (threadIdx.x >> 1);
            const int half = threadIdx.x & 1;
            float s = 0.f;
            if (i < k1) s = half_row_dot(a.kp + (kp_base + crow + i) * kD, half, sm.qbar);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            if (i < k1 && half == 0) dst[i] = orderable(s);
        }
    };
    if (r_part > 0 && big_cut) {
        // Keys of a large cut cluster are written once, split across the cluster's CTAs.
        const int64_t k0 = (int64_t)csz * rank / S, k1 = (int64_t)csz * (rank + 1) / S;
        score_keys(k0, k1, gkeys, sm.cut->row);
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    if (r_part > 0 && p_hi > p_lo) {
        const int32_t crow = sm.cut->row;
        const uint32_t* skeys = sm.pkey;
        auto key_at = [&](int i) -> uint32_t { return big_cut ? __ldcg(gkeys + i) : skeys[i]; };
        if (!big_cut) {
            score_keys(0, csz, sm.pkey, crow);
            if (threadIdx.x < 4) sm.pkey[csz + threadIdx.x] = 0u;  // pad: never outranks a key
        }
        __syncthreads();
        if (!big_cut && csz <= kNT) {
            // comparison rank (ties: lower index), tpe threads per token, 4 keys per load
            const int tpe = csz <= 32 ? 8 : (csz <= 64 ? 4 : (csz <= 128 ? 2 : 1));
            const int e = threadIdx.x / tpe, sub = threadIdx.x % tpe;
            int32_t rk = 0;
            if (e < csz) {
                const uint32_t ke = sm.pkey[e];
                const uint4* k4 = reinterpret_cast<const uint4*>(sm.pkey);
                const int n4 = (csz + 3) >> 2;
#pragma unroll 4
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
            int32_t tot;
            const int32_t pos = block_excl_scan(sel, sm.wbuf, &tot);
            if (sel && pos >= p_lo && pos < p_hi) sm.prow[pos - p_lo] = crow + e;
        } else {
            // radix select over 4 digits of 8 bits, most significant first: the threshold key
            // theta and `need` = how many keys equal to theta are taken (the lowest-index
            // ones), so that exactly r_part tokens are selected.
            uint32_t prefix = 0, mask = 0;
            int32_t need = r_part;
            int32_t* hist = (int32_t*)sm.wcomb;  // 256 counters (scratch, unused until phase 5)
            for (int pass = 0; pass < 4; ++pass) {
                const int shift = 24 - 8 * pass;
                for (int i = threadIdx.x; i < 256; i += kNT) hist[i] = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < csz; i += kNT) {
                    const uint32_t k = key_at(i);
                    if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
                }
                __syncthreads();
                if (warp == 0) {
                    // lane l owns bins 255-8l .. 248-8l (descending)
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
                    int32_t above = incl - tot;  // keys in higher bins
                    if (above < need && need <= incl) {
                        for (int e = 0; e < 8; ++e) {
                            if (above + cnt[e] >= need) {
                                sm.wbuf[32] = 255 - 8 * lane - e;
                                sm.wbuf[33] = above;
                                break;
                            }
                            above += cnt[e];
                        }
                    }
                }
                __syncthreads();
                const uint32_t d = (uint32_t)sm.wbuf[32];
                need -= sm.wbuf[33];
                prefix |= d << shift;
                mask |= 255u << shift;
                __syncthreads();
            }
            const uint32_t theta = prefix;
            int32_t eq_run = 0, sel_run = 0;
            for (int base = 0; base < csz; base += kNT) {
                const int i = base + threadIdx.x;
                const uint32_t k = i < csz ? key_at(i) : 0u;
                const int32_t eq = (i < csz && k == theta) ? 1 : 0;
                int32_t eq_tot;
                const int32_t eq_before = eq_run + block_excl_scan(eq, sm.wbuf, &eq_tot);
                const int32_t sel = (i < csz) && (k > theta || (eq && eq_before < need));
                int32_t sel_tot;
                const int32_t pos = sel_run + block_excl_scan(sel, sm.wbuf, &sel_tot);
                if (sel && pos >= p_lo && pos < p_hi) sm.prow[pos - p_lo] = crow + i;
                eq_run += eq_tot;
                sel_run += sel_tot;
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- phase 4: gather + attend
    const int hw = threadIdx.x >> 4, l16 = threadIdx.x & 15;
    const float4* qg4 = reinterpret_cast<const float4*>(sm.qg) + l16 * 2;  // this lane's 8 dims
    float mrun[G], lrun[G], acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        mrun[g] = -INFINITY;
        lrun[g] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
    }
    int32_t* sel_out = a.sel_idx ? a.sel_idx + (int64_t)unit * a.budget : nullptr;
    const int32_t* ids = a.ids + kp_base;
    for (int64_t c0 = lo; c0 < hi; c0 += kRowChunk) {
        const int n = (int)((hi - c0) < kRowChunk ? (hi - c0) : kRowChunk);
        if (threadIdx.x < n) {
            const int64_t idx = c0 + threadIdx.x;
            int32_t row, oid;
            if (idx < base_w) {
                row = -1 - (int32_t)idx;  // sink / pending row
                oid = idx < a.n_sink ? (int32_t)idx : (int32_t)(a.m + idx);
            } else if (idx < base_p) {
                const int32_t x = (int32_t)(idx - base_w);
                int lo2 = 0, hi2 = n_whole - 1;  // last k with spre[k] <= x
                while (lo2 < hi2) {
                    const int mid = (lo2 + hi2 + 1) >> 1;
                    if (sm.spre[mid] <= x) lo2 = mid; else hi2 = mid - 1;
                }
                row = sm.srow[lo2] + (x - sm.spre[lo2]);
                oid = sel_out ? ids[row] : 0;
            } else {
                row = sm.prow[idx - base_p - p_lo];
                oid = sel_out ? ids[row] : 0;
            }
            sm.rows[threadIdx.x] = row;
            if (sel_out) sel_out[idx] = oid;
        }
        __syncthreads();
        // The trip count is the same for every thread of the CTA: the full-mask shuffles
        // below need both half-warps of a warp in every iteration.
        for (int j0 = 0; j0 < n; j0 += 4 * (kNT / 16)) {
            uint4 kw[4], vw[4];
            bool valid[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int j = j0 + hw + t * (kNT / 16);
                valid[t] = j < n;
                kw[t] = make_uint4(0u, 0u, 0u, 0u);
                vw[t] = kw[t];
                if (valid[t]) {
                    const int32_t row = sm.rows[j];
                    const uint16_t* kr = row >= 0 ? a.kp + (kp_base + row) * kD
                                                  : a.spk + (sp_base + (-1 - row)) * kD;
                    const uint16_t* vr = row >= 0 ? a.vp + (kp_base + row) * kD
                                                  : a.spv + (sp_base + (-1 - row)) * kD;
                    kw[t] = ldg_nc_v4(kr + l16 * 8);
                    vw[t] = ldg_nc_v4(vr + l16 * 8);
                }
            }
            // logits of the 4 rows for every head (full-mask shuffles: all lanes)
            float z[4][G];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float k0 = bf16_lo(kw[t].x), k1 = bf16_hi(kw[t].x), k2 = bf16_lo(kw[t].y),
                            k3 = bf16_hi(kw[t].y), k4 = bf16_lo(kw[t].z), k5 = bf16_hi(kw[t].z),
                            k6 = bf16_lo(kw[t].w), k7 = bf16_hi(kw[t].w);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 qa = qg4[g * (kD / 4)];
                    const float4 qb = qg4[g * (kD / 4) + 1];
                    float s = qa.x * k0;
                    s = fmaf(qa.y, k1, s);
                    s = fmaf(qa.z, k2, s);
                    s = fmaf(qa.w, k3, s);
                    s = fmaf(qb.x, k4, s);
                    s = fmaf(qb.y, k5, s);
                    s = fmaf(qb.z, k6, s);
                    s = fmaf(qb.w, k7, s);
                    z[t][g] = s;
                }
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1)
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int g = 0; g < G; ++g) z[t][g] += __shfl_xor_sync(0xffffffffu, z[t][g], o);
            if (!valid[0]) continue;  // no row of this group for this half-warp
            // one online-softmax update per head for the whole group
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float mx = mrun[g];
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    if (valid[t]) mx = fmaxf(mx, z[t][g]);
                const float corr = mrun[g] == -INFINITY ? 0.f : exp2f(mrun[g] - mx);
                float p[4];
                float psum = 0.f;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    p[t] = valid[t] ? exp2f(z[t][g] - mx) : 0.f;
                    psum += p[t];
                }
                lrun[g] = lrun[g] * corr + psum;
                mrun[g] = mx;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[g][e] *= corr;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint32_t vv[4] = {vw[t].x, vw[t].y, vw[t].z, vw[t].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[g][2 * e] = fmaf(p[t], bf16_lo(vv[e]), acc[g][2 * e]);
                        acc[g][2 * e + 1] = fmaf(p[t], bf16_hi(vv[e]), acc[g][2 * e + 1]);
                    }
                }
            }
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- phase 5: combine
    // half-warp pair -> warp
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float mo = __shfl_xor_sync(0xffffffffu, mrun[g], 16);
        const float lo_ = __shfl_xor_sync(0xffffffffu, lrun[g], 16);
        const float mn = fmaxf(mrun[g], mo);
        const float ca = mrun[g] == -INFINITY ? 0.f : exp2f(mrun[g] - mn);
        const float cb = mo == -INFINITY ? 0.f : exp2f(mo - mn);
        lrun[g] = lrun[g] * ca + lo_ * cb;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], 16);
            acc[g][e] = acc[g][e] * ca + ao * cb;
        }
        mrun[g] = mn;
    }
    if (lane < 16) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float* w = sm.wcomb + (warp * G + g) * 130;
            if (lane == 0) {
                w[128] = mrun[g];
                w[129] = lrun[g];
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) w[lane * 8 + e] = acc[g][e];
        }
    }
    __syncthreads();
    // per-head merge scales of the 8 warps, computed once
    float* wsc = sm.scl;                     // [kWarps][G]
    float* rsc = sm.scl + kWarps * G;        // [S][G]
    float* sums = sm.scl + (kWarps + S) * G; // [G] max, [G] sum
    // thread (g, w) in groups of 8 lanes: warp w's state for head g
    static_assert(kWarps == 8, "the merge below maps one lane per warp in groups of 8");
    if (threadIdx.x < 8 * G) {
        // lanes of this warp taking part: 8 per head, heads in order (groups stay aligned)
        const int active = min(32, 8 * G - 32 * warp);
        const uint32_t gmask = active >= 32 ? 0xffffffffu : ((1u << active) - 1u);
        const int g = threadIdx.x >> 3, w = threadIdx.x & 7;
        const float mw = sm.wcomb[(w * G + g) * 130 + 128];
        float mx = mw;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, o));
        const float sc = mw == -INFINITY ? 0.f : exp2f(mw - mx);
        wsc[w * G + g] = sc;
        float l = sm.wcomb[(w * G + g) * 130 + 129] * sc;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) l += __shfl_xor_sync(gmask, l, o);
        if (w == 0) {
            sums[g] = mx;
            sums[G + g] = l;
        }
    }
    __syncthreads();
    // warps -> CTA partial, written into CTA 0's combine buffer
    {
        const uint32_t dst0 = map_shared_rank(smem_u32(sm.ccomb), 0);
        for (int t = threadIdx.x; t < G * 130; t += kNT) {
            const int g = t / 130, e = t % 130;
            float v;
            if (e == 128) {
                v = sums[g];
            } else if (e == 129) {
                v = sums[G + g];
            } else {
                v = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) v = fmaf(sm.wcomb[(w * G + g) * 130 + e], wsc[w * G + g], v);
            }
            st_cluster_f32(dst0 + (uint32_t)(((rank * G + g) * 130 + e) * 4), v);
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();
    if (rank == 0) {
        // thread (g, r) in groups of S lanes (S is a power of two <= 16)
        if (threadIdx.x < S * G) {
            const int active = min(32, S * G - 32 * warp);
            const uint32_t gmask = active >= 32 ? 0xffffffffu : ((1u << active) - 1u);
            const int g = threadIdx.x / S, r = threadIdx.x % S;
            const float mr = sm.ccomb[(r * G + g) * 130 + 128];
            float mx = mr;
            for (int o = S >> 1; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, o));
            const float sc = mr == -INFINITY ? 0.f : exp2f(mr - mx);
            rsc[r * G + g] = sc;
            float l = sm.ccomb[(r * G + g) * 130 + 129] * sc;
            for (int o = S >> 1; o > 0; o >>= 1) l += __shfl_xor_sync(gmask, l, o);
            if (r == 0) sums[G + g] = 1.f / l;
        }
        __syncthreads();
        float* o = a.out + ((int64_t)b * a.Hkv * G + (int64_t)h * G) * kD;
        for (int t = threadIdx.x; t < G * kD; t += kNT) {
            const int g = t / kD, d = t % kD;
            float num = 0.f;
            for (int r = 0; r < S; ++r) num = fmaf(sm.ccomb[(r * G + g) * 130 + d], rsc[r * G + g], num);
            o[t] = num * sums[G + g];
        }
        if (a.sel_count && threadIdx.x == 0) a.sel_count[unit] = (int32_t)T;
    }
    if (sel_out && rank == (uint32_t)(S - 1)) {
        for (int64_t i = T + threadIdx.x; i < a.budget; i += kNT) sel_out[i] = -1;
    }
}

// Rows of partial tokens one CTA may own: twice the even share of the budget. The dedicated
// partial CTA is used only when the partial fill fits it; otherwise the even split applies,
// whose share is at most budget / S + 1.
int32_t prow_capacity(int budget, int S) { return (int32_t)(2 * ((int64_t)budget / S) + 2); }

size_t smem_bytes(int G, int S, int C, int budget) {
    const int32_t pc = prow_capacity(budget, S);
    size_t b = 0;
    auto add = [&](size_t x) { b += (x + 15) & ~(size_t)15; };
    add(sizeof(float) * G * kD);
    add(sizeof(float) * kD);
    add(sizeof(int2) * C);
    add(sizeof(int32_t) * C);
    add(sizeof(int32_t) * (C + 1));
    add(sizeof(int32_t) * (C + 1));
    add(sizeof(uint32_t) * kPartCap);
    add(sizeof(int32_t) * pc);
    add(sizeof(int32_t) * kRowChunk);
    add(sizeof(int32_t) * 64);
    add(sizeof(float) * kWarps * G * 130);
    add(sizeof(float) * ((kWarps + S) * G + 2 * G));
    add(sizeof(float) * S * G * 130);
    add(sizeof(CutInfo));
    return b;
}

struct Plan {
    int S = 0;
    size_t smem = 0;
};

// One launch plan per (device, group size, units, C, budget), found once. The cluster size S
// is the largest power of two <= 16 whose clusters for all units are resident at once (one
// wave), with U * S <= 2 * SMs; otherwise the smallest S that fits in shared memory.
template <int G>
int plan_for(const DecodeArgs& a, int num_sms, Plan* out) {
    static std::mutex mtx;
    static std::map<std::tuple<int, int, int, int>, Plan> cache;
    static size_t smem_set = 0;
    static bool nonportable_set = false;
    int dev = 0;
    cudaGetDevice(&dev);
    const int U = a.B * a.Hkv;
    const auto key = std::make_tuple(dev, U, a.C, a.budget);
    std::lock_guard<std::mutex> lock(mtx);
    auto it = cache.find(key);
    if (it != cache.end()) {
        *out = it->second;
        return CKV_OK;
    }
    auto kern = select_attend_kernel<G>;
    Plan best{};
    for (int S = 16; S >= 1; S /= 2) {
        const size_t smem = smem_bytes(G, S, a.C, a.budget);
        if (smem > 227 * 1024) continue;
        if ((int64_t)U * S > 2 * (int64_t)num_sms && S > 1) continue;
        if (smem > smem_set) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return cuda_fail(e, "select_attend: set smem");
            smem_set = smem;
        }
        if (S > 8 && !nonportable_set) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return cuda_fail(e, "select_attend: non-portable cluster");
            nonportable_set = true;
        }
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(U * S));
        cfg.blockDim = dim3(kNT);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        cudaError_t e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            continue;
        }
        if (nclusters <= 0) continue;
        if (best.S == 0) best = Plan{S, smem};  // fallback: fits, maybe several waves
        if (nclusters >= U) {
            best = Plan{S, smem};
            break;
        }
        best = Plan{S, smem};
    }
    if (best.S == 0) {
        set_error("select_and_attend: no launch shape fits (budget or C too large for shared memory)");
        return CKV_ECAPACITY;
    }
    cache[key] = best;
    *out = best;
    return CKV_OK;
}

template <int G>
int launch_g(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    Plan plan;
    int rc = plan_for<G>(a, num_sms, &plan);
    if (rc != CKV_OK) return rc;
    const int U = a.B * a.Hkv;
    const int S = plan.S;
    const int32_t pc = prow_capacity(a.budget, S);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(U * S));
    cfg.blockDim = dim3(kNT);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = (unsigned)S;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, select_attend_kernel<G>, a, (int32_t)S, pc);
    if (e != cudaSuccess) return cuda_fail(e, "select_attend: launch");
    return CKV_OK;
}

}  // namespace

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
