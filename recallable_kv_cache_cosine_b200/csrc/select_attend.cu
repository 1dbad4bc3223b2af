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
//   1. each CTA scores a slice of the C centroids (fp32) and broadcasts (score, size) to every
//      CTA of the cluster through distributed shared memory;
//   2. each CTA ranks its own slice against all C scores, which gives each cluster's rank and
//      the number of tokens ranked before it. Whole clusters and the cut cluster follow
//      without a sort. The whole clusters' (prefix, first row) are broadcast, indexed by rank;
//   3. the selected rows form one index space: sinks, pending, whole clusters by rank, then
//      the partial tokens. CTA r takes an equal share of it. The CTAs whose share reaches
//      the partial tokens rank the cut cluster's tokens by qbar . k (comparison rank for
//      small clusters, radix select for large ones);
//   4. half-warps stream their rows with 16-byte loads and run an online softmax for the
//      G query heads;
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

// Orderable key of qbar . k for one 256-byte key row, computed by one thread: 16 independent
// 16-byte loads, then an fp32 dot product in dimension order.
CKV_DEV uint32_t row_key(const uint16_t* row, const float* qbar) {
    float s = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
    uint4 w[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) w[t] = ldg_nc_v4(row + 64 * half + 8 * t);
#pragma unroll
    for (int t0 = 0; t0 < 8; ++t0) {
        const int t = 8 * half + t0;
        const float4 qa = reinterpret_cast<const float4*>(qbar)[2 * t];
        const float4 qb = reinterpret_cast<const float4*>(qbar)[2 * t + 1];
        s = fmaf(qa.x, bf16_lo(w[t0].x), s);
        s = fmaf(qa.y, bf16_hi(w[t0].x), s);
        s = fmaf(qa.z, bf16_lo(w[t0].y), s);
        s = fmaf(qa.w, bf16_hi(w[t0].y), s);
        s = fmaf(qb.x, bf16_lo(w[t0].z), s);
        s = fmaf(qb.y, bf16_hi(w[t0].z), s);
        s = fmaf(qb.z, bf16_lo(w[t0].w), s);
        s = fmaf(qb.w, bf16_hi(w[t0].w), s);
    }
    }
    return orderable(s);
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
    float* sc;        // [C] scores
    int32_t* sz;      // [C] sizes
    int32_t* spre;    // [C] prefix of the whole cluster of rank k
    int32_t* srow;    // [C] first store row of the whole cluster of rank k
    uint32_t* pkey;   // [kPartCap] cut-cluster token keys
    int32_t* prow;    // [kRowChunk.. ] partial rows for this CTA's share
    int32_t* rows;    // [kRowChunk] row list of the current chunk
    int32_t* wbuf;    // [64] scan / misc scratch
    float* wcomb;     // [kWarps][G][130]
    float* ccomb;     // [S][G][130] (filled in CTA 0)
    CutInfo* cut;
};

template <int G>
__global__ void __launch_bounds__(kNT, (G <= 4) ? 2 : 1) select_attend_kernel(const DecodeArgs a, int32_t S,
                                                            int32_t prow_cap) {
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
        sm.sc = (float*)take(sizeof(float) * C);
        sm.sz = (int32_t*)take(sizeof(int32_t) * C);
        sm.spre = (int32_t*)take(sizeof(int32_t) * (C + 1));
        sm.srow = (int32_t*)take(sizeof(int32_t) * (C + 1));
        sm.pkey = (uint32_t*)take(sizeof(uint32_t) * kPartCap);
        sm.prow = (int32_t*)take(sizeof(int32_t) * prow_cap);
        sm.rows = (int32_t*)take(sizeof(int32_t) * kRowChunk);
        sm.wbuf = (int32_t*)take(sizeof(int32_t) * 64);
        sm.wcomb = (float*)take(sizeof(float) * kWarps * G * 130);
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
    // per round. The first round's centroid and size loads are issued before the query
    // loads, so both share one memory round trip.
    const int32_t pend = a.pending;
    const int64_t R = (int64_t)a.budget - a.n_sink - pend;  // >= 0 (host-checked)
    const int q8 = lane >> 3, l8 = lane & 7;
    constexpr int kPerRound = kWarps * 4;
    float4 mv[4];
    int32_t csize = 0;
    auto load_centroid = [&](int c) {
        if (c < c_end) {
            const float4* row = reinterpret_cast<const float4*>(mu + (int64_t)c * kD) + l8 * 4;
#pragma unroll
            for (int t = 0; t < 4; ++t) mv[t] = row[t];
            csize = off[c + 1] - off[c];
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) mv[t] = make_float4(0.f, 0.f, 0.f, 0.f);
            csize = 0;
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
            for (int r = l8; r < S; r += 8) {
                st_cluster_f32(map_shared_rank(smem_u32(&sm.sc[c]), r), s);
                st_cluster_u32(map_shared_rank(smem_u32(&sm.sz[c]), r), (uint32_t)csize);
            }
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();

    // ---------------------------------------------------------------- phase 2: ranks
    for (int c = c_begin + warp; c < c_end; c += kWarps) {
        const float s = sm.sc[c];
        int32_t rk = 0;
        int64_t pre = 0;
        for (int j = lane; j < C; j += 32) {
            const float t = sm.sc[j];
            if (t > s || (t == s && j < c)) {
                ++rk;
                pre += sm.sz[j];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            rk += __shfl_xor_sync(0xffffffffu, rk, o);
            pre += __shfl_xor_sync(0xffffffffu, pre, o);
        }
        const int32_t size = sm.sz[c];
        if (pre + size <= R) {  // whole cluster
            if (lane < S) {
                st_cluster_u32(map_shared_rank(smem_u32(&sm.spre[rk]), lane), (uint32_t)pre);
                st_cluster_u32(map_shared_rank(smem_u32(&sm.srow[rk]), lane), (uint32_t)off[c]);
            }
        } else if (pre <= R) {  // the cut cluster (R < pre + size)
            if (lane < S) {
                const uint32_t base = map_shared_rank(smem_u32(sm.cut), lane);
                st_cluster_u32(base + 0, (uint32_t)c);
                st_cluster_u32(base + 4, (uint32_t)pre);
                st_cluster_u32(base + 8, (uint32_t)rk);
                st_cluster_u32(base + 12, (uint32_t)off[c]);
                st_cluster_u32(base + 16, (uint32_t)size);
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
    const int64_t lo = T * rank / S, hi = T * (rank + 1) / S;

    // ---------------------------------------------------------------- phase 3: partial
    // This CTA's share of the partial tokens: positions [p_lo, p_hi) in store order.
    const int64_t p_lo = lo > base_p ? lo - base_p : 0;
    const int64_t p_hi = hi > base_p ? hi - base_p : 0;
    const int32_t csz = has_cut ? sm.cut->size : 0;
    const bool big_cut = csz > kPartCap;
    uint32_t* gkeys = a.part_scratch ? reinterpret_cast<uint32_t*>(a.part_scratch) +
                                           (int64_t)unit * a.part_ustride
                                     : nullptr;
    if (r_part > 0 && big_cut) {
        // Keys of a large cut cluster are written once, split across the cluster's CTAs.
        const int32_t crow = sm.cut->row;
        const int64_t k0 = (int64_t)csz * rank / S, k1 = (int64_t)csz * (rank + 1) / S;
        for (int64_t i = k0 + threadIdx.x; i < k1; i += kNT)
            gkeys[i] = row_key(a.kp + (kp_base + crow + i) * kD, sm.qbar);
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    if (r_part > 0 && p_hi > p_lo) {
        const int32_t crow = sm.cut->row;
        const uint32_t* skeys = sm.pkey;
        auto key_at = [&](int i) -> uint32_t { return big_cut ? __ldcg(gkeys + i) : skeys[i]; };
        if (!big_cut) {
            for (int i = threadIdx.x; i < csz; i += kNT)
                sm.pkey[i] = row_key(a.kp + (kp_base + crow + i) * kD, sm.qbar);
        }
        __syncthreads();
        // Threshold: key theta and `need` = how many keys equal to theta are taken (the
        // lowest-index ones), so that exactly r_part tokens are selected.
        uint32_t theta;
        int32_t need;
        if (csz <= kNT) {
            // comparison rank (ties: lower index)
            int32_t sel = 0;
            if (threadIdx.x < csz) {
                const uint32_t ki = key_at(threadIdx.x);
                int32_t rk = 0;
                for (int j = 0; j < csz; ++j) {
                    const uint32_t kj = key_at(j);
                    rk += (kj > ki) || (kj == ki && j < (int)threadIdx.x);
                }
                sel = rk < r_part;
            }
            int32_t tot;
            const int32_t pos = block_excl_scan(sel, sm.wbuf, &tot);
            if (sel && pos >= p_lo && pos < p_hi) sm.prow[pos - p_lo] = crow + threadIdx.x;
            theta = 0;
            need = 0;
            (void)theta;
            (void)need;
        } else {
            // radix select over 4 digits of 8 bits, most significant first
            uint32_t prefix = 0, mask = 0;
            need = r_part;
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
            theta = prefix;
            // select: key > theta, or key == theta among the first `need` such keys
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
                oid = ids[row];
            } else {
                row = sm.prow[idx - base_p - p_lo];
                oid = ids[row];
            }
            sm.rows[threadIdx.x] = row;
            if (sel_out) sel_out[idx] = oid;
        }
        __syncthreads();
        // The trip count is the same for every thread of the CTA: the full-mask shuffles
        // below need both half-warps of a warp in every iteration.
        for (int j0 = 0; j0 < n; j0 += 4 * (kNT / 16)) {
            uint4 kw[4], vw[4];
            int valid[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int j = j0 + hw + t * (kNT / 16);
                valid[t] = j < n;
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
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                // Every lane runs the shuffles below; rows past the chunk end only skip
                // the state update.
                if (!valid[t]) {
                    kw[t] = make_uint4(0u, 0u, 0u, 0u);
                    vw[t] = kw[t];
                }
                float kf[8], vf[8];
                const uint32_t kk[4] = {kw[t].x, kw[t].y, kw[t].z, kw[t].w};
                const uint32_t vv[4] = {vw[t].x, vw[t].y, vw[t].z, vw[t].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[2 * e] = bf16_lo(kk[e]);
                    kf[2 * e + 1] = bf16_hi(kk[e]);
                    vf[2 * e] = bf16_lo(vv[e]);
                    vf[2 * e + 1] = bf16_hi(vv[e]);
                }
                float z[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 qa = qg4[g * (kD / 4)];
                    const float4 qb = qg4[g * (kD / 4) + 1];
                    float s = qa.x * kf[0];
                    s = fmaf(qa.y, kf[1], s);
                    s = fmaf(qa.z, kf[2], s);
                    s = fmaf(qa.w, kf[3], s);
                    s = fmaf(qb.x, kf[4], s);
                    s = fmaf(qb.y, kf[5], s);
                    s = fmaf(qb.z, kf[6], s);
                    s = fmaf(qb.w, kf[7], s);
                    z[g] = s;
                }
#pragma unroll
                for (int o = 8; o > 0; o >>= 1)
#pragma unroll
                    for (int g = 0; g < G; ++g) z[g] += __shfl_xor_sync(0xffffffffu, z[g], o);
                if (!valid[t]) continue;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float mn = fmaxf(mrun[g], z[g]);
                    const float corr = exp2f(mrun[g] - mn);
                    const float pz = exp2f(z[g] - mn);
                    lrun[g] = lrun[g] * corr + pz;
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pz, vf[e], acc[g][e] * corr);
                    mrun[g] = mn;
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
    // warps -> CTA partial, written into CTA 0's combine buffer
    {
        const uint32_t dst0 = map_shared_rank(smem_u32(sm.ccomb), 0);
        for (int t = threadIdx.x; t < G * 130; t += kNT) {
            const int g = t / 130, e = t % 130;
            float mx = -INFINITY;
            for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, sm.wcomb[(w * G + g) * 130 + 128]);
            float v;
            if (e == 128) {
                v = mx;
            } else {
                float sacc = 0.f;
                for (int w = 0; w < kWarps; ++w) {
                    const float mw = sm.wcomb[(w * G + g) * 130 + 128];
                    const float cw = mw == -INFINITY ? 0.f : exp2f(mw - mx);
                    sacc += sm.wcomb[(w * G + g) * 130 + e] * cw;
                }
                v = sacc;
            }
            st_cluster_f32(dst0 + (uint32_t)(((rank * G + g) * 130 + e) * 4), v);
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();
    if (rank == 0) {
        float* o = a.out + ((int64_t)b * a.Hkv * G + (int64_t)h * G) * kD;
        for (int t = threadIdx.x; t < G * kD; t += kNT) {
            const int g = t / kD, d = t % kD;
            float mx = -INFINITY;
            for (int r = 0; r < S; ++r) mx = fmaxf(mx, sm.ccomb[(r * G + g) * 130 + 128]);
            float num = 0.f, den = 0.f;
            for (int r = 0; r < S; ++r) {
                const float* pr = sm.ccomb + (r * G + g) * 130;
                const float cw = pr[128] == -INFINITY ? 0.f : exp2f(pr[128] - mx);
                num += pr[d] * cw;
                den += pr[129] * cw;
            }
            o[t] = num / den;
        }
        if (a.sel_count && threadIdx.x == 0) a.sel_count[unit] = (int32_t)T;
    }
    if (sel_out && rank == (uint32_t)(S - 1)) {
        for (int64_t i = T + threadIdx.x; i < a.budget; i += kNT) sel_out[i] = -1;
    }
}

size_t smem_bytes(int G, int S, int C, int budget) {
    const int32_t pc = (int32_t)((int64_t)budget / S + 2);
    size_t b = 0;
    auto add = [&](size_t x) { b += (x + 15) & ~(size_t)15; };
    add(sizeof(float) * G * kD);
    add(sizeof(float) * kD);
    add(sizeof(float) * C);
    add(sizeof(int32_t) * C);
    add(sizeof(int32_t) * (C + 1));
    add(sizeof(int32_t) * (C + 1));
    add(sizeof(uint32_t) * kPartCap);
    add(sizeof(int32_t) * pc);
    add(sizeof(int32_t) * kRowChunk);
    add(sizeof(int32_t) * 64);
    add(sizeof(float) * kWarps * G * 130);
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
    const int32_t pc = (int32_t)((int64_t)a.budget / S + 2);
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
