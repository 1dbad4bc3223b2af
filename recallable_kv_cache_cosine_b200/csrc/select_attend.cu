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
//   1. each CTA scores a slice of the C centroids (fp32; a quarter-warp per centroid, the
//      next round's loads in flight during the current one) and broadcasts the scores to
//      every CTA of the cluster through distributed shared memory. Every CTA loads the
//      cluster boundaries itself;
//   2. every CTA then computes the whole selection on its own, without a second exchange:
//      the walk in descending score order stops at the first cluster whose inclusive token
//      count exceeds the remaining budget, so that cluster (the cut) is the weighted
//      quantile of the scores with the cluster sizes as weights. The scores are mapped
//      monotonically onto 256 linear buckets; a size-weighted histogram gives the bucket that
//      holds the cut, and the clusters of that bucket and above (a dozen or so) are compacted
//      and ranked exactly among themselves for their prefix sums;
//   3. the selected rows form one index space: sinks, pending (in append order, from the
//      two-window pending ring), whole clusters by rank, then the partial tokens of the cut
//      cluster. With a partial fill and S > 1, CTA S-1 takes exactly the partial tokens: it
//      copies the cut cluster's K and V rows into shared memory (started during the
//      selection when the histogram isolates the cut), ranks the tokens by qbar . k there
//      and attends the top ones in place. The other CTAs split the rest;
//   4. rows reach a two-slot shared-memory ring through cp.async (16 bytes per thread,
//      coalesced rows, XOR-swizzled 16-byte chunks); all of a CTA's rows are in flight at
//      once when they fit the ring. Each warp runs flash-decode on 16-row tiles with
//      tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulate): S^T = K Q^T with the
//      rows as M and the G query heads as N, an online softmax per head, then O^T += V^T P
//      with P split into bf16 high and low parts;
//   5. the warp partials (max, sum, accumulator) are merged per CTA, and the CTA partials in
//      CTA 0 through distributed shared memory, which writes the fp32 output.
// The kernel triggers programmatic dependent launch at entry and prefetches its centroid
// slice into L2 before waiting on the previous grid. A compile-time flag instantiates it for
// one selection per query head (G = 1 over (sequence, query head) units).
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
constexpr int kRowBytes = 2 * kD * 2;  // one K row and one V row, bf16

CKV_DEV uint32_t orderable(float f) {
    f = f + 0.0f;  // -0 -> +0
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 16-byte chunk j of ring row p, XOR-swizzled by the row's low 3 bits.
CKV_DEV uint32_t swz_addr(uint32_t base, int p, int j) {
    return base + (uint32_t)p * 256u + ((uint32_t)(j ^ (p & 7)) << 4);
}
CKV_DEV void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
CKV_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
CKV_DEV void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

// qbar . k over one half (64 dims) of a 256-byte key row in global memory: 8 independent
// 16-byte loads, then fp32 FMAs in dimension order.
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

CKV_DEV float from_orderable(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// The bin (of 256, scanned from the top) whose inclusive cumulative weight first exceeds
// `need`, computed by a whole warp; every lane returns it.
CKV_DEV int radix_bin_warp(const int32_t* hist, int32_t need) {
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
    const bool mine = above <= need && need < incl;
    if (mine) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (need < above + cnt[e]) {
                bin = 255 - 8 * lane - e;
                break;
            }
            above += cnt[e];
        }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, mine);
    return __shfl_sync(0xffffffffu, bin, who ? __ffs(who) - 1 : 0);
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

struct Smem {
    uint16_t* ringK;  // [RB][128] K rows of the current chunk(s)
    uint16_t* ringV;  // [RB][128] V rows
    float* wcomb;     // [kWarps][G][130]  (aliases the ring, after the last chunk)
    uint32_t* pkey;   // [kPartCap + 4]    (aliases the ring, before the first chunk)
    float* qg;        // [G][128], scaled by log2(e)/sqrt(128)
    float* qbar;      // [128]
    float* score;     // [C] every cluster's score (written through distributed shared memory)
    int32_t* off;     // [C + 1] cluster boundaries
    int32_t* spre;    // [C + 1] prefix of the whole cluster of rank k
    int32_t* srow;    // [C + 1] first store row of the whole cluster of rank k
    uint64_t* word;   // [cand_slots(C)] candidates: order key (score bits, inverted index)
    int32_t* wsz;     // [cand_slots(C)] candidates: sizes
    int32_t* hist;    // [256] histogram weights
    int32_t* hcnt;    // [256] histogram counts (clusters with tokens)
    uint32_t* rkey;   // [RB + 4] keys of a cut cluster held in the ring
    int32_t* prow;    // [prow_cap] partial rows of this CTA's share (ring positions or rows)
    int32_t* wbuf;    // [96] scan / misc scratch
    float* scl;       // [(kWarps + S) * G] merge scales, then [2 * G] sums
    float* ccomb;     // [S][G][130] (filled in CTA 0)
    int32_t* rsrc;    // [RB] source row of every ring row
    uint16_t* qh;     // [G][128] the queries, bf16 as given
    uint16_t* pbuf;   // [kWarps][2][8][16] softmax weights of a tile (bf16 high, low)
    uint64_t* full;   // mbarrier of the cut cluster's bulk copies
};

// Candidate list slots: kWarps lists of 32 * ceil(C / kNT) entries.
__host__ __device__ inline int cand_slots(int C) { return kNT * ((C + kNT - 1) / kNT); }

CKV_DEV size_t ring_bytes_of(int G, int RB) {
    size_t r = (size_t)RB * kRowBytes;
    const size_t w = sizeof(float) * kWarps * G * 130;
    const size_t k = sizeof(uint32_t) * (kPartCap + 4);
    if (w > r) r = w;
    if (k > r) r = k;
    return r;
}

// kPerHead: one selection per query head. The kernel then runs with G = 1 over virtual
// units (b, query head): virtual unit v reads the store of KV unit v / a.qsplit and its own
// query, output and selection rows.
template <int G, bool kPerHead>
__global__ void __launch_bounds__(kNT, 2)
    select_attend_kernel(const DecodeArgs a, int32_t S, int32_t prow_cap, int32_t RB) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int C = a.C;
    const uint32_t rank = cluster_ctarank();
    const int unit = blockIdx.x / S;
    const int su = kPerHead ? unit / a.qsplit : unit;  // the store's unit
    const int b = unit / a.Hkv, h = unit % a.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    Smem sm;
    {
        uint8_t* p = smem_raw;
        auto take = [&](size_t bytes) {
            uint8_t* r = p;
            p += (bytes + 127) & ~(size_t)127;
            return r;
        };
        uint8_t* ring = take(ring_bytes_of(G, RB));
        sm.ringK = (uint16_t*)ring;
        sm.ringV = sm.ringK + (size_t)RB * kD;
        sm.wcomb = (float*)ring;
        sm.pkey = (uint32_t*)ring;
        sm.qg = (float*)take(sizeof(float) * G * kD);
        sm.qbar = (float*)take(sizeof(float) * kD);
        sm.score = (float*)take(sizeof(float) * C);
        sm.off = (int32_t*)take(sizeof(int32_t) * (C + 1));
        sm.spre = (int32_t*)take(sizeof(int32_t) * (C + 1));
        sm.srow = (int32_t*)take(sizeof(int32_t) * (C + 1));
        sm.word = (uint64_t*)take(sizeof(uint64_t) * cand_slots(C));
        sm.wsz = (int32_t*)take(sizeof(int32_t) * cand_slots(C));
        sm.hist = (int32_t*)take(sizeof(int32_t) * 256);
        sm.hcnt = (int32_t*)take(sizeof(int32_t) * 256);
        sm.rkey = (uint32_t*)take(sizeof(uint32_t) * (RB + 4));
        sm.prow = (int32_t*)take(sizeof(int32_t) * prow_cap);
        sm.wbuf = (int32_t*)take(sizeof(int32_t) * 96);
        sm.scl = (float*)take(sizeof(float) * ((kWarps + S) * G + 2 * G));
        sm.ccomb = (float*)take(sizeof(float) * S * G * 130);
        sm.rsrc = (int32_t*)take(sizeof(int32_t) * RB);
        sm.qh = (uint16_t*)take(sizeof(uint16_t) * G * kD);
        sm.pbuf = (uint16_t*)take(sizeof(uint16_t) * kWarps * 256);
        sm.full = (uint64_t*)take(sizeof(uint64_t));
    }

    const int64_t kp_base = (int64_t)su * a.kp_ustride;
    const int64_t sp_base = (int64_t)su * a.sp_ustride;
    const int32_t* off = a.offsets + (int64_t)su * a.off_ustride;
    const float* mu = a.mu + (int64_t)su * a.mu_ustride * kD;
    const int c_begin = (int)((int64_t)C * rank / S);
    const int c_end = (int)((int64_t)C * (rank + 1) / S);

    // ---------------------------------------------------------------- phase 0
    pdl_launch_dependents();
    if (tid == 0) {
        if (c_end > c_begin)
            prefetch_l2_bulk(mu + (int64_t)c_begin * kD, (uint32_t)(c_end - c_begin) * kD * 4);
        sm.wbuf[45] = 0;  // cut cluster copies issued
        mbar_init(sm.full, 1);
        fence_mbar_init();
    }
    if (tid * 32 <= C) prefetch_l2(off + tid * 32);  // the boundaries, one 128-byte line each
    if (rank == 0 && tid == 0) {  // sinks, then the pending rows (up to two runs of the ring)
        const int32_t run1 = min(a.pending, a.pring - a.pstart);
        const int64_t r0[3] = {0, a.n_sink + a.pstart, a.n_sink};
        const int32_t nr[3] = {a.n_sink, run1, a.pending - run1};
        for (int k = 0; k < 3; ++k)
            if (nr[k] > 0) {
                prefetch_l2_bulk(a.spk + (sp_base + r0[k]) * kD, (uint32_t)nr[k] * kD * 2);
                prefetch_l2_bulk(a.spv + (sp_base + r0[k]) * kD, (uint32_t)nr[k] * kD * 2);
            }
    }
    cluster_arrive_relaxed();
    pdl_wait();

    // ---------------------------------------------------------------- phase 1: scores
    // A quarter-warp (8 lanes) per centroid, 16 dimensions per lane: 32 centroids per CTA
    // per round. The first round's centroid loads and the boundary loads are issued before
    // the query loads, so they share one memory round trip; later rounds are loaded one
    // round ahead.
    const int32_t pend = a.pending;
    const int32_t R = a.budget - a.n_sink - pend;  // >= 0 (host-checked)
    const int q8 = lane >> 3, l8 = lane & 7;
    constexpr int kPerRound = kWarps * 4;
    auto load_centroid = [&](int c, float4* mv) {
        if (c < c_end) {
            const float4* row = reinterpret_cast<const float4*>(mu + (int64_t)c * kD) + l8 * 4;
#pragma unroll
            for (int t = 0; t < 4; ++t) mv[t] = row[t];
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) mv[t] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    float4 mv[4];
    load_centroid(c_begin + warp * 4 + q8, mv);
    for (int i = tid; i <= C; i += kNT) sm.off[i] = off[i];
    {
        const uint16_t* q = a.q + ((int64_t)b * a.Hkv * G + (int64_t)h * G) * kD;
        const float scale = kLog2e * rsqrtf((float)kD);
        for (int i = tid; i < kD; i += kNT) {
            float s = 0.f;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const uint16_t raw = q[g * kD + i];
                const float x = __uint_as_float((uint32_t)raw << 16);
                s += x;
                sm.qg[g * kD + i] = x * scale;
                sm.qh[g * kD + i] = raw;
            }
            sm.qbar[i] = s;
        }
    }
    __syncthreads();
    cluster_wait_acquire();  // every CTA of the cluster is running
    for (int r0 = 0; r0 < c_end - c_begin; r0 += kPerRound) {
        const int c = c_begin + r0 + warp * 4 + q8;
        const bool more = r0 + kPerRound < c_end - c_begin;  // CTA-uniform
        float4 mn[4];
        if (more) load_centroid(c + kPerRound, mn);
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
            for (int r = l8; r < S; r += 8) st_cluster_f32(map_shared_rank(smem_u32(&sm.score[c]), r), s);
        }
        if (more) {
#pragma unroll
            for (int t = 0; t < 4; ++t) mv[t] = mn[t];
        }
    }
    cluster_arrive_release();
    cluster_wait_acquire();

    // ---------------------------------------------------------------- phase 2: selection
    // Every CTA holds all C scores and sizes and computes the same selection. The walk in
    // descending (score, -index) order stops at the first cluster whose inclusive token count
    // exceeds R: the cut. Scores are bucketed by a monotone map onto 256 linear buckets
    // between the smallest and the largest score, so bucket order never contradicts score
    // order. A size-weighted histogram gives the bucket that holds the cut; the clusters of
    // that bucket and above (the candidates) are compacted and ranked exactly among
    // themselves. A candidate is whole when its prefix plus its size fits R; the cut is the
    // candidate whose prefix fits and whose prefix plus size does not.
    const int32_t m_tot = sm.off[C] - sm.off[0];
    const bool has_cut = m_tot > R;  // otherwise every cluster is whole
    float smin = 0.f, inv = 0.f;
    int32_t bstar = 0;
    auto bucket = [&](float sc) {
        const float t = (sc + 0.0f - smin) * inv;
        return (int)fminf(fmaxf(t, 0.f), 255.f);
    };
    if (has_cut) {
        // smallest and largest score (order keys; one warp reduction each)
        uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
        for (int c = tid; c < C; c += kNT) {
            const uint32_t k = orderable(sm.score[c]);
            kmn = min(kmn, k);
            kmx = max(kmx, k);
        }
        kmn = __reduce_min_sync(0xffffffffu, kmn);
        kmx = __reduce_max_sync(0xffffffffu, kmx);
        uint32_t* kb = reinterpret_cast<uint32_t*>(sm.wbuf + 48);  // [8] minima, [8] maxima
        if (lane == 0) {
            kb[warp] = kmn;
            kb[8 + warp] = kmx;
        }
        sm.hist[tid] = 0;
        sm.hcnt[tid] = 0;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            kmn = min(kmn, kb[w]);
            kmx = max(kmx, kb[8 + w]);
        }
        const float mn = from_orderable(kmn), mx = from_orderable(kmx);
        const float range = mx - mn;
        smin = mn;
        inv = range > 1e-30f ? 255.99f / range : 0.f;  // finite; 0 puts every score in bucket 0
        for (int c = tid; c < C; c += kNT) {
            const int32_t w = sm.off[c + 1] - sm.off[c];
            if (w > 0) {
                const int bk = bucket(sm.score[c]);
                atomicAdd(&sm.hist[bk], w);
                atomicAdd(&sm.hcnt[bk], 1);
            }
        }
        __syncthreads();
        // every warp finds the cut's bucket itself (no extra block barrier)
        bstar = radix_bin_warp(sm.hist, R);
        // When bstar holds a single cluster with tokens, that cluster is the cut: CTA S-1,
        // which fills the partial tokens, starts copying its K and V rows now, while the
        // whole clusters are still being ranked.
        if ((int)rank == S - 1 && S > 1 && sm.hcnt[bstar] == 1) {
            for (int c = tid; c < C; c += kNT) {
                const int32_t w = sm.off[c + 1] - sm.off[c];
                if (w > 0 && w <= RB && w <= kNT && bucket(sm.score[c]) == bstar) {
                    const int64_t row = kp_base + sm.off[c];
                    const uint32_t bytes = (uint32_t)w * kD * 2;
                    mbar_arrive_expect_tx(sm.full, 2 * bytes);
                    bulk_load(sm.ringK, a.kp + row * kD, bytes, sm.full);
                    bulk_load(sm.ringV, a.vp + row * kD, bytes, sm.full);
                    sm.wbuf[45] = 1;
                }
            }
        }
    }
    // Candidates: every cluster without a cut, else the buckets >= bstar. Each warp compacts
    // the clusters it visits into its own list (kWarps lists of cap entries, any order).
    const int cap = 32 * ((C + kNT - 1) / kNT);
    int32_t n_mine = 0;
    for (int c0 = 0; c0 < C; c0 += kNT) {
        const int c = c0 + tid;
        bool cand = false;
        uint32_t k = 0;
        if (c < C) {
            const float sc = sm.score[c];
            k = orderable(sc);
            cand = !has_cut || bucket(sc) >= bstar;
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, cand);
        if (cand) {
            const int pos = warp * cap + n_mine + __popc(bal & ((1u << lane) - 1u));
            sm.word[pos] = ((uint64_t)k << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)c);
            sm.wsz[pos] = sm.off[c + 1] - sm.off[c];
        }
        n_mine += __popc(bal);
    }
    if (lane == 0) sm.wbuf[64 + warp] = n_mine;
    __syncthreads();
    int32_t pref[kWarps + 1];  // list starts in the flat candidate order
    pref[0] = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) pref[w + 1] = pref[w] + sm.wbuf[64 + w];
    const int32_t n_cand = pref[kWarps];
    // flat candidate index f -> slot in the warp lists
    auto slot_of = [&](int f) {
        int slot = f;
#pragma unroll
        for (int v = 1; v < kWarps; ++v)
            if (f >= pref[v]) slot = f - pref[v] + v * cap;
        return slot;
    };
    // rank and prefix of every candidate: 8 threads per candidate
    for (int i0 = 0; i0 < n_cand; i0 += kNT / 8) {
        const int i = i0 + (tid >> 3), sub = tid & 7;
        const int si = i < n_cand ? slot_of(i) : 0;
        const uint64_t ki = i < n_cand ? sm.word[si] : ~0ull;
        int32_t rk = 0, pre = 0;
#pragma unroll 4
        for (int j = sub; j < n_cand; j += 8) {
            const int sj = slot_of(j);
            const bool before = sm.word[sj] > ki;
            rk += before ? 1 : 0;
            pre += before ? sm.wsz[sj] : 0;
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
            rk += __shfl_xor_sync(0xffffffffu, rk, o);
            pre += __shfl_xor_sync(0xffffffffu, pre, o);
        }
        if (i < n_cand && sub == 0) {
            const int c = (int)(0xFFFFFFFFu - (uint32_t)(ki & 0xFFFFFFFFull));
            const int32_t sz = sm.wsz[si];
            if (pre + sz <= R || !has_cut) {  // whole
                sm.spre[rk] = pre;
                sm.srow[rk] = sm.off[c];
            } else if (pre <= R) {  // the cut
                sm.wbuf[36] = c;
                sm.wbuf[37] = pre;
                sm.wbuf[38] = rk;
            }
        }
    }
    __syncthreads();
    const int32_t cut_c = has_cut ? sm.wbuf[36] : -1;
    const int32_t n_whole = has_cut ? sm.wbuf[38] : C;

    // Index-space quantities are below the budget (int32).
    const int32_t W = has_cut ? sm.wbuf[37] : m_tot;  // tokens in whole clusters
    const int32_t r_part = has_cut ? R - W : 0;
    const int32_t csz = has_cut ? sm.off[cut_c + 1] - sm.off[cut_c] : 0;
    const int32_t crow = has_cut ? sm.off[cut_c] : 0;
    const int32_t base_w = a.n_sink + pend;
    const int32_t base_p = base_w + W;
    const int32_t T = base_p + r_part;
    // Work split of the selection index space [0, T). With a partial fill, CTA S-1 takes
    // exactly the partial tokens (it also ranks them) and the other CTAs split the rest.
    const bool dedicated = r_part > 0 && S > 1 && r_part <= prow_cap;
    int32_t lo, hi;
    if (dedicated) {
        if ((int)rank == S - 1) {
            lo = base_p;
            hi = T;
        } else {
            lo = split_point(base_p, rank, S - 1);
            hi = split_point(base_p, rank + 1, S - 1);
        }
    } else {
        lo = split_point(T, rank, S);
        hi = split_point(T, rank + 1, S);
    }
    const int32_t p_lo = lo > base_p ? lo - base_p : 0;
    const int32_t p_hi = hi > base_p ? hi - base_p : 0;
    const bool big_cut = csz > kPartCap;
    const bool resident = dedicated && (int)rank == S - 1 && csz <= RB && csz <= kNT;
    int32_t* sel_out = a.sel_idx ? a.sel_idx + (int64_t)unit * a.budget : nullptr;
    const int32_t* ids = a.ids + kp_base;

    // ---------------------------------------------------------------- phase 3/4: rows
    // Rows reach shared memory through cp.async (16 bytes per thread; 16 threads per 256-byte
    // row) into an XOR-swizzled ring: the 16-byte chunk j of ring row p sits at chunk
    // j ^ (p & 7), so the 8 rows of an ldmatrix tile fall in 8 different bank groups.
    // rsrc[p] names the source of ring row p: a store row (>= 0) or a sink / pending row
    // (-1 - index).
    const uint32_t ringK = smem_u32(sm.ringK), ringV = smem_u32(sm.ringV);
    // parts: 1 = K rows, 2 = V rows, 3 = both (one commit group)
    auto copy_rows = [&](int p0, int n, int parts) {
        const int per_row = parts == 3 ? 32 : 16;
        for (int i = tid; i < n * per_row; i += kNT) {
            const int p = p0 + i / per_row, j = i & 15;
            const int part = parts == 3 ? (i >> 4) & 1 : parts - 1;
            const int32_t r = sm.rsrc[p];
            const uint16_t* src = r >= 0 ? (part ? a.vp : a.kp) + (kp_base + r) * kD
                                         : (part ? a.spv : a.spk) + (sp_base + (-1 - r)) * kD;
            cp_async16(swz_addr(part ? ringV : ringK, p, j), src + j * 8);
        }
        cp_async_commit();
    };
    // Sources (and, when asked for, original token ids) of the selection positions [c0, c1),
    // written to ring rows p0 ...
    auto fill_rsrc = [&](int32_t c0, int32_t c1, int p0) {
        for (int32_t idx = c0 + tid; idx < c1; idx += kNT) {
            int32_t r;
            if (idx < base_w) {  // a sink, or pending token idx - n_sink of the ring
                r = -1 - (idx < a.n_sink ? idx : a.n_sink + (a.pstart + idx - a.n_sink) % a.pring);
            } else if (idx < base_p) {
                const int32_t x = idx - base_w;
                int k0 = 0, khi = n_whole - 1;  // last k with spre[k] <= x
                while (k0 < khi) {
                    const int mid = (k0 + khi + 1) >> 1;
                    if (sm.spre[mid] <= x) k0 = mid; else khi = mid - 1;
                }
                r = sm.srow[k0] + (x - sm.spre[k0]);
            } else {
                r = sm.prow[idx - base_p - p_lo];
            }
            sm.rsrc[p0 + (idx - c0)] = r;
            if (sel_out) sel_out[idx] = r >= 0 ? ids[r] : (idx < a.n_sink ? idx : (int32_t)(a.m + idx));
        }
    };

    // Attention on tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate), per warp over
    // 16-row tiles of the ring: S^T = K Q^T with the kv rows as M and the G heads as N (<= 8),
    // then O^T += V^T P with the head dimension as M. P is split into bf16 high and low parts
    // (two MMAs) so that the product keeps about 16 bits of the softmax weight.
    const int g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3;
    uint32_t qb[8][2];  // Q^T fragments: Q[head g8][16 s + 2 t4 ...], unscaled bf16
#pragma unroll
    for (int s8 = 0; s8 < 8; ++s8) {
        qb[s8][0] = g8 < G ? *reinterpret_cast<const uint32_t*>(sm.qh + g8 * kD + 16 * s8 + 2 * t4) : 0u;
        qb[s8][1] = g8 < G ? *reinterpret_cast<const uint32_t*>(sm.qh + g8 * kD + 16 * s8 + 2 * t4 + 8) : 0u;
    }
    float oacc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
    float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};  // heads 2 t4, 2 t4 + 1
    uint16_t* pw = sm.pbuf + warp * 256;  // [2][8 heads][16 rows] bf16 (high, low)
    const float qscale = kLog2e * rsqrtf((float)kD);
    // rows: ring row of tile row t is pos[t] (pos != nullptr) or p0 + t;
    // swz: rows XOR-swizzled (cp.async ring) or plain (bulk copies of the cut cluster)
    auto attend = [&](int p0, int n, const int32_t* pos, bool swz) {
        auto addr = [&](uint32_t base, int p, int j) {
            return base + (uint32_t)p * 256u + ((uint32_t)(j ^ (swz ? (p & 7) : 0)) << 4);
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
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(addr(ringK, pk, 2 * s8 + (mi >> 1)), a0, a1, a2, a3);
                mma_bf16_16816((s8 & 1) ? sb : sa, a0, a1, a2, a3, qb[s8][0], qb[s8][1]);
            }
            // S^T: [0], [1] = row g8, heads 2 t4, 2 t4 + 1; [2], [3] = row g8 + 8
            const bool v0 = r0 + g8 < n, v1 = r0 + g8 + 8 < n;
            float pr[4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float z0 = v0 ? (sa[hh] + sb[hh]) * qscale : -INFINITY;
                const float z1 = v1 ? (sa[2 + hh] + sb[2 + hh]) * qscale : -INFINITY;
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
                const __nv_bfloat16 hi = __float2bfloat16_rn(pr[e]);
                const __nv_bfloat16 lo = __float2bfloat16_rn(pr[e] - __bfloat162float(hi));
                pw[hd * 16 + rr] = __bfloat16_as_ushort(hi);
                pw[128 + hd * 16 + rr] = __bfloat16_as_ushort(lo);
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
                ldsm_x4_trans(addr(ringV, pv, 2 * mt + (mi & 1)), a0, a1, a2, a3);
                mma_bf16_16816(oacc[mt], a0, a1, a2, a3, ph0, ph1);
                mma_bf16_16816(oacc[mt], a0, a1, a2, a3, pl0, pl1);
            }
        }
    };

    const int32_t n_rows = resident ? csz : hi - lo;
    const int chunk = (resident || n_rows <= RB) ? RB : RB / 2;
    const int n_chunks = resident ? 1 : (n_rows + chunk - 1) / chunk;
    auto issue = [&](int ch) {  // every thread
        const int32_t c0 = lo + ch * chunk;
        const int32_t c1 = (c0 + chunk < hi) ? c0 + chunk : hi;
        const int p0 = n_chunks == 1 ? 0 : (ch & 1) * chunk;
        fill_rsrc(c0, c1, p0);
        __syncthreads();
        copy_rows(p0, c1 - c0, 3);
    };

    if (resident) {
        // ---- the cut cluster in shared memory (plain 256-byte rows): two bulk copies, issued
        // during the selection when the histogram isolated the cut, else now
        if (tid == 0 && sm.wbuf[45] == 0) {
            const uint32_t bytes = (uint32_t)csz * kD * 2;
            mbar_arrive_expect_tx(sm.full, 2 * bytes);
            bulk_load(sm.ringK, a.kp + (kp_base + crow) * kD, bytes, sm.full);
            bulk_load(sm.ringV, a.vp + (kp_base + crow) * kD, bytes, sm.full);
        }
        mbar_wait(sm.full, 0, a.err);
        // qbar . k, a half-warp per row (16-byte reads covering one 256-byte row), 8 rows
        // per half-warp in flight
        const int hw = tid >> 4, l16 = tid & 15;
        const float4 qa = reinterpret_cast<const float4*>(sm.qbar)[l16 * 2];
        const float4 qb4 = reinterpret_cast<const float4*>(sm.qbar)[l16 * 2 + 1];
        for (int r0 = 0; r0 < csz; r0 += 8 * (kNT / 16)) {
            float s[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int e = r0 + hw + k * (kNT / 16);
                s[k] = 0.f;
                if (e < csz) {
                    const uint4 w = lds_v4(ringK + (uint32_t)e * 256u + l16 * 16);
                    float t = qa.x * bf16_lo(w.x);
                    t = fmaf(qa.y, bf16_hi(w.x), t);
                    t = fmaf(qa.z, bf16_lo(w.y), t);
                    t = fmaf(qa.w, bf16_hi(w.y), t);
                    t = fmaf(qb4.x, bf16_lo(w.z), t);
                    t = fmaf(qb4.y, bf16_hi(w.z), t);
                    t = fmaf(qb4.z, bf16_lo(w.w), t);
                    s[k] = fmaf(qb4.w, bf16_hi(w.w), t);
                }
            }
            __syncwarp();  // all 8 rows' products first, then the reductions
#pragma unroll
            for (int o = 8; o > 0; o >>= 1)
#pragma unroll
                for (int k = 0; k < 8; ++k) s[k] += __shfl_xor_sync(0xffffffffu, s[k], o);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int e = r0 + hw + k * (kNT / 16);
                if (e < csz && l16 == 0) sm.rkey[e] = orderable(s[k]);
            }
        }
        if (tid < 4) sm.rkey[csz + tid] = 0u;  // pad: never outranks a key
        __syncthreads();
        // comparison rank (ties: lower index), tpe threads per token, 4 keys per load
        const int tpe = csz <= 32 ? 8 : (csz <= 64 ? 4 : (csz <= 128 ? 2 : 1));
        const int e = tid / tpe, sub = tid % tpe;
        int32_t rk = 0;
        if (e < csz) {
            const uint32_t ke = sm.rkey[e];
            const uint4* k4 = reinterpret_cast<const uint4*>(sm.rkey);
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
        if (sel) {
            sm.prow[pos] = e;
            if (sel_out) sel_out[base_p + pos] = ids[crow + e];
        }
        __syncthreads();
        attend(0, r_part, sm.prow, false);
    } else {
        if (sm.wbuf[45] != 0) mbar_wait(sm.full, 0, a.err);  // cut copies land before the ring is reused
        // ---- partial tokens of this CTA's share outside the ring path: rows into prow
        uint32_t* gkeys = a.part_scratch ? reinterpret_cast<uint32_t*>(a.part_scratch) +
                                               (int64_t)unit * a.part_ustride
                                         : nullptr;
        auto score_keys = [&](int64_t k0, int64_t k1, uint32_t* dst) {
            // two threads per row, one memory round trip per pass
            for (int64_t i0 = k0; i0 < k1; i0 += kNT / 2) {
                const int64_t i = i0 + (tid >> 1);
                const int half = tid & 1;
                float s = 0.f;
                if (i < k1) s = half_row_dot(a.kp + (kp_base + crow + i) * kD, half, sm.qbar);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                if (i < k1 && half == 0) dst[i] = orderable(s);
            }
        };
        if (r_part > 0 && big_cut) {
            // Keys of a large cut cluster are written once, split across the cluster's CTAs.
            const int64_t k0 = (int64_t)csz * rank / S, k1 = (int64_t)csz * (rank + 1) / S;
            score_keys(k0, k1, gkeys);
            cluster_arrive_release();
            cluster_wait_acquire();
        }
        if (r_part > 0 && p_hi > p_lo) {
            auto key_at = [&](int i) -> uint32_t { return big_cut ? __ldcg(gkeys + i) : sm.pkey[i]; };
            if (!big_cut) {
                score_keys(0, csz, sm.pkey);
                if (tid < 4) sm.pkey[csz + tid] = 0u;  // pad: never outranks a key
            }
            __syncthreads();
            if (!big_cut && csz <= kNT) {
                const int tpe = csz <= 32 ? 8 : (csz <= 64 ? 4 : (csz <= 128 ? 2 : 1));
                const int e = tid / tpe, sub = tid % tpe;
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
                // radix select over 4 digits of 8 bits, most significant first: the threshold
                // key theta and `pneed` = how many keys equal to theta are taken (the
                // lowest-index ones), so that exactly r_part tokens are selected.
                uint32_t prefix = 0, mask = 0;
                int32_t pneed = r_part;
                for (int pass = 0; pass < 4; ++pass) {
                    const int shift = 24 - 8 * pass;
                    sm.hist[tid] = 0;
                    __syncthreads();
                    for (int i = tid; i < csz; i += kNT) {
                        const uint32_t k = key_at(i);
                        if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & 255u], 1);
                    }
                    __syncthreads();
                    if (warp == 0) radix_pick_bin(sm.hist, pneed, false, sm.wbuf + 32);
                    __syncthreads();
                    pneed -= sm.wbuf[33];
                    prefix |= (uint32_t)sm.wbuf[32] << shift;
                    mask |= 255u << shift;
                }
                const uint32_t theta = prefix;
                int32_t eq_run = 0, sel_run = 0;
                for (int base = 0; base < csz; base += kNT) {
                    const int i = base + tid;
                    const uint32_t k = i < csz ? key_at(i) : 0u;
                    const int32_t eq = (i < csz && k == theta) ? 1 : 0;
                    int32_t eq_tot;
                    const int32_t eq_before = eq_run + block_excl_scan(eq, sm.wbuf, &eq_tot);
                    const int32_t sel = (i < csz) && (k > theta || (eq && eq_before < pneed));
                    int32_t sel_tot;
                    const int32_t pos = sel_run + block_excl_scan(sel, sm.wbuf, &sel_tot);
                    if (sel && pos >= p_lo && pos < p_hi) sm.prow[pos - p_lo] = crow + i;
                    eq_run += eq_tot;
                    sel_run += sel_tot;
                }
            }
            __syncthreads();
        }
        if (n_chunks > 0) issue(0);
        if (n_chunks > 1) issue(1);
        for (int ch = 0; ch < n_chunks; ++ch) {
            if (ch + 1 < n_chunks) cp_async_wait<1>(); else cp_async_wait<0>();
            __syncthreads();
            const int32_t c0 = lo + ch * chunk;
            const int n = (hi - c0) < chunk ? (hi - c0) : chunk;
            attend(n_chunks == 1 ? 0 : (ch & 1) * chunk, n, nullptr, true);
            if (ch + 2 < n_chunks) {
                __syncthreads();  // every warp is done with this slot
                issue(ch + 2);
            }
        }
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
            float* w = sm.wcomb + (warp * G + hd) * 130;
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
    float* wsc = sm.scl;                     // [kWarps][G]
    float* rsc = sm.scl + kWarps * G;        // [S][G]
    float* sums = sm.scl + (kWarps + S) * G; // [G] max, [G] sum
    // thread (g, w) in groups of 8 lanes: warp w's state for head g
    static_assert(kWarps == 8, "the merge below maps one lane per warp in groups of 8");
    if (tid < 8 * G) {
        // lanes of this warp taking part: 8 per head, heads in order (groups stay aligned)
        const int active = min(32, 8 * G - 32 * warp);
        const uint32_t gmask = active >= 32 ? 0xffffffffu : ((1u << active) - 1u);
        const int g = tid >> 3, w = tid & 7;
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
        for (int t = tid; t < G * 130; t += kNT) {
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
        if (tid < S * G) {
            const int active = min(32, S * G - 32 * warp);
            const uint32_t gmask = active >= 32 ? 0xffffffffu : ((1u << active) - 1u);
            const int g = tid / S, r = tid % S;
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
        for (int t = tid; t < G * kD; t += kNT) {
            const int g = t / kD, d = t % kD;
            float num = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r)
                if (r < S) num = fmaf(sm.ccomb[(r * G + g) * 130 + d], rsc[r * G + g], num);
            o[t] = num * sums[G + g];
        }
        if (a.sel_count && tid == 0) a.sel_count[unit] = (int32_t)T;
    }
    if (sel_out && rank == (uint32_t)(S - 1)) {
        for (int32_t i = T + tid; i < a.budget; i += kNT) sel_out[i] = -1;
    }
}

// Rows of partial tokens one CTA may own: twice the even share of the budget. The dedicated
// partial CTA is used only when the partial fill fits it; otherwise the even split applies,
// whose share is at most budget / S + 1.
int32_t prow_capacity(int budget, int S) { return (int32_t)(2 * ((int64_t)budget / S) + 2); }

size_t smem_bytes(int G, int S, int C, int budget, int RB) {
    const int32_t pc = prow_capacity(budget, S);
    size_t b = 0;
    auto add = [&](size_t x) { b += (x + 127) & ~(size_t)127; };
    size_t ring = (size_t)RB * kRowBytes;
    ring = ring > sizeof(float) * kWarps * G * 130 ? ring : sizeof(float) * kWarps * G * 130;
    ring = ring > sizeof(uint32_t) * (kPartCap + 4) ? ring : sizeof(uint32_t) * (kPartCap + 4);
    add(ring);
    add(sizeof(float) * G * kD);
    add(sizeof(float) * kD);
    add(sizeof(float) * C);
    add(sizeof(int32_t) * (C + 1));
    add(sizeof(int32_t) * (C + 1));
    add(sizeof(int32_t) * (C + 1));
    add(sizeof(uint64_t) * cand_slots(C));
    add(sizeof(int32_t) * cand_slots(C));
    add(sizeof(int32_t) * 256);
    add(sizeof(int32_t) * 256);
    add(sizeof(uint32_t) * (RB + 4));
    add(sizeof(int32_t) * pc);
    add(sizeof(int32_t) * 96);
    add(sizeof(float) * ((kWarps + S) * G + 2 * G));
    add(sizeof(float) * S * G * 130);
    add(sizeof(int32_t) * RB);
    add(sizeof(uint16_t) * G * kD);
    add(sizeof(uint16_t) * kWarps * 256);
    add(sizeof(uint64_t));
    return b;
}

// Ring rows for a cluster size S: enough for one CTA's even share of the budget in one
// chunk (128 to 256 rows), reduced while two CTAs would not fit one SM's shared memory.
int ring_rows(int G, int S, int C, int budget) {
    const int64_t share = (int64_t)budget / (S > 1 ? S - 1 : 1) + 2;
    int rb = (int)(share > 256 ? 256 : ((share + 31) / 32) * 32);
    if (rb < 128) rb = 128;  // also holds most cut clusters whole
    const size_t two_per_sm = 113 * 1024;
    while (rb > 64 && smem_bytes(G, S, C, budget, rb) > two_per_sm) rb -= 32;
    return rb;
}

struct Plan {
    int S = 0;
    int RB = 0;
    size_t smem = 0;
};

// Clusters of S CTAs with `smem` bytes each that can be resident at once (0 when none). Raises
// the kernel's shared-memory limit and allows 16-CTA clusters as needed.
int max_active_clusters(void (*kern)(DecodeArgs, int32_t, int32_t, int32_t), int S, size_t smem,
                        size_t* smem_set, bool* nonportable_set, int* nclusters) {
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

// One launch plan per (device, group size, units, C, budget), found once. The cluster size S
// is the largest power of two <= 16 whose clusters for all units are resident at once (one
// wave), with U * S <= 2 * SMs; otherwise the smallest S that fits in shared memory.
template <int G, bool kPerHead>
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
    auto kern = select_attend_kernel<G, kPerHead>;
    Plan best{};
    // Few units: one CTA per SM (a 256-row ring makes two CTAs too large for one SM) and at
    // most half of the SMs per launch, so that the next launch's CTAs, started early by
    // programmatic dependent launch, wait on other SMs instead of sharing these.
    for (int S = 16; S >= 2 && best.S == 0; S /= 2) {
        if ((int64_t)U * S * 2 > num_sms) continue;
        const int RB = 256;
        const size_t smem = smem_bytes(G, S, a.C, a.budget, RB);
        if (smem > 227 * 1024 || smem < 116 * 1024) continue;
        int nclusters = 0;
        const int rc = max_active_clusters(kern, S, smem, &smem_set, &nonportable_set, &nclusters);
        if (rc != CKV_OK) return rc;
        if (nclusters >= U) best = Plan{S, RB, smem};
    }
    for (int S = 16; S >= 1 && best.S == 0; S /= 2) {
        const int RB = ring_rows(G, S, a.C, a.budget);
        const size_t smem = smem_bytes(G, S, a.C, a.budget, RB);
        if (smem > 227 * 1024) continue;
        if ((int64_t)U * S > 2 * (int64_t)num_sms && S > 1) continue;
        int nclusters = 0;
        const int rc = max_active_clusters(kern, S, smem, &smem_set, &nonportable_set, &nclusters);
        if (rc != CKV_OK) return rc;
        if (nclusters <= 0) continue;
        best = Plan{S, RB, smem};
        if (nclusters >= U) break;
    }
    if (best.S == 0) {
        set_error("select_and_attend: no launch shape fits (budget or C too large for shared memory)");
        return CKV_ECAPACITY;
    }
    cache[key] = best;
    *out = best;
    return CKV_OK;
}

template <int G, bool kPerHead = false>
int launch_g(const DecodeArgs& a, int num_sms, cudaStream_t s) {
    Plan plan;
    int rc = plan_for<G, kPerHead>(a, num_sms, &plan);
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
    cudaError_t e = cudaLaunchKernelEx(&cfg, select_attend_kernel<G, kPerHead>, a, (int32_t)S, pc,
                                       (int32_t)plan.RB);
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
