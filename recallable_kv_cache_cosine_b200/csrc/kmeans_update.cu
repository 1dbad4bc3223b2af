// K-means init and centroid update for ClusterKV prefill clustering (sm_100a, CUDA cores).
//
// Page: "大模型KV Cache压缩技术：ClusterKV的语义空间优化" (ClusterKV explainer).
//  - section 3.1: a cluster's centroid is the mean of its member keys, mu = (1/n) sum k_i;
//  - section 3.2: K-means over the non-sink keys (seeded; init reading below);
//  - section 4.1: each cluster's KV is stored contiguously. The update therefore builds
//    the cluster-major layout with a stable counting sort (histogram -> exclusive scan ->
//    scatter), and the mean is a segmented reduction that reads the keys in that order.
//    The last iteration also writes the permuted K and V rows into the cluster store.
//
// Determinism: integer counts only (no float atomics). Each centroid is summed in a fixed
// order (every dimension by one thread over the members in ascending key index, in four
// interleaved partial sums added in a fixed order), so runs are bit-reproducible.
#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

// Writes mu (fp32) and mu_hat = bf16_rn(mu / |mu|) for one centroid. The calling warp holds
// dims 4*lane .. 4*lane+3 in `v`. A zero centroid gives mu_hat = 0.
CKV_DEV void store_centroid(float4 v, float* mu_row, uint16_t* muhat_row) {
    const int lane = lane_id();
    float ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float nrm = __fsqrt_rn(ss);
    reinterpret_cast<float4*>(mu_row)[lane] = v;
    uint2 h = make_uint2(0u, 0u);
    if (nrm > 0.f) {
        const __nv_bfloat16 a = __float2bfloat16_rn(__fdiv_rn(v.x, nrm));
        const __nv_bfloat16 b = __float2bfloat16_rn(__fdiv_rn(v.y, nrm));
        const __nv_bfloat16 c = __float2bfloat16_rn(__fdiv_rn(v.z, nrm));
        const __nv_bfloat16 d = __float2bfloat16_rn(__fdiv_rn(v.w, nrm));
        h.x = (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
        h.y = (uint32_t)__bfloat16_as_ushort(c) | ((uint32_t)__bfloat16_as_ushort(d) << 16);
    }
    reinterpret_cast<uint2*>(muhat_row)[lane] = h;
}

// ---------------------------------------------------------------------- init
// Seeded init: the first C entries of a Fisher-Yates shuffle of 0..m-1, driven by SplitMix64
// with key seed ^ (unit << 32) ^ window, each draw mapped into [0, m-i) by Lemire's
// multiply-shift. The sequential shuffle is: for i < C, j_i = i + draw_i; chosen[i] = a[j_i];
// a[j_i] = a[i] (position i is never read again). SplitMix64 is counter-based, so every j_i
// is computed at once, and every chosen[i] is resolved without the loop: a position p >= i
// changed before step i only as the target of an earlier step, so a[p] before step i is the
// value position s held just before step s, s being the last step < i with j_s = p (prev[i]),
// or p itself if there is none; and the value position s held before step s is, by the same
// rule, found by following the last step < s with j = s until a step whose own position was
// never a target: that step's index is the value. The centroids are split over CTAs of 64;
// each thread scans the earlier targets for its step and follows the (short) chain, and each
// warp then loads its 8 chosen key rows with all loads in flight.
constexpr int kInitPerCta = 64;  // centroids resolved and loaded per CTA (8 per warp)

__global__ void __launch_bounds__(256) kmeans_init_kernel(KeysView k, int32_t C, uint64_t seed,
                                                          int64_t unit_base, uint64_t window,
                                                          int32_t* init_idx, float* mu,
                                                          int64_t mu_ustride, uint16_t* mu_hat,
                                                          int64_t muhat_ustride) {
    pdl_launch_dependents();  // let the next kernel in the stream be scheduled early
    pdl_wait();               // the previous kernel's writes are visible from here on
    extern __shared__ int32_t sm[];
    const int u = blockIdx.y;
    const int c_lo = blockIdx.x * kInitPerCta;           // this CTA's centroids [c_lo, c_hi)
    const int c_hi = min(C, c_lo + kInitPerCta);
    const int32_t m = (int32_t)k.m;
    int32_t* target = sm;                // [c_hi] j_i of every step this CTA's chains can reach
    int32_t* chosen = sm + c_hi;         // [kInitPerCta]
    const uint64_t key = seed ^ ((uint64_t)(unit_base + u) << 32) ^ window;
    for (int i = threadIdx.x; i < c_hi; i += blockDim.x) {
        uint64_t st = key + (uint64_t)i * 0x9E3779B97F4A7C15ull;  // state before draw i
        const uint64_t x = splitmix64_next(st);
        target[i] = i + (int32_t)bounded_draw(x, (uint32_t)(m - i));
    }
    __syncthreads();
    // chosen[c] for c in [c_lo, c_hi), one warp per 8 centroids: prev = the last step < c with
    // the same target, then the link chain (the last step < s whose target is s) down to a
    // step never targeted before. Every search is warp-wide: the lanes stride over the earlier
    // steps and the largest match wins.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto last_before = [&](int lim, int32_t val) {  // largest s < lim with target[s] == val
        int32_t best = -1;
        for (int s0 = 0; s0 < lim; s0 += 32) {  // warp-uniform trip count
            const int st = s0 + lane;
            if (st < lim && target[st] == val) best = st;
        }
        return (int32_t)__reduce_max_sync(0xffffffffu, (uint32_t)(best + 1)) - 1;
    };
    for (int j = 0; j < 8; ++j) {
        const int c = c_lo + warp * 8 + j;
        if (c >= c_hi) break;  // warp-uniform
        int32_t x = last_before(c, target[c]);
        int32_t idx = target[c];
        if (x >= 0) {
            for (;;) {  // every step strictly lowers x
                const int32_t lk = last_before(x, x);
                if (lk < 0) break;
                x = lk;
            }
            idx = x;
        }
        if (lane == 0) chosen[c - c_lo] = idx;
    }
    __syncthreads();
    // one warp per 8 centroids, all 8 key rows in flight at once
    const uint16_t* keys = k.base + ((int64_t)u * k.n_rows + k.row0) * kD;
    uint2 w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = c_lo + warp * 8 + j;
        if (c < c_hi) w[j] = reinterpret_cast<const uint2*>(keys + (int64_t)chosen[c - c_lo] * kD)[lane_id()];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = c_lo + warp * 8 + j;
        if (c >= c_hi) break;  // warp-uniform
        const float4 v = make_float4(bf16_lo(w[j].x), bf16_hi(w[j].x), bf16_lo(w[j].y), bf16_hi(w[j].y));
        store_centroid(v, mu + ((int64_t)u * mu_ustride + c) * kD,
                       mu_hat + ((int64_t)u * muhat_ustride + c) * kD);
        if (init_idx && lane_id() == 0) init_idx[(int64_t)u * C + c] = chosen[c - c_lo];
    }
}

// ---------------------------------------------------------------------- count
// chunk[u][ch][c] = number of keys of chunk ch (kChunk keys) assigned to c.
__global__ void __launch_bounds__(256) kmeans_count_kernel(const int32_t* assign, int64_t a_ustride,
                                                           int64_t m, int32_t C, int32_t nch,
                                                           int32_t* chunk, uint32_t* err) {
    pdl_launch_dependents();  // let the next kernel in the stream be scheduled early
    pdl_wait();               // the previous kernel's writes are visible from here on
    extern __shared__ int32_t hist[];
    const int ch = blockIdx.x, u = blockIdx.y;
    for (int c = threadIdx.x; c < C; c += blockDim.x) hist[c] = 0;
    __syncthreads();
    const int64_t lo = (int64_t)ch * kChunk;
    const int64_t hi = lo + kChunk < m ? lo + kChunk : m;
    const int32_t* a = assign + (int64_t)u * a_ustride;
    for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
        const int32_t c = a[i];
        if ((uint32_t)c < (uint32_t)C) {
            atomicAdd(&hist[c], 1);
        } else if (err) {
            atomicOr(err, kErrBadState);  // caller-supplied assignment out of range: skipped
        }
    }
    __syncthreads();
    int32_t* out = chunk + ((int64_t)u * nch + ch) * C;
    for (int c = threadIdx.x; c < C; c += blockDim.x) out[c] = hist[c];
}

// ---------------------------------------------------------------------- scan
// Per unit: sizes[c] = sum over chunks; offsets = exclusive scan of sizes, and offsets[C] =
// the keys counted (m, unless the count kernel skipped out-of-range assignments; the mean
// kernel then never reaches perm entries that the scatter did not write);
// chunk[u][ch][c] becomes the number of keys of cluster c in chunks before ch.
__global__ void __launch_bounds__(512) kmeans_scan_kernel(int32_t* chunk, int32_t nch, int32_t C,
                                                           int64_t m, int32_t* offsets,
                                                           int64_t off_ustride) {
    pdl_launch_dependents();  // let the next kernel in the stream be scheduled early
    pdl_wait();               // the previous kernel's writes are visible from here on
    extern __shared__ int32_t sz[];  // [C] then [32] warp totals
    int32_t* wsum = sz + C;
    const int u = blockIdx.x;
    int32_t* ck = chunk + (int64_t)u * nch * C;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        int32_t run = 0;
        for (int ch0 = 0; ch0 < nch; ch0 += 16) {
            int32_t h[16];  // 16 loads in flight per batch
#pragma unroll
            for (int t = 0; t < 16; ++t) h[t] = ch0 + t < nch ? ck[(int64_t)(ch0 + t) * C + c] : 0;
#pragma unroll
            for (int t = 0; t < 16; ++t)
                if (ch0 + t < nch) {
                    ck[(int64_t)(ch0 + t) * C + c] = run;
                    run += h[t];
                }
        }
        sz[c] = run;
    }
    __syncthreads();
    // exclusive scan of sz[0..C) with a contiguous run per thread
    const int per = (C + blockDim.x - 1) / blockDim.x;
    const int c0 = threadIdx.x * per;
    int32_t local = 0;
    for (int j = 0; j < per; ++j)
        if (c0 + j < C) local += sz[c0 + j];
    int32_t incl = local;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int32_t run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
    int32_t* off = offsets + (int64_t)u * off_ustride;
    for (int j = 0; j < per; ++j)
        if (c0 + j < C) {
            off[c0 + j] = run;
            run += sz[c0 + j];
        }
    if (threadIdx.x == 0) off[C] = wsum[31];  // total over the warps: the keys counted
}

// ---------------------------------------------------------------------- scatter
// One CTA of 8 warps per chunk of 1024 keys. Warp w takes keys [128 w, 128 w + 128) of the
// chunk, 32 at a time in index order: lanes with equal clusters are grouped with match.any and
// ranked by lane on top of the warp's running count of that cluster. Then, per cluster, a scan
// over the 8 warps starting at the cluster's offset plus the chunk's prefix gives each warp's
// first position, and every key lands at that position plus its rank. Keys of one cluster
// therefore keep their index order: a stable counting sort.
constexpr int kScatterWarps = 8;
constexpr int kScatterKeysPerWarp = kChunk / kScatterWarps;  // 128

__global__ void __launch_bounds__(kScatterWarps * 32) kmeans_scatter_kernel(
    const int32_t* assign, int64_t a_ustride, int64_t m, int32_t C, int32_t nch,
    const int32_t* chunk, const int32_t* offsets, int64_t off_ustride, int32_t* perm,
    int64_t perm_ustride, int32_t* zero_next) {
    pdl_launch_dependents();  // let the next kernel in the stream be scheduled early
    pdl_wait();               // the previous kernel's writes are visible from here on
    extern __shared__ int32_t cntw[];  // [kScatterWarps][C] counts, then first positions
    int32_t* sa = cntw + kScatterWarps * C;  // [kChunk] assignments (-1: none / out of range)
    int32_t* srank = sa + kChunk;            // [kChunk] rank among the warp's keys of its cluster
    const int ch = blockIdx.x, u = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t lo = (int64_t)ch * kChunk;
    const int64_t hi = lo + kChunk < m ? lo + kChunk : m;
    const int32_t* a = assign + (int64_t)u * a_ustride;
    for (int i = tid; i < kChunk; i += kScatterWarps * 32) {
        int32_t c = lo + i < hi ? a[lo + i] : -1;
        if ((uint32_t)c >= (uint32_t)C) c = -1;  // out of range (flagged by the count kernel)
        sa[i] = c;
    }
    for (int i = tid; i < kScatterWarps * C; i += kScatterWarps * 32) cntw[i] = 0;
    if (zero_next) {  // this chunk's row of the next iteration's count buffer
        int32_t* z = zero_next + ((int64_t)u * nch + ch) * C;
        for (int c = tid; c < C; c += kScatterWarps * 32) z[c] = 0;
    }
    __syncthreads();
    int32_t* mine = cntw + warp * C;
    const uint32_t lt = (1u << lane) - 1u;
    for (int r = 0; r < kScatterKeysPerWarp / 32; ++r) {  // warp-uniform trip count
        const int i = warp * kScatterKeysPerWarp + r * 32 + lane;
        const int32_t c = sa[i];
        const uint32_t same = __match_any_sync(0xffffffffu, c);
        const int32_t before = c >= 0 ? mine[c] : 0;
        __syncwarp();
        if (c >= 0 && (same & lt) == 0) mine[c] = before + __popc(same);
        srank[i] = before + __popc(same & lt);
        __syncwarp();
    }
    __syncthreads();
    const int32_t* off = offsets + (int64_t)u * off_ustride;
    const int32_t* base = chunk + ((int64_t)u * nch + ch) * C;
    for (int c = tid; c < C; c += kScatterWarps * 32) {
        int32_t run = off[c] + base[c];
#pragma unroll
        for (int w = 0; w < kScatterWarps; ++w) {
            const int32_t t = cntw[w * C + c];
            cntw[w * C + c] = run;
            run += t;
        }
    }
    __syncthreads();
    int32_t* pm = perm + (int64_t)u * perm_ustride;
    for (int i = tid; i < kChunk; i += kScatterWarps * 32) {
        const int32_t c = sa[i];
        if (c >= 0) pm[cntw[(i / kScatterKeysPerWarp) * C + c] + srank[i]] = (int32_t)(lo + i);
    }
}

// ---------------------------------------------------------------------- mean
// One CTA (4 warps) per cluster: mu_c = (1/|c|) sum of the member keys (fp32); empty clusters
// keep mu_c; then mu_hat. The member list, then the members' key rows, are gathered into
// shared memory (cp.async, 16 bytes per thread, up to kMeanRows rows per pass, one memory
// round trip per pass). Thread d sums dimension d over the rows in member order into four
// partial sums (rows 4i, 4i+1, 4i+2, 4i+3 of each pass), added in a fixed order, so the
// result is run-to-run exact. With a relayout the pass also writes the key rows, their V rows
// and the original token ids into the cluster-major store.
constexpr int kMeanThreads = 128;  // one thread per dimension
constexpr int kMeanRows = 128;

CKV_DEV void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kMeanThreads) kmeans_mean_kernel(KeysView k, const int32_t* perm,
                                                                   int64_t perm_ustride,
                                                                   const int32_t* offsets,
                                                                   int64_t off_ustride, int32_t C,
                                                                   float* mu, int64_t mu_ustride,
                                                                   uint16_t* mu_hat,
                                                                   int64_t muhat_ustride,
                                                                   Relayout rl) {
    // The relayout pass ends a prefill: it writes the cluster store, which the decode kernel
    // reads before its own dependency wait, so it lets its dependents start only when it ends.
    if (rl.kp == nullptr) pdl_launch_dependents();
    pdl_wait();  // the previous kernel's writes are visible from here on
    static_assert(kMeanThreads == kD, "one thread per dimension");
    __shared__ __align__(16) uint16_t srow[kMeanRows * kD];
    __shared__ int32_t sidx[kMeanRows];
    __shared__ __align__(16) float ssum[kD];
    const int tid = threadIdx.x;
    const int c = blockIdx.x;
    const int u = blockIdx.y;
    const int32_t* off = offsets + (int64_t)u * off_ustride;
    const int32_t lo = off[c], hi = off[c + 1];
    const int32_t* pm = perm + (int64_t)u * perm_ustride;
    const int64_t ubase = (int64_t)u * k.n_rows + k.row0;
    const uint16_t* keys = k.base + ubase * kD;
    const bool relay = rl.kp != nullptr;
    const uint16_t* vals = relay ? rl.V + ubase * kD : nullptr;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    for (int32_t j0 = lo; j0 < hi; j0 += kMeanRows) {
        const int n = (hi - j0) < kMeanRows ? (hi - j0) : kMeanRows;
        if (j0 > lo) __syncthreads();  // the previous pass is done with srow and sidx
        for (int r = tid; r < n; r += kMeanThreads) sidx[r] = pm[j0 + r];
        __syncthreads();
        for (int i = tid; i < n * 16; i += kMeanThreads) {
            const int r = i >> 4, ch = i & 15;
            cp_async16(srow + r * kD + ch * 8, keys + (int64_t)sidx[r] * kD + ch * 8);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (relay) {  // V rows and token ids while the key rows arrive
            for (int i = tid; i < n * 16; i += kMeanThreads) {
                const int r = i >> 4, ch = i & 15;
                const int64_t dst = (int64_t)u * rl.ustride_rows + j0 + r;  // stored row j0 + r
                reinterpret_cast<uint4*>(rl.vp + dst * kD)[swz(j0 + r, ch)] =
                    reinterpret_cast<const uint4*>(vals + (int64_t)sidx[r] * kD)[ch];
            }
            for (int r = tid; r < n; r += kMeanThreads)
                rl.ids[(int64_t)u * rl.ustride_rows + j0 + r] = rl.id_base + sidx[r];
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        const uint16_t* col = srow + tid;
        int r = 0;
        for (; r + 4 <= n; r += 4) {
            acc0 += __uint_as_float((uint32_t)col[(r + 0) * kD] << 16);
            acc1 += __uint_as_float((uint32_t)col[(r + 1) * kD] << 16);
            acc2 += __uint_as_float((uint32_t)col[(r + 2) * kD] << 16);
            acc3 += __uint_as_float((uint32_t)col[(r + 3) * kD] << 16);
        }
        for (; r < n; ++r) acc0 += __uint_as_float((uint32_t)col[r * kD] << 16);
        if (relay) {
            for (int i = tid; i < n * 16; i += kMeanThreads) {
                const int rr = i >> 4, ch = i & 15;
                const int64_t dst = (int64_t)u * rl.ustride_rows + j0 + rr;
                reinterpret_cast<uint4*>(rl.kp + dst * kD)[swz(j0 + rr, ch)] =
                    reinterpret_cast<const uint4*>(srow + rr * kD)[ch];
            }
        }
    }
    ssum[tid] = (acc0 + acc1) + (acc2 + acc3);
    __syncthreads();
    if (tid >= 32) return;
    const int lane = tid;
    float4 v = reinterpret_cast<const float4*>(ssum)[lane];
    float* mrow = mu + ((int64_t)u * mu_ustride + c) * kD;
    if (hi > lo) {
        const float n = (float)(hi - lo);
        v = make_float4(__fdiv_rn(v.x, n), __fdiv_rn(v.y, n), __fdiv_rn(v.z, n), __fdiv_rn(v.w, n));
    } else {
        v = reinterpret_cast<const float4*>(mrow)[lane];
    }
    store_centroid(v, mrow, mu_hat + ((int64_t)u * muhat_ustride + c) * kD);
}

__global__ void copy_sinks_kernel(const uint16_t* K, const uint16_t* V, int64_t n, int32_t n_sink,
                                  uint16_t* spk, uint16_t* spv, int64_t sp_ustride) {
    // The last kernel of a prefill: no early trigger, so a following decode kernel, which
    // reads the cluster store before its dependency wait, starts once the store is complete.
    pdl_wait();  // the previous kernel's writes are visible from here on
    const int u = blockIdx.x;
    const int64_t words = (int64_t)n_sink * kD / 8;  // 16-byte words
    const uint4* ks = reinterpret_cast<const uint4*>(K + (int64_t)u * n * kD);
    const uint4* vs = reinterpret_cast<const uint4*>(V + (int64_t)u * n * kD);
    uint4* kd = reinterpret_cast<uint4*>(spk + (int64_t)u * sp_ustride * kD);
    uint4* vd = reinterpret_cast<uint4*>(spv + (int64_t)u * sp_ustride * kD);
    for (int64_t i = threadIdx.x; i < words; i += blockDim.x) {  // stored row i / 16
        const int64_t o = (i & ~15ll) | swz(i >> 4, (int)(i & 15));
        kd[o] = ks[i];
        vd[o] = vs[i];
    }
}

}  // namespace

int launch_kmeans_init(const KeysView& k, int32_t C, uint64_t seed, int64_t unit_base,
                       uint64_t window, int32_t* init_idx, float* mu, int64_t mu_ustride,
                       uint16_t* mu_hat, int64_t muhat_ustride, uint32_t* err, cudaStream_t s) {
    (void)err;
    const size_t smem = ((size_t)C + kInitPerCta) * sizeof(int32_t);  // C <= 4096: <= 17 KB
    int rc = ensure_smem((const void*)kmeans_init_kernel, smem, "init: set smem");
    if (rc != CKV_OK) return rc;
    const dim3 grid((unsigned)((C + kInitPerCta - 1) / kInitPerCta), (unsigned)k.U);
    cudaError_t e = launch_pdl(kmeans_init_kernel, grid, dim3(256), smem, s, k, C, seed, unit_base,
                               window, init_idx, mu, mu_ustride, mu_hat, muhat_ustride);
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "init: launch");
}

int launch_kmeans_update(const KeysView& k, const int32_t* assign, int64_t assign_ustride,
                         int32_t C, float* mu, int64_t mu_ustride, uint16_t* mu_hat,
                         int64_t muhat_ustride, int32_t* offsets, int64_t off_ustride,
                         int32_t* perm, int64_t perm_ustride, int32_t* chunk_ws,
                         const Relayout* relayout, uint32_t* err, cudaStream_t s, bool counted,
                         int32_t* zero_next) {
    const int32_t nch = (int32_t)n_chunks(k.m);
    cudaError_t e;
    const size_t hsmem = (size_t)C * sizeof(int32_t);
    const size_t scsmem = ((size_t)kScatterWarps * C + 2 * kChunk) * sizeof(int32_t);
    const size_t ssmem = (size_t)(C + 32) * sizeof(int32_t);
    int rc = ensure_smem((const void*)kmeans_count_kernel, hsmem, "count: set smem");
    if (rc == CKV_OK) rc = ensure_smem((const void*)kmeans_scatter_kernel, scsmem, "scatter: set smem");
    if (rc == CKV_OK) rc = ensure_smem((const void*)kmeans_scan_kernel, ssmem, "scan: set smem");
    if (rc != CKV_OK) return rc;
    if (nch > 0 && !counted) {
        e = launch_pdl(kmeans_count_kernel, dim3(nch, k.U), dim3(256), hsmem, s, assign,
                       assign_ustride, k.m, C, nch, chunk_ws, err);
        if (e != cudaSuccess) return cuda_fail(e, "update: count launch");
    }
    e = launch_pdl(kmeans_scan_kernel, dim3(k.U), dim3(512), ssmem, s, chunk_ws, nch, C, k.m,
                   offsets, off_ustride);
    if (e != cudaSuccess) return cuda_fail(e, "update: scan launch");
    if (nch > 0) {
        e = launch_pdl(kmeans_scatter_kernel, dim3(nch, k.U), dim3(kScatterWarps * 32), scsmem, s, assign,
                       assign_ustride, k.m, C, nch, chunk_ws, offsets, off_ustride, perm,
                       perm_ustride, zero_next);
        if (e != cudaSuccess) return cuda_fail(e, "update: scatter launch");
    }
    Relayout rl{};
    if (relayout) rl = *relayout;
    e = launch_pdl(kmeans_mean_kernel, dim3(C, k.U), dim3(kMeanThreads), 0, s, k, perm, perm_ustride,
                   offsets, off_ustride, C, mu, mu_ustride, mu_hat, muhat_ustride, rl);
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "update: launch");
}

int launch_copy_sinks(const uint16_t* K, const uint16_t* V, int64_t n, int32_t U, int32_t n_sink,
                      uint16_t* spk, uint16_t* spv, int64_t sp_ustride_rows, cudaStream_t s) {
    cudaError_t e = launch_pdl(copy_sinks_kernel, dim3(U), dim3(256), 0, s, K, V, n, n_sink, spk,
                               spv, sp_ustride_rows);
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "sinks: launch");
}

}  // namespace ckv
