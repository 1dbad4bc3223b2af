// Drift check and split of drifted clusters for ClusterKV decode (sm_100a).
//
// Page: "大模型KV Cache压缩技术：ClusterKV的语义空间优化" (ClusterKV explainer), section 3.2,
// decode phase: centroid drift is detected, and a cluster whose mean intra-cluster distance
// is above a threshold is split. The page fixes neither the distance, nor the threshold, nor
// the split. Readings:
//   - drift_c = mean over the members of c of (1 - cos(k_i, mu_c)), the clustering's cosine
//     distance to the stored centroid (a cosine with a zero vector counts as 0, an empty
//     cluster has drift 0);
//   - the threshold is a parameter;
//   - a cluster with drift above the threshold and at least two members is split by cosine
//     K-means with 2 clusters on its own rows (the prefill's init rule and iteration count),
//     at most `room` clusters per unit, lowest index first; `room` is the caller's maximum
//     clamped to the clusters left, and every unit ends with exactly C + room clusters
//     (units that split fewer pad with empty clusters), so the host knows the new count
//     without reading anything back.
// The two halves take indices c' and c' + 1 (c' = c + splits below c); later clusters shift
// up. Rows move only inside the cluster's own segment (first half, then second half, each in
// its previous order), so the token ids stay ascending inside every cluster.
//
// Five launches, one pass each:
//   drift    one warp per (unit, cluster), 16 rows in flight: the mean cosine distance, fp32;
//   plan     one CTA per unit: flags, the cap, the new index of every cluster (a block scan),
//            and the unit's list of clusters to split;
//   kmeans   one CTA per (list entry, unit) for at most `room` entries: 2-means on the
//            segment (staged in shared memory up to 192 rows, else read from global memory),
//            then the stable partition of its K/V rows and ids through a row scratch;
//   scatter  one warp per (cluster, unit): the cluster's centroid(s) and offset(s) go to
//            their new indices in a scratch copy; units with fewer splits than the layer's
//            maximum get empty clusters (no rows, zero centroid) so that every unit of the
//            layer has the same cluster count. An empty cluster never adds a selected row;
//   copy     the scratch copy back into the store (a move in place would have to run
//            serially, highest index first).
#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

constexpr int kDriftWarps = 8;
constexpr int kPlanThreads = 256;
constexpr int kSplitThreads = 256;
constexpr int kStageRows = 192;  // segments up to this size are staged in shared memory

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;  // the xor butterfly leaves the same value in every lane
}

__device__ __forceinline__ bool segment_ok(int32_t lo, int32_t hi, int64_t m) {
    return lo >= 0 && hi >= lo && (int64_t)hi <= m;
}

__global__ void __launch_bounds__(kDriftWarps * 32) drift_kernel(const SplitArgs a) {
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.y, c = blockIdx.x * kDriftWarps + warp;
    if (c >= a.C) return;
    const int32_t* off = a.offsets + (int64_t)u * a.off_ustride;
    int32_t lo = off[c], hi = off[c + 1];
    if (!segment_ok(lo, hi, a.m)) {
        if (lane == 0) atomicOr(a.err, kErrBadState);
        lo = hi = 0;
    }
    const float4 mu = reinterpret_cast<const float4*>(a.mu + ((int64_t)u * a.mu_ustride + c) * kD)[lane];
    const float mm = warp_sum(mu.x * mu.x + mu.y * mu.y + mu.z * mu.z + mu.w * mu.w);
    const float nm = __fsqrt_rn(mm);
    const uint16_t* base = a.kp + (int64_t)u * a.kp_ustride * kD;  // lane: dims 4 lane .. + 3
    float acc = 0.f;
    constexpr int kInFlight = 16;
    for (int32_t j = lo; j < hi; j += kInFlight) {  // warp-uniform trip count
        uint2 w[kInFlight];
#pragma unroll
        for (int r = 0; r < kInFlight; ++r)
            if (j + r < hi)
                w[r] = *reinterpret_cast<const uint2*>(base + (int64_t)(j + r) * kD + swz_elem(j + r, lane * 4));
        // the lane's partial k.mu (value 2 r) and k.k (value 2 r + 1) of the 16 rows, reduced
        // together: each exchange halves the values a lane keeps (xor 16: 16 values, xor 8:
        // 8, ... xor 1: one), so lane l ends with the full value l (31 shuffles for 32 sums)
        float v[2 * kInFlight];
#pragma unroll
        for (int r = 0; r < kInFlight; ++r) {
            v[2 * r] = v[2 * r + 1] = 0.f;
            if (j + r < hi) {
                const float k0 = bf16_lo(w[r].x), k1 = bf16_hi(w[r].x), k2 = bf16_lo(w[r].y),
                            k3 = bf16_hi(w[r].y);
                v[2 * r] = k0 * mu.x + k1 * mu.y + k2 * mu.z + k3 * mu.w;
                v[2 * r + 1] = k0 * k0 + k1 * k1 + k2 * k2 + k3 * k3;
            }
        }
#pragma unroll
        for (int half = 16; half >= 1; half >>= 1) {
            const bool hi_lane = (lane & half) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float keep = hi_lane ? v[half + i] : v[i];
                const float give = hi_lane ? v[i] : v[half + i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, give, half);
            }
        }
        const float kk = __shfl_xor_sync(0xffffffffu, v[0], 1);  // row lane >> 1's k.k, at even lanes
        if ((lane & 1) == 0 && j + (lane >> 1) < hi) {
            const float dot = v[0];
            const float cs = (kk > 0.f && mm > 0.f) ? __fdiv_rn(dot, __fmul_rn(__fsqrt_rn(kk), nm)) : 0.f;
            acc += 1.f - cs;
        }
    }
    acc = warp_sum(acc);
    const float drift = hi > lo ? __fdiv_rn(acc, (float)(hi - lo)) : 0.f;
    if (lane == 0) {
        a.drift[(int64_t)u * a.Cmax + c] = drift;
        if (a.drift_out) a.drift_out[(int64_t)u * a.C + c] = drift;
    }
}

// plan[u][c] = 2 * (new index of c) + (1 if c splits). count[u] = splits of unit u.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const SplitArgs a) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ int wsum[kPlanThreads / 32];
    __shared__ int carry;
    const int u = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t* off = a.offsets + (int64_t)u * a.off_ustride;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < a.C; base += kPlanThreads) {
        const int c = base + tid;
        bool f = false;
        if (c < a.C) {
            const int32_t lo = off[c], hi = off[c + 1];
            f = segment_ok(lo, hi, a.m) && hi - lo >= 2 && a.drift[(int64_t)u * a.Cmax + c] > a.tau;
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) wsum[warp] = __popc(bal);
        __syncthreads();
        int before = carry + __popc(bal & ((1u << lane) - 1u)), total = 0;
        for (int w = 0; w < kPlanThreads / 32; ++w) {
            if (w < warp) before += wsum[w];
            total += wsum[w];
        }
        if (c < a.C) {
            const bool kept = f && before < a.room;
            const int ni = c + min(before, a.room);
            a.plan[(int64_t)u * a.Cmax + c] = 2 * ni + (kept ? 1 : 0);
            if (kept) a.tasks[(int64_t)u * a.Cmax + before] = c;  // the unit's split list
        }
        __syncthreads();
        if (tid == 0) carry += total;
        __syncthreads();
    }
    if (tid == 0) a.count[u] = min(carry, a.room);
}

__global__ void __launch_bounds__(kSplitThreads) split_kmeans_kernel(const SplitArgs a) {
    pdl_launch_dependents();
    pdl_wait();
    const int k = blockIdx.x, u = blockIdx.y;
    if (k >= a.count[u]) return;  // whole CTA: fewer splits in this unit
    const int c = a.tasks[(int64_t)u * a.Cmax + k];
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint16_t* skey = (uint16_t*)smem_raw;                     // [kStageRows][128] bf16
    int32_t* slab = (int32_t*)(skey + (size_t)kStageRows * kD);  // [kStageRows]
    float* smu = (float*)(slab + kStageRows);                 // [2][128]
    float* smh = smu + 2 * kD;                                // [2][128] bf16 values as fp32
    float* sred = smh + 2 * kD;                               // [2 parts][2 halves][128]
    int32_t* sidx = (int32_t*)(sred + 4 * kD);                // [2] init rows
    int32_t* scnt = sidx + 2;                                 // [1] rows in the second half

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t* off = a.offsets + (int64_t)u * a.off_ustride;
    const int32_t lo = off[c], hi = off[c + 1], s = hi - lo;
    if (!segment_ok(lo, hi, a.m) || s < 2) {  // the plan only marks segments of 2+ rows
        if (tid == 0) atomicOr(a.err, kErrBadState);
        return;
    }
    const int64_t row0 = (int64_t)u * a.kp_ustride + lo;  // first row of the segment
    const uint16_t* gk = a.kp + row0 * kD;
    const bool staged = s <= kStageRows;
    if (staged)  // in logical order (stored row lo + t / 16)
        for (int t = tid; t < s * (kD / 8); t += kSplitThreads)
            reinterpret_cast<uint4*>(skey)[t] = reinterpret_cast<const uint4*>(gk)[(t & ~15) | swz(lo + (t >> 4), t & 15)];
    const uint16_t* rows = staged ? skey : gk;
    // offset of logical element d of segment row i in `rows`
    auto col = [&](int64_t i, int d) { return staged ? d : swz_elem(lo + i, d); };
    int32_t* lab = staged ? slab : a.lab + row0;
    if (tid == 0) {
        // first two entries of a Fisher-Yates shuffle of 0..s-1 (SplitMix64 draws mapped by
        // Lemire's multiply-shift): the first draw j0 is taken as is; the second j1 >= 1 lands
        // on j1 itself unless the first swap moved entry 0 there.
        uint64_t state = a.seed ^ ((uint64_t)(a.unit_base + u) << 32) ^ a.window_no;
        state ^= (uint64_t)(c + 1) * 0x9E3779B97F4A7C15ull;
        const int j0 = (int)bounded_draw(splitmix64_next(state), (uint32_t)s);
        const int j1 = 1 + (int)bounded_draw(splitmix64_next(state), (uint32_t)(s - 1));
        sidx[0] = j0;
        sidx[1] = j1 == j0 ? 0 : j1;
    }
    __syncthreads();
    {
        const int ch = tid >> 7, d = tid & (kD - 1);
        smu[ch * kD + d] = __uint_as_float((uint32_t)rows[(int64_t)sidx[ch] * kD + col(sidx[ch], d)] << 16);
    }
    __syncthreads();
    for (int it = 0; it < a.iters; ++it) {
        if (warp < 2) {  // normalise: mu_hat = bf16_rn(mu / |mu|), zero for a zero centroid
            const float4 v = reinterpret_cast<const float4*>(smu + warp * kD)[lane];
            const float nrm = __fsqrt_rn(warp_sum(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w));
            float4 h4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (nrm > 0.f) {
                h4.x = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.x, nrm)));
                h4.y = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.y, nrm)));
                h4.z = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.z, nrm)));
                h4.w = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.w, nrm)));
            }
            reinterpret_cast<float4*>(smh + warp * kD)[lane] = h4;
        }
        if (tid == 0) scnt[0] = 0;
        __syncthreads();
        // assign, one warp per row, four rows in flight: the second half wins only on a
        // strictly larger dot
        const float4 h0 = reinterpret_cast<const float4*>(smh)[lane];
        const float4 h1 = reinterpret_cast<const float4*>(smh + kD)[lane];
        constexpr int kNW = kSplitThreads / 32;
        for (int i0 = warp; i0 < s; i0 += 4 * kNW) {
            float p0[4], p1[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = i0 + r * kNW;
                p0[r] = p1[r] = 0.f;
                if (i < s) {
                    const uint2 w = *reinterpret_cast<const uint2*>(rows + (int64_t)i * kD + col(i, lane * 4));
                    const float k0 = bf16_lo(w.x), k1 = bf16_hi(w.x), k2 = bf16_lo(w.y),
                                k3 = bf16_hi(w.y);
                    p0[r] = fmaf(k3, h0.w, fmaf(k2, h0.z, fmaf(k1, h0.y, k0 * h0.x)));
                    p1[r] = fmaf(k3, h1.w, fmaf(k2, h1.z, fmaf(k1, h1.y, k0 * h1.x)));
                }
            }
            // the 8 lane sums (value 2 r: row r's dot with the first half, 2 r + 1: with the
            // second) reduced together: xor 16 keeps four values per lane, xor 8 two, xor 4
            // one, xor 2 and 1 finish; lane l ends with value l >> 2 (9 shuffles, not 40)
            float v[8];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                v[2 * r] = p0[r];
                v[2 * r + 1] = p1[r];
            }
#pragma unroll
            for (int half = 4; half >= 1; half >>= 1) {
                const bool up = (lane & (4 * half)) != 0;  // lane bits 4, 3, 2
#pragma unroll
                for (int t = 0; t < half; ++t) {
                    const float keep = up ? v[half + t] : v[t];
                    const float give = up ? v[t] : v[half + t];
                    v[t] = keep + __shfl_xor_sync(0xffffffffu, give, 4 * half);
                }
            }
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
            const float other = __shfl_xor_sync(0xffffffffu, v[0], 4);  // the row's other half
            int ones = 0;
            if ((lane & 7) == 0) {  // lane 8 r holds row r's first-half dot, lane 8 r + 4 its second
                const int r = lane >> 3, i = i0 + r * kNW;
                if (i < s) {
                    const int l = other > v[0] ? 1 : 0;
                    lab[i] = l;
                    ones = l;
                }
            }
            ones = __reduce_add_sync(0xffffffffu, ones);
            if (lane == 0 && ones) atomicAdd(scnt, ones);
        }
        __syncthreads();
        {  // update: thread (part, d) sums dimension d of both halves over the rows of its
           // parity (part 0: even rows, part 1: odd rows) in segment order; part 0 + part 1
            const int part = tid >> 7, d = tid & (kD - 1);
            float a0 = 0.f, a1 = 0.f;
            for (int j = part; j < s; j += 2) {
                const float v = __uint_as_float((uint32_t)rows[(int64_t)j * kD + col(j, d)] << 16);
                if (lab[j]) a1 += v;
                else a0 += v;
            }
            sred[(part * 2 + 0) * kD + d] = a0;
            sred[(part * 2 + 1) * kD + d] = a1;
        }
        __syncthreads();
        {
            const int ch = tid >> 7, d = tid & (kD - 1);
            const int cnt = ch ? scnt[0] : s - scnt[0];
            if (cnt > 0)  // an empty half keeps mu
                smu[ch * kD + d] = __fdiv_rn(sred[ch * kD + d] + sred[(2 + ch) * kD + d], (float)cnt);
        }
        __syncthreads();
    }
    const int n0 = s - scnt[0];
    // destination of every row: a stable partition (first half, then second half)
    if (warp == 0) {
        int c0 = 0, c1 = 0;
        const uint32_t lt = (1u << lane) - 1u;
        for (int b = 0; b < s; b += 32) {
            const int i = b + lane;
            const int l = i < s ? lab[i] : 2;
            const uint32_t m0 = __ballot_sync(0xffffffffu, l == 0);
            const uint32_t m1 = __ballot_sync(0xffffffffu, l == 1);
            if (i < s) lab[i] = l == 0 ? c0 + __popc(m0 & lt) : n0 + c1 + __popc(m1 & lt);
            c0 += __popc(m0);
            c1 += __popc(m1);
        }
    }
    // the segment's rows and ids into the row scratch (same rows), then back permuted
    uint16_t* rk = a.rk + row0 * kD;
    uint16_t* rv = a.rv + row0 * kD;
    int32_t* rid = a.rid + row0;
    uint16_t* kp = a.kp + row0 * kD;
    uint16_t* vp = a.vp + row0 * kD;
    int32_t* ids = a.ids + row0;
    for (int t = tid; t < s * (kD / 8); t += kSplitThreads) {
        reinterpret_cast<uint4*>(rk)[t] = reinterpret_cast<const uint4*>(kp)[t];
        reinterpret_cast<uint4*>(rv)[t] = reinterpret_cast<const uint4*>(vp)[t];
    }
    for (int i = tid; i < s; i += kSplitThreads) rid[i] = ids[i];
    __syncthreads();
    for (int t = tid; t < s * (kD / 8); t += kSplitThreads) {
        // stored chunk w of row lo + i holds logical chunk w ^ key(lo + i): it moves to row
        // lo + lab[i] at that logical chunk's position there
        const int i = t / (kD / 8), w = t % (kD / 8);
        const int64_t dst = (int64_t)lab[i] * (kD / 8) + swz(lo + lab[i], swz(lo + i, w));
        reinterpret_cast<uint4*>(kp)[dst] = reinterpret_cast<const uint4*>(rk)[t];
        reinterpret_cast<uint4*>(vp)[dst] = reinterpret_cast<const uint4*>(rv)[t];
    }
    for (int i = tid; i < s; i += kSplitThreads) ids[lab[i]] = rid[i];
    float* cmu = a.cmu + ((int64_t)u * a.Cmax + c) * 2 * kD;
    cmu[tid] = smu[tid];  // 256 threads = 2 halves x 128
    if (tid == 0) a.n0[(int64_t)u * a.Cmax + c] = n0;
}

// One warp per (cluster, unit): the cluster's centroid(s) and offset(s) into the scratch copy
// at the new index. The warps past the unit's last cluster write its empty padding clusters
// and the closing offset.
__global__ void __launch_bounds__(kDriftWarps * 32) scatter_kernel(const SplitArgs a) {
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.y, c = blockIdx.x * kDriftWarps + warp;
    const int Cu = a.C + a.count[u], Cn = a.C + a.room;
    const int32_t* off = a.offsets + (int64_t)u * a.off_ustride;
    float4* mu2 = reinterpret_cast<float4*>(a.mu2 + (int64_t)u * a.Cmax * kD);
    int32_t* off2 = a.off2 + (int64_t)u * (a.Cmax + 1);
    if (c < a.C) {
        const int p = a.plan[(int64_t)u * a.Cmax + c];
        const int ni = p >> 1;
        if (p & 1) {
            const float4* cm = reinterpret_cast<const float4*>(a.cmu + ((int64_t)u * a.Cmax + c) * 2 * kD);
            mu2[(int64_t)ni * (kD / 4) + lane] = cm[lane];
            mu2[(int64_t)(ni + 1) * (kD / 4) + lane] = cm[kD / 4 + lane];
            if (lane == 0) {
                off2[ni] = off[c];
                off2[ni + 1] = off[c] + a.n0[(int64_t)u * a.Cmax + c];
            }
        } else {
            mu2[(int64_t)ni * (kD / 4) + lane] =
                reinterpret_cast<const float4*>(a.mu + ((int64_t)u * a.mu_ustride + c) * kD)[lane];
            if (lane == 0) off2[ni] = off[c];
        }
    } else {
        const int c2 = Cu + (c - a.C);  // padding cluster c2, or the closing offset at Cn
        if (c2 < Cn) mu2[(int64_t)c2 * (kD / 4) + lane] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c2 <= Cn && lane == 0) off2[c2] = (int32_t)a.m;
    }
}

// The scratch copy back into the store: clusters [0, Cn) and offsets [0, Cn].
__global__ void __launch_bounds__(kDriftWarps * 32) copy_back_kernel(const SplitArgs a) {
    // The last kernel of a split: no early trigger, so a following decode kernel, which reads
    // the cluster store before its dependency wait, starts once the store is complete.
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.y, c = blockIdx.x * kDriftWarps + warp;
    const int Cn = a.C + a.room;
    if (c > Cn) return;
    if (c < Cn)
        reinterpret_cast<float4*>(a.mu + ((int64_t)u * a.mu_ustride + c) * kD)[lane] =
            reinterpret_cast<const float4*>(a.mu2 + ((int64_t)u * a.Cmax + c) * kD)[lane];
    if (lane == 0)
        a.offsets[(int64_t)u * a.off_ustride + c] = a.off2[(int64_t)u * (a.Cmax + 1) + c];
}

}  // namespace

int launch_split(const SplitArgs& a, cudaStream_t s) {
    if (a.C < 1 || a.U < 1 || a.iters < 1 || a.room < 0) {
        set_error("split: bad sizes");
        return CKV_EINVAL;
    }
    cudaError_t e = launch_pdl(drift_kernel, dim3((a.C + kDriftWarps - 1) / kDriftWarps, a.U),
                               dim3(kDriftWarps * 32), 0, s, a);
    if (e != cudaSuccess) return cuda_fail(e, "split: drift launch");
    e = launch_pdl(plan_kernel, dim3(a.U), dim3(kPlanThreads), 0, s, a);
    if (e != cudaSuccess) return cuda_fail(e, "split: plan launch");
    const size_t smem = (size_t)kStageRows * kD * 2 + (size_t)kStageRows * 4 + 8 * kD * 4 + 16;
    const int rc = ensure_smem((const void*)split_kmeans_kernel, smem, "split: set smem");
    if (rc != CKV_OK) return rc;
    if (a.room > 0) {
        e = launch_pdl(split_kmeans_kernel, dim3(a.room, a.U), dim3(kSplitThreads), smem, s, a);
        if (e != cudaSuccess) return cuda_fail(e, "split: kmeans launch");
    }
    // grids cover every cluster a unit ends with (C + room) plus the closing offset
    const dim3 gw((a.C + a.room + 1 + kDriftWarps - 1) / kDriftWarps, a.U);
    e = launch_pdl(scatter_kernel, gw, dim3(kDriftWarps * 32), 0, s, a);
    if (e != cudaSuccess) return cuda_fail(e, "split: scatter launch");
    e = launch_pdl(copy_back_kernel, gw, dim3(kDriftWarps * 32), 0, s, a);
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "split: copy launch");
}

}  // namespace ckv
