// Incremental clustering and token append for ClusterKV decode (sm_100a).
//
// Page: "大模型KV Cache压缩技术：ClusterKV的语义空间优化" (ClusterKV explainer), section 3.2:
// after every 320 generated tokens an incremental clustering runs. Reading: cosine K-means
// with 4 clusters and 10 Lloyd iterations on those 320 pending tokens alone. The init is the
// prefill rule, keyed by (seed, unit, window number). The new clusters are appended after the
// existing ones, which are left unchanged.
//
// The window is read from the pending ring (two windows of rows after the sinks: the one being
// clustered and the one still filling) at the row the host passes.
//
// The window is small (320 x 128 bf16 = 80 KB), so one CTA per unit runs the whole clustering
// in shared memory: init, 10 x (normalise, assign, stable counting sort, mean), then it writes
// the permuted K/V rows, their token ids, the new offsets and the new centroids into the
// cluster store. Assignment uses fp32 FMA over the bf16 operands (the same products as the
// prefill tensor-core path, with fp32 accumulation).
#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

constexpr int kRT = 512;

__global__ void __launch_bounds__(kRT) recluster_kernel(const ReclusterArgs a) {
    // No early trigger: this kernel writes the cluster store (new rows, offsets and
    // centroids), which the decode kernel reads before its dependency wait.
    pdl_wait();               // the previous kernel's writes are visible from here on
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int W = a.window, Cn = a.C_new;
    uint16_t* skey = (uint16_t*)smem_raw;                         // [W][128] bf16
    float* smu = (float*)(skey + (size_t)W * kD);                 // [Cn][128]
    float* smh = smu + Cn * kD;                                   // [Cn][128] bf16 values as fp32
    int32_t* sasg = (int32_t*)(smh + Cn * kD);                    // [W]
    int32_t* sperm = sasg + W;                                    // [W]
    int32_t* sarr = sperm + W;                                    // [W] Fisher-Yates array
    int32_t* soff = sarr + W;                                     // [Cn + 1]
    int32_t* scnt = soff + Cn + 1;                                // [Cn]

    const int u = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = kRT / 32;
    const uint16_t* wk = a.spk + ((int64_t)u * a.sp_ustride + a.win_row0) * kD;
    const uint16_t* wv = a.spv + ((int64_t)u * a.sp_ustride + a.win_row0) * kD;
    // window keys into shared memory, in logical order (stored row win_row0 + i / 16)
    for (int i = tid; i < W * kD / 8; i += kRT)
        reinterpret_cast<uint4*>(skey)[i] =
            reinterpret_cast<const uint4*>(wk)[(i & ~15) | swz(a.win_row0 + (i >> 4), i & 15)];
    for (int i = tid; i < W; i += kRT) sarr[i] = i;
    __syncthreads();
    if (tid == 0) {
        uint64_t state = a.seed ^ ((uint64_t)(a.unit_base + u) << 32) ^ a.window_no;
        for (int i = 0; i < Cn; ++i) {
            const uint64_t x = splitmix64_next(state);
            const int j = i + (int)bounded_draw(x, (uint32_t)(W - i));
            const int t = sarr[i];
            sarr[i] = sarr[j];
            sarr[j] = t;
        }
    }
    __syncthreads();
    for (int t = tid; t < Cn * kD; t += kRT) {
        const int c = t / kD, d = t % kD;
        smu[t] = __uint_as_float((uint32_t)skey[sarr[c] * kD + d] << 16);
    }
    __syncthreads();

    float* mtrace = a.mu_trace ? a.mu_trace + (int64_t)u * (a.iters + 1) * Cn * kD : nullptr;
    int32_t* atrace = a.assign_trace ? a.assign_trace + (int64_t)u * a.iters * W : nullptr;

    for (int it = 0; it < a.iters; ++it) {
        if (mtrace)
            for (int t = tid; t < Cn * kD; t += kRT) mtrace[(int64_t)it * Cn * kD + t] = smu[t];
        // normalise: mu_hat = bf16_rn(mu / |mu|)
        for (int c = warp; c < Cn; c += nw) {
            const float4 v = reinterpret_cast<const float4*>(smu + c * kD)[lane];
            float ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float nrm = __fsqrt_rn(ss);
            float4 h4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (nrm > 0.f) {
                h4.x = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.x, nrm)));
                h4.y = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.y, nrm)));
                h4.z = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.z, nrm)));
                h4.w = __bfloat162float(__float2bfloat16_rn(__fdiv_rn(v.w, nrm)));
            }
            reinterpret_cast<float4*>(smh + c * kD)[lane] = h4;
        }
        if (tid < Cn) scnt[tid] = 0;
        __syncthreads();
        // assign (ties: lower c). Thread i walks its key row's 64 words starting at word
        // (i mod 32), so the 32 lanes of a warp, each on its own row, read 32 different banks
        // at every step (rows are 256 bytes apart: the same word of each would share a bank).
        for (int i = tid; i < W; i += kRT) {
            const uint32_t* kw = reinterpret_cast<const uint32_t*>(skey + i * kD);
            const int rot = i & 31;
            float best = -INFINITY;
            int bi = 0;
            for (int c = 0; c < Cn; ++c) {
                const float2* m2 = reinterpret_cast<const float2*>(smh + c * kD);
                float s = 0.f;
                for (int t = 0; t < kD / 2; ++t) {
                    const int wi = (t + rot) & (kD / 2 - 1);
                    const uint32_t w = kw[wi];
                    const float2 mm = m2[wi];
                    s = fmaf(bf16_lo(w), mm.x, s);
                    s = fmaf(bf16_hi(w), mm.y, s);
                }
                if (s > best) {
                    best = s;
                    bi = c;
                }
            }
            sasg[i] = bi;
            atomicAdd(&scnt[bi], 1);
            if (atrace) atrace[(int64_t)it * W + i] = bi;
        }
        __syncthreads();
        if (tid == 0) {
            int run = 0;
            for (int c = 0; c < Cn; ++c) {
                soff[c] = run;
                run += scnt[c];
            }
            soff[Cn] = run;
        }
        __syncthreads();
        // stable counting sort: position = offset + number of earlier keys in the cluster
        for (int i = tid; i < W; i += kRT) {
            const int c = sasg[i];
            int before = 0;
            for (int j = 0; j < i; ++j) before += sasg[j] == c;
            sperm[soff[c] + before] = i;
        }
        __syncthreads();
        // mean in member order; empty clusters keep mu
        for (int t = tid; t < Cn * kD; t += kRT) {
            const int c = t / kD, d = t % kD;
            const int lo = soff[c], hi = soff[c + 1];
            if (hi > lo) {
                float acc = 0.f;
                for (int j = lo; j < hi; ++j)
                    acc += __uint_as_float((uint32_t)skey[sperm[j] * kD + d] << 16);
                smu[t] = __fdiv_rn(acc, (float)(hi - lo));
            }
        }
        __syncthreads();
    }
    if (mtrace)
        for (int t = tid; t < Cn * kD; t += kRT) mtrace[(int64_t)a.iters * Cn * kD + t] = smu[t];

    // append to the store
    const int64_t row0 = (int64_t)u * a.kp_ustride + a.m_old;
    for (int t = tid; t < W * (kD / 8); t += kRT) {  // stored row m_old + j, logical chunk w
        const int j = t / (kD / 8), w = t % (kD / 8);
        const int src = sperm[j];
        const int o = swz(a.m_old + j, w);
        reinterpret_cast<uint4*>(a.kp + (row0 + j) * kD)[o] =
            reinterpret_cast<const uint4*>(skey + src * kD)[w];
        reinterpret_cast<uint4*>(a.vp + (row0 + j) * kD)[o] =
            reinterpret_cast<const uint4*>(wv + (int64_t)src * kD)[swz(a.win_row0 + src, w)];
    }
    for (int j = tid; j < W; j += kRT) a.ids[row0 + j] = (int32_t)(a.n_sink + a.m_old + sperm[j]);
    int32_t* off = a.offsets + (int64_t)u * a.off_ustride;
    for (int c = tid; c <= Cn; c += kRT) off[a.C_old + c] = (int32_t)(a.m_old + soff[c]);
    float* mu = a.mu + ((int64_t)u * a.mu_ustride + a.C_old) * kD;
    for (int t = tid; t < Cn * kD; t += kRT) mu[t] = smu[t];
}

__global__ void append_kernel(const uint16_t* k, const uint16_t* v, uint16_t* spk, uint16_t* spv,
                              int64_t sp_ustride, int32_t row) {
    pdl_launch_dependents();  // let the next kernel in the stream be scheduled early
    pdl_wait();               // the previous kernel's writes are visible from here on
    const int u = blockIdx.x, t = threadIdx.x;  // 16 threads x 16 bytes per row
    const int64_t dst = ((int64_t)u * sp_ustride + row) * kD;  // stored row `row`
    reinterpret_cast<uint4*>(spk + dst)[swz(row, t)] = reinterpret_cast<const uint4*>(k + (int64_t)u * kD)[t];
    reinterpret_cast<uint4*>(spv + dst)[swz(row, t)] = reinterpret_cast<const uint4*>(v + (int64_t)u * kD)[t];
}

}  // namespace

int launch_recluster(const ReclusterArgs& a, cudaStream_t s) {
    const size_t smem = (size_t)a.window * kD * 2 + (size_t)a.C_new * kD * 4 * 2 +
                        (size_t)a.window * 4 * 3 + (size_t)(2 * a.C_new + 1) * 4 + 16;
    if (smem > 227 * 1024) {
        set_error("recluster: window too large for shared memory");
        return CKV_EINVAL;
    }
    const int rc = ensure_smem((const void*)recluster_kernel, smem, "recluster: set smem");
    if (rc != CKV_OK) return rc;
    cudaError_t e = launch_pdl(recluster_kernel, dim3(a.U), dim3(kRT), smem, s, a);
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "recluster: launch");
}

int launch_append(const uint16_t* k, const uint16_t* v, int32_t U, uint16_t* spk, uint16_t* spv,
                  int64_t sp_ustride_rows, int32_t row, cudaStream_t s) {
    cudaError_t e = launch_pdl(append_kernel, dim3(U), dim3(16), 0, s, k, v, spk, spv,
                               sp_ustride_rows, row);
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "append: launch");
}

}  // namespace ckv
