// fp8 (e4m3) copy of the clustered K and V rows, for attending far clusters at lower
// precision (sm_100a).
//
// Page: "大模型KV Cache压缩技术：ClusterKV的语义空间优化" (ClusterKV explainer), section 7 (outlook):
// a lower-precision KV cache for clusters far from the current query. The page gives no
// format; the reading here: every clustered row keeps, next to its bf16 values, an fp8 e4m3
// copy with one fp32 scale per row, scale = max|x| / 448 (fp32 division), code =
// e4m3(x / scale) rounded to nearest, ties to even, saturating at 448, both steps in fp32.
// A zero row has scale 0 and zero codes. The dequantised value is e4m3(code) * scale.
//
// One warp per row: lane l holds elements 4 l .. 4 l + 3 (one 8-byte load), the row maximum
// is a warp reduction, and the four codes leave as one 4-byte store; lane 0 writes the scale.
#include <cuda_fp8.h>

#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

constexpr int kQuantWarps = 8;

CKV_DEV uint32_t quantize4(uint2 w, float* scale_out) {
    const float x0 = bf16_lo(w.x), x1 = bf16_hi(w.x), x2 = bf16_lo(w.y), x3 = bf16_hi(w.y);
    float mx = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float scale = __fdiv_rn(mx, 448.0f);
    *scale_out = scale;
    if (!(scale > 0.f)) return 0u;
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(x0, scale), __fdiv_rn(x1, scale)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(x2, scale), __fdiv_rn(x3, scale)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// Rows [r0, r0 + nrows) of every unit u < U: kp/vp [U][ustride][128] bf16 ->
// kp8/vp8 [U][ustride][128] e4m3, ks/vs [U][ustride] fp32.
__global__ void __launch_bounds__(kQuantWarps * 32) quantize_rows_kernel(
    const uint16_t* kp, const uint16_t* vp, uint8_t* kp8, uint8_t* vp8, float* ks, float* vs,
    int64_t ustride, int64_t r0, int64_t nrows, int32_t U) {
    // No early trigger: this kernel ends the calls that write the cluster store when the fp8
    // copy is kept, and the decode kernel reads the store before its dependency wait.
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t total = nrows * U;
    for (int64_t w = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5); w < total;
         w += (int64_t)gridDim.x * kQuantWarps) {  // warp-uniform trip count
        const int64_t u = w / nrows, r = r0 + w % nrows;
        const int64_t row = u * ustride + r;
        float sk, sv;
        const uint32_t ck = quantize4(reinterpret_cast<const uint2*>(kp + row * kD)[lane], &sk);
        const uint32_t cv = quantize4(reinterpret_cast<const uint2*>(vp + row * kD)[lane], &sv);
        reinterpret_cast<uint32_t*>(kp8 + row * kD)[lane] = ck;
        reinterpret_cast<uint32_t*>(vp8 + row * kD)[lane] = cv;
        if (lane == 0) {
            ks[row] = sk;
            vs[row] = sv;
        }
    }
}

}  // namespace

int launch_quantize_rows(const uint16_t* kp, const uint16_t* vp, uint8_t* kp8, uint8_t* vp8,
                         float* ks, float* vs, int64_t ustride, int64_t r0, int64_t nrows,
                         int32_t U, cudaStream_t s) {
    if (nrows <= 0 || U <= 0) return CKV_OK;
    const int64_t warps = nrows * U;
    const int64_t want = (warps + kQuantWarps - 1) / kQuantWarps;
    const int grid = (int)(want < 8 * 148 ? want : 8 * 148);
    cudaError_t e = launch_pdl(quantize_rows_kernel, dim3(grid), dim3(kQuantWarps * 32), 0, s, kp,
                               vp, kp8, vp8, ks, vs, ustride, r0, nrows, U);
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "fp8 copy: launch");
}

}  // namespace ckv
