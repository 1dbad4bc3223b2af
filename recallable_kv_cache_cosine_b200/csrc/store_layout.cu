// The chunk order of stored rows: every stored K/V row keeps its logical chunk c at chunk
// position c ^ (r & 7), r = the row's index from its unit's first row (16-byte chunks of bf16
// rows, 8-byte units of fp8 rows). The map is its own inverse, so one in-place pass turns a
// run of rows from logical into stored order and back; the import and export calls use it.
#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

constexpr int kSwzRows = 8;  // rows per block, a warp each

template <typename Unit>
__global__ void __launch_bounds__(kSwzRows * 32) swizzle_rows_kernel(Unit* rows, int64_t r0, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * kSwzRows + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (i >= n) return;  // warp-uniform
    Unit* row = rows + i * 16;
    Unit v{};
    if (lane < 16) v = row[lane];
    __syncwarp();  // every unit is read before any is written
    if (lane < 16) row[swz(r0 + i, lane)] = v;
}

}  // namespace

int launch_swizzle_rows(void* rows, int32_t unit_bytes, int64_t r0, int64_t n, cudaStream_t s) {
    if (n <= 0) return CKV_OK;
    const dim3 grid((unsigned)((n + kSwzRows - 1) / kSwzRows));
    if (unit_bytes == 16)
        swizzle_rows_kernel<uint4><<<grid, kSwzRows * 32, 0, s>>>((uint4*)rows, r0, n);
    else
        swizzle_rows_kernel<uint2><<<grid, kSwzRows * 32, 0, s>>>((uint2*)rows, r0, n);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "swizzle rows: launch");
}

}  // namespace ckv
