// K-means centroid update that allocates no device memory.
//
// Some callers cannot allocate device memory around this library. Three examples: an
// inference engine that takes all of its device memory from its own pool at start-up and
// treats any later allocation as a fault; a decode loop that must never stall, since
// cudaMalloc and cudaFree can synchronise the device; a plugin that runs inside a host
// application which owns the device memory. The regular stage call ckv_kmeans_update needs
// a context, and creating a context allocates its workspace. This variant runs the same
// update kernels (counting sort by cluster, then the mean of each cluster) without a
// context. Their only scratch buffer is the per-chunk cluster counts of the counting sort,
// and here it lives in a fixed-size array compiled into the library.
//
// The array is a file-scope __device__ array, so every GPU that loads the library holds it
// until the process exits. Its device address is looked up once per device, on that
// device's first call, with cudaGetSymbolAddress (host code cannot use the symbol itself
// as a device pointer). All calls on a device share the array. Calls whose kernels overlap
// on the GPU (for example on two streams) race on it. Every count the kernels read is
// written earlier in the same call, so the previous call's contents never leak into a
// result.
#include <mutex>
#include <string>

#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

// 2^21 int32 counts = 8 MiB per device. One call needs U * ceil(m / 1024) * C of them:
// for example 8 units of 32752 keys with C = 400 need 102400, and 8 units of 131056 keys
// with C = 1600 need 1638400.
constexpr int64_t kScratchInts = (int64_t)1 << 21;
static __device__ __align__(256) int32_t g_update_scratch[kScratchInts];

int scratch_address(int32_t** out) {
    static std::mutex mtx;
    static int32_t* addr[256] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "kmeans_update_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= 256) {
        set_error("kmeans_update_noalloc: device index out of range");
        return CKV_EINVAL;
    }
    std::lock_guard<std::mutex> lock(mtx);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_update_scratch);
        if (e != cudaSuccess || !p) {
            return cuda_fail(e == cudaSuccess ? cudaErrorInvalidSymbol : e,
                             "kmeans_update_noalloc: cudaGetSymbolAddress");
        }
        addr[dev] = (int32_t*)p;
    }
    *out = addr[dev];
    return CKV_OK;
}

bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

int bad(const std::string& m) {
    set_error("kmeans_update_noalloc: " + m);
    return CKV_EINVAL;
}

}  // namespace
}  // namespace ckv

using namespace ckv;

extern "C" int ckv_kmeans_update_noalloc(const void* keys, int64_t n_rows, int64_t row0, int64_t m,
                                         int32_t U, const int32_t* assign, int32_t C, float* mu,
                                         void* mu_hat, int32_t* offsets, int32_t* perm,
                                         void* stream) {
    if (!aligned16(keys)) return bad("keys must be non-null and 16-byte aligned");
    if (!assign || !aligned16(mu) || !aligned16(mu_hat) || !offsets || !perm)
        return bad("null or misaligned output");
    if (U < 1) return bad("U must be >= 1");
    if (m < 1 || m > (int64_t)INT32_MAX / 2) return bad("m out of range");
    if (row0 < 0 || row0 + m > n_rows) return bad("rows [row0, row0+m) exceed n_rows");
    if (C < 1 || C > CKV_MAX_CLUSTERS || C > m) return bad("C must be in 1..min(4096, m)");
    const int64_t need = (int64_t)U * n_chunks(m) * C;
    if (need > kScratchInts) {
        return bad("needs " + std::to_string(need) + " int32 counts of scratch (U * ceil(m/1024) * C)"
                   "; the fixed array holds " + std::to_string(kScratchInts));
    }
    int32_t* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != CKV_OK) return rc;
    KeysView kv{(const uint16_t*)keys, n_rows, row0, m, U};
    return launch_kmeans_update(kv, assign, m, C, mu, C, (uint16_t*)mu_hat, C, offsets, C + 1, perm,
                                m, scratch, nullptr, nullptr, (cudaStream_t)stream);
}
