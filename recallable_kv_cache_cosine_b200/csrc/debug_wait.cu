// Test hook for the library's failure detection: one bounded device wait that runs out.
//
// Every wait in the library's kernels (on an mbarrier that a bulk copy, a TMA load or a
// tensor-core commit completes) gives up after a time limit, sets the device error word and
// lets the kernel unwind, so that a lost arrival surfaces as CKV_ETIMEOUT from
// ckv_check_device_error instead of a hung GPU. In normal operation those waits never run
// out. This kernel makes one run out on purpose, without faulting anything: one thread
// initialises an mbarrier that expects one arrival, issues no copy and never arrives, and
// waits on it with the given limit. When the limit passes it sets the error word and
// returns. No asynchronous copy is outstanding, so the CTA may exit at once.
#include "ckv_common.cuh"
#include "ckv_internal.h"

namespace ckv {
namespace {

__global__ void expire_wait_kernel(uint32_t* err, uint64_t limit_ns, uint32_t* waited_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const uint64_t t0 = globaltimer();
    const bool ok = mbar_wait_for(&bar, 0, err, limit_ns);  // nothing arrives: runs out
    const uint64_t dt = globaltimer() - t0;
    if (waited_ns) *waited_ns = (uint32_t)(dt < 0xFFFFFFFFull ? dt : 0xFFFFFFFFull);
    if (ok && err) atomicOr(err, kErrBadState);  // an arrival nobody made: report it
}

}  // namespace

int launch_expire_wait(uint32_t* err, uint64_t limit_ns, uint32_t* waited_ns, cudaStream_t s) {
    expire_wait_kernel<<<1, 32, 0, s>>>(err, limit_ns, waited_ns);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? CKV_OK : cuda_fail(e, "expire_wait: launch");
}

}  // namespace ckv
