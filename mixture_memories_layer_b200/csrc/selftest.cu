// Self-test of the failure path that every pipelined kernel of the library
// shares: a bounded barrier wait that runs out.  One thread initialises a
// barrier, then waits on it with mbar_wait_limit -- the wait mbar_wait is
// made of -- while nothing ever arrives.  When the limit passes, the wait
// raises the CTA's abort flag and records MOM_DEVERR_TIMEOUT in the
// workspace's error record, and the kernel returns normally: no trap, no
// fault, the context stays usable.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mom {
namespace {

using namespace sm100;

__global__ void wait_timeout_kernel(void* err, long long limit) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_barrier_init();
    abort_flag = 0;
    // phase 0 never completes: nobody arrives
    (void)mbar_wait_limit(b, 0, &abort_flag, err, MOM_SELFTEST_WAIT_SITE, limit);
}

}  // namespace
}  // namespace mom

extern "C" mom_status mom_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t limit_cycles, void* stream) {
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (limit_cycles < 1 || limit_cycles > 4000000000LL) return MOM_ERR_ARG;
    mom::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ws, (long long)limit_cycles);
    mom::count_launches(1);
    return cudaGetLastError() == cudaSuccess ? MOM_OK : MOM_ERR_CUDA;
}
