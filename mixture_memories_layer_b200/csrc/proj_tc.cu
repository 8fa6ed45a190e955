// Grouped projections on the tcgen05 tensor cores (bf16).  Placeholder until
// the tensor-core GEMM lands: reports every shape as unsupported, so the
// CUDA-core kernel runs.
#include "common.cuh"
#include "kernels.h"

namespace mom {
bool proj_tc_supported(const ProjArgs&, int) { return false; }
cudaError_t launch_proj_tc(const ProjArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace mom
