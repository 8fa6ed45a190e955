// Chunked Gated DeltaNet on the tcgen05 tensor cores (bf16).  Placeholder
// until the tensor-core kernel lands: reports every shape as unsupported, so
// the token-serial CUDA-core kernel runs.
#include "common.cuh"
#include "kernels.h"

namespace mom {
bool gdn_tc_supported(const GdnArgs&, int) { return false; }
size_t gdn_tc_ws_bytes(int64_t, int, int, int) { return 0; }
cudaError_t launch_gdn_tc(const GdnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace mom
