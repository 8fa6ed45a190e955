// Row copies with an optional gather index, in 16-byte granules: the packing
// and unpacking of the routed rows a memory-parallel layer sends to the ranks
// that own their memories (memory count scaling: "MoM: Mixture-of-Memories
// Fixes Linear Attention Recall", Memory count scaling).  One warp per row,
// each lane moving 16 bytes per step: HBM-bound, coalesced on both sides.
#include "common.cuh"
#include "kernels.h"

namespace mom {
namespace {

__global__ void __launch_bounds__(256)
copy_rows_kernel(const unsigned char* __restrict__ src, int64_t n_src, int64_t src_stride, int64_t src_off,
                 const int32_t* __restrict__ idx, int64_t n_rows, int64_t row_bytes, unsigned char* __restrict__ dst,
                 int64_t dst_stride, int64_t dst_off, void* err) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t chunks = row_bytes >> 4;
    for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n_rows; i += warps) {
        int64_t s = idx ? (int64_t)idx[i] : i;
        if (s < 0 || s >= n_src) {
            if (lane == 0) record_error(err, MOM_DEVERR_ROW_INDEX, i);
            s = -1;
        }
        const uint4* from = reinterpret_cast<const uint4*>(src + (s >= 0 ? s : 0) * src_stride + src_off);
        uint4* to = reinterpret_cast<uint4*>(dst + i * dst_stride + dst_off);
        for (int64_t c = lane; c < chunks; c += 32) to[c] = s >= 0 ? __ldg(from + c) : make_uint4(0, 0, 0, 0);
    }
}

}  // namespace

cudaError_t launch_copy_rows(const void* src, int64_t n_src, int64_t src_stride, int64_t src_off, const int32_t* idx,
                             int64_t n_rows, int64_t row_bytes, void* dst, int64_t dst_stride, int64_t dst_off,
                             void* err, cudaStream_t st) {
    if (n_rows == 0 || row_bytes == 0) return cudaSuccess;
    const int64_t want = cdiv(n_rows, 8);
    const unsigned grid = (unsigned)(want < 148 * 8 ? want : 148 * 8);
    copy_rows_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const unsigned char*>(src), n_src, src_stride, src_off,
                                           idx, n_rows, row_bytes, reinterpret_cast<unsigned char*>(dst), dst_stride,
                                           dst_off, err);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
