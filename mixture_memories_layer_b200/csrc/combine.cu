// Combine and un-permute ("MoM: Linear Sequence Modeling with
// Mixture-of-Memories", Summary: outputs are combined with the router
// weights; the authors' blog post, hardware-efficient implementation:
// summing the weighted per-memory outputs equals reading the mixed memory):
//
//   out[t] = o_sh[t] + sum_j gate[t, j] * o_p[row_of[t*K + j]]
//
// HBM-bound: one thread per 8 output elements, 16-byte (bf16) or 2x16-byte
// (f32) loads and stores; float32 arithmetic.
#include "common.cuh"
#include "kernels.h"

namespace mom {

template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ o_sh, const T* __restrict__ o_p, const int32_t* __restrict__ row_of,
               const float* __restrict__ gate, int64_t n_tok, int K, int HD, T* __restrict__ out, void* ws) {
    const int per_tok = HD / 8;
    const int64_t total = n_tok * per_tok;
    const int64_t n_rows = n_tok * K;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_tok;
        const int c = (int)(i % per_tok) * 8;
        float acc[8], v[8];
        load_vec<8>(o_sh + t * HD + c, acc);
        for (int j = 0; j < K; ++j) {
            const int64_t r = row_of[t * K + j];
            if (r < 0 || r >= n_rows) { record_error(ws, MOM_DEVERR_ROW_INDEX, t); continue; }
            const float g = gate[t * K + j];
            load_vec<8>(o_p + r * HD + c, v);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(g, v[e], acc[e]);
        }
        store_vec<8>(out + t * HD + c, acc);
    }
}

cudaError_t launch_combine(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                           int64_t n_tok, int K, int H, int d, int dt, void* out, void* ws, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    const int HD = H * d;
    const int64_t total = n_tok * (HD / 8);
    int64_t g = cdiv(total, 256);
    if (g > 148 * 32) g = 148 * 32;
    if (dt == MOM_BF16)
        combine_kernel<bf16><<<(unsigned)g, 256, 0, st>>>((const bf16*)o_sh, (const bf16*)o_p, row_of, gate, n_tok, K, HD, (bf16*)out, ws);
    else
        combine_kernel<float><<<(unsigned)g, 256, 0, st>>>((const float*)o_sh, (const float*)o_p, row_of, gate, n_tok, K, HD, (float*)out, ws);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
