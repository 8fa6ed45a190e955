// Combine and un-permute ("MoM: Linear Sequence Modeling with
// Mixture-of-Memories", Summary: outputs are combined with the router
// weights; the authors' blog post, hardware-efficient implementation:
// summing the weighted per-memory outputs equals reading the mixed memory):
//
//   out[t] = o_sh[t] + sum_j gate[t, j] * o_p[row_of[t*K + j]]
//
// HBM-bound: 16-byte (bf16) or 2x16-byte (f32) loads and stores, float32
// arithmetic.
#include "common.cuh"
#include "kernels.h"

namespace mom {

// One thread per 8 output elements, no loop: the router slots' rows and
// gates are read first, then the shared output and all K memory rows are
// in flight together (top_k <= KMAX per pass).
template <typename T, int KMAX>
__global__ void __launch_bounds__(256, 4)
combine_kernel(const T* __restrict__ o_sh, const T* __restrict__ o_p, const int32_t* __restrict__ row_of,
               const float* __restrict__ gate, int64_t n_tok, int K, int HD, T* __restrict__ out, void* ws) {
    const int per_tok = HD / 8;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_tok * per_tok) return;
    const int64_t n_rows = n_tok * K;
    const int64_t t = i / per_tok;
    const int c = (int)(i % per_tok) * 8;
    float acc[8];
    load_vec<8>(o_sh + t * HD + c, acc);
    for (int j0 = 0; j0 < K; j0 += KMAX) {
        int64_t r[KMAX];
        float g[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            r[j] = -1;
            g[j] = 0.f;
            if (j0 + j < K) {
                r[j] = __ldg(row_of + t * K + j0 + j);
                g[j] = __ldg(gate + t * K + j0 + j);
                if (r[j] < 0 || r[j] >= n_rows) {
                    record_error(ws, MOM_DEVERR_ROW_INDEX, t);
                    r[j] = -1;
                }
            }
        }
        float v[KMAX][8];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (r[j] >= 0) load_vec<8>(o_p + r[j] * HD + c, v[j]);
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (r[j] >= 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(g[j], v[j][e], acc[e]);
            }
        }
    }
    store_vec<8>(out + t * HD + c, acc);
}

cudaError_t launch_combine(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                           int64_t n_tok, int K, int H, int d, int dt, void* out, void* ws, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    const int HD = H * d;
    const int64_t total = n_tok * (HD / 8);
    const unsigned g = (unsigned)cdiv(total, 256);
    if (dt == MOM_BF16) {
        if (K <= 2)
            combine_kernel<bf16, 2><<<g, 256, 0, st>>>((const bf16*)o_sh, (const bf16*)o_p, row_of, gate, n_tok, K, HD, (bf16*)out, ws);
        else
            combine_kernel<bf16, 4><<<g, 256, 0, st>>>((const bf16*)o_sh, (const bf16*)o_p, row_of, gate, n_tok, K, HD, (bf16*)out, ws);
    } else {
        if (K <= 2)
            combine_kernel<float, 2><<<g, 256, 0, st>>>((const float*)o_sh, (const float*)o_p, row_of, gate, n_tok, K, HD, (float*)out, ws);
        else
            combine_kernel<float, 4><<<g, 256, 0, st>>>((const float*)o_sh, (const float*)o_p, row_of, gate, n_tok, K, HD, (float*)out, ws);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
