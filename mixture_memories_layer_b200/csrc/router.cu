// Router (one matmul, one softmax, one top-k, one renormalisation -- "MoM:
// Mixture-of-Memories Fixes Linear Attention Recall", Router mechanics, step
// by step) and the per-token gate projections beta / log alpha.
//
// Both are skinny products x W^T with at most a few dozen output columns:
// HBM-bound on reading x once.  One warp per token: each lane takes 8
// consecutive features per step (one 16-byte load of bf16), keeps one
// partial sum per output column, and the warp butterfly-reduces them.  The
// weights (<= 64 KB) stay in L1/L2.
#include "common.cuh"
#include "kernels.h"

namespace mom {

// Partial dot products of one token row with NC weight rows, reduced across
// the warp.  Every lane ends with all NC sums.  ncol <= NC.
template <typename T, int NC>
__device__ __forceinline__ void warp_row_dots(const T* __restrict__ xr, const T* __restrict__ w,
                                              int ncol, int D, int lane, float* acc) {
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[c] = 0.f;
    for (int f = lane * 8; f < D; f += 256) {
        float xv[8];
        load_vec<8>(xr + f, xv);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            if (c < ncol) {
                float wv[8];
                load_vec<8>(w + (size_t)c * D + f, wv);
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) s = fmaf(xv[i], wv[i], s);
                acc[c] += s;
            }
        }
    }
    warp_sum_n<NC>(acc);
}

template <typename T, int MAXM>
__global__ void __launch_bounds__(256)
router_topk_kernel(const T* __restrict__ x, const T* __restrict__ w_r, const float* __restrict__ b_r,
                   int64_t n_tok, int D, int M, int K,
                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate, float* __restrict__ logits) {
    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    for (int64_t t = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5); t < n_tok;
         t += (int64_t)gridDim.x * warps) {
        float lg[MAXM];
        warp_row_dots<T, MAXM>(x + t * D, w_r, M, D, lane, lg);
#pragma unroll
        for (int m = 0; m < MAXM; ++m)
            if (m < M && b_r) lg[m] += b_r[m];
        if (logits) {
#pragma unroll
            for (int m = 0; m < MAXM; ++m)
                if (m < M && lane == m) logits[t * M + m] = lg[m];
        }
        // top-k by logit; strict '>' keeps the lower index on equal logits
        uint32_t chosen = 0;
        float first = 0.f, denom = 0.f;
        int my_idx = 0;
        float my_val = 0.f;
        for (int j = 0; j < K; ++j) {
            int bi = -1;
            float bv = 0.f;
#pragma unroll
            for (int m = 0; m < MAXM; ++m) {
                if (m < M && !((chosen >> m) & 1u) && (bi < 0 || lg[m] > bv)) { bi = m; bv = lg[m]; }
            }
            chosen |= 1u << bi;
            if (j == 0) first = bv;
            float e = expf(bv - first);   // softmax restricted to the chosen, renormalised
            denom += e;
            if (lane == j) { my_idx = bi; my_val = e; }
        }
        if (lane < K) {
            topk_idx[t * K + lane] = my_idx;
            topk_gate[t * K + lane] = my_val / denom;
        }
    }
}

// beta = sigmoid(x W_beta^T); log_alpha = -exp(A) softplus(x W_a^T + b_a).
// w_gate rows: W_beta (H rows) then W_a (H rows).  Heads in groups of 16.
template <typename T>
__global__ void __launch_bounds__(256)
gate_proj_kernel(const T* __restrict__ x, const T* __restrict__ w_gate, const float* __restrict__ A,
                 const float* __restrict__ b_a, int64_t n_tok, int D, int H,
                 float* __restrict__ beta, float* __restrict__ log_alpha) {
    constexpr int G = 16;
    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    for (int64_t t = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5); t < n_tok;
         t += (int64_t)gridDim.x * warps) {
        for (int h0 = 0; h0 < H; h0 += G) {
            const int nh = min(G, H - h0);
            float zb[G], za[G];
            warp_row_dots<T, G>(x + t * D, w_gate + (size_t)h0 * D, nh, D, lane, zb);
            warp_row_dots<T, G>(x + t * D, w_gate + (size_t)(H + h0) * D, nh, D, lane, za);
#pragma unroll
            for (int i = 0; i < G; ++i) {
                if (i < nh && lane == i) {
                    const int h = h0 + i;
                    beta[t * H + h] = sigmoidf_(zb[i]);
                    log_alpha[t * H + h] = -expf(A[h]) * softplusf_(za[i] + b_a[h]);
                }
            }
        }
    }
}

static int grid_for_tokens(int64_t n_tok, int warps_per_block) {
    int64_t g = cdiv(n_tok, warps_per_block);
    return (int)(g < 148 * 16 ? g : 148 * 16);
}

cudaError_t launch_router(const void* x, const void* w_r, const float* b_r, int dt, int64_t n_tok, int D,
                          int M, int K, int32_t* idx, float* gate, float* logits, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    if (skinny_ok(dt, D, M)) return launch_router_skinny(x, w_r, b_r, n_tok, D, M, K, idx, gate, logits, st);
    dim3 grid(grid_for_tokens(n_tok, 8)), block(256);
    if (dt == MOM_BF16) {
        if (M <= 8)
            router_topk_kernel<bf16, 8><<<grid, block, 0, st>>>((const bf16*)x, (const bf16*)w_r, b_r, n_tok, D, M, K, idx, gate, logits);
        else if (M <= 16)
            router_topk_kernel<bf16, 16><<<grid, block, 0, st>>>((const bf16*)x, (const bf16*)w_r, b_r, n_tok, D, M, K, idx, gate, logits);
        else
            router_topk_kernel<bf16, 32><<<grid, block, 0, st>>>((const bf16*)x, (const bf16*)w_r, b_r, n_tok, D, M, K, idx, gate, logits);
    } else {
        if (M <= 8)
            router_topk_kernel<float, 8><<<grid, block, 0, st>>>((const float*)x, (const float*)w_r, b_r, n_tok, D, M, K, idx, gate, logits);
        else if (M <= 16)
            router_topk_kernel<float, 16><<<grid, block, 0, st>>>((const float*)x, (const float*)w_r, b_r, n_tok, D, M, K, idx, gate, logits);
        else
            router_topk_kernel<float, 32><<<grid, block, 0, st>>>((const float*)x, (const float*)w_r, b_r, n_tok, D, M, K, idx, gate, logits);
    }
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gate_proj(const void* x, const void* w_gate, const float* A, const float* b_a, int dt,
                             int64_t n_tok, int D, int H, float* beta, float* log_alpha, void* err, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    if (skinny_ok(dt, D, 2 * H)) return launch_gate_skinny(x, w_gate, A, b_a, n_tok, D, H, beta, log_alpha, err, st);
    dim3 grid(grid_for_tokens(n_tok, 8)), block(256);
    if (dt == MOM_BF16)
        gate_proj_kernel<bf16><<<grid, block, 0, st>>>((const bf16*)x, (const bf16*)w_gate, A, b_a, n_tok, D, H, beta, log_alpha);
    else
        gate_proj_kernel<float><<<grid, block, 0, st>>>((const float*)x, (const float*)w_gate, A, b_a, n_tok, D, H, beta, log_alpha);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
