// Skinny projections that read x once: the router logits (M columns, then
// softmax / top-k / renormalisation: "MoM: Mixture-of-Memories Fixes Linear
// Attention Recall", Router mechanics, step by step) and the per-token gates
// beta = sigmoid(x W_beta^T), log alpha = -exp(A) softplus(x W_a^T + b_a)
// (Gated DeltaNet gating, as MoM's memories use it).
//
// Both are x W^T with at most 32 output columns: HBM-bound on x.  A CTA
// takes 16 tokens; its four warps split d_model four ways and each runs
// m16n8k16 bf16 tensor-core products with fp32 accumulation, so the FMA
// work costs nothing next to the loads.  The k order inside an MMA is free
// as long as x and W use the same one: lane (g, c) of a warp holds, for the
// token rows g and g + 8, the 8 contiguous features 8c..8c+7 of a 32-wide
// block (one 16-byte load per row) and the same 8 features of weight row g
// -- the first four feed one MMA, the last four the next.  Each lane keeps
// 16 such loads in flight.  The four warps' partial sums meet in shared
// memory and the epilogue (top-k, sigmoid/softplus) runs per token.
#include "common.cuh"
#include "kernels.h"

namespace mom {
namespace {

constexpr int WARPS = 4;        // split of d_model inside the CTA
constexpr int TOK = 16;         // tokens per CTA (the MMA's M)
constexpr int BATCH = 8;        // 32-feature blocks loaded at once per lane

__device__ __forceinline__ uint4 ld_stream(const bf16* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_cached(const bf16* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Partial sums of 16 token rows (t0 ..) against NT*8 weight rows over the
// features [f_beg, f_end) of this warp, written to red[warp][row][col].
template <int NT>
__device__ __forceinline__ void warp_tile(const bf16* __restrict__ x, int64_t t0, int64_t n_tok, int D,
                                          const bf16* __restrict__ w, int ncol, int f_beg, int f_end,
                                          float* __restrict__ red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const bool ok0 = t0 + g < n_tok, ok1 = t0 + g + 8 < n_tok;
    const bf16* x0 = x + (t0 + g) * D + 8 * c;
    const bf16* x1 = x0 + (int64_t)8 * D;
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    for (int f = f_beg; f < f_end; f += 32 * BATCH) {
        uint4 xa[BATCH], xb[BATCH];
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int fb = f + 32 * b;
            xa[b] = (ok0 && fb < f_end) ? ld_stream(x0 + fb) : zero;
            xb[b] = (ok1 && fb < f_end) ? ld_stream(x1 + fb) : zero;
        }
#pragma unroll
        for (int b = 0; b < BATCH; ++b) {
            const int fb = f + 32 * b;
            if (fb < f_end) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int row = n * 8 + g;
                    const uint4 wv = row < ncol ? ld_cached(w + (int64_t)row * D + fb + 8 * c) : zero;
                    mma_bf16_16816(acc[n], xa[b].x, xb[b].x, xa[b].y, xb[b].y, wv.x, wv.y);
                    mma_bf16_16816(acc[n], xa[b].z, xb[b].z, xa[b].w, xb[b].w, wv.z, wv.w);
                }
            }
        }
    }
    // d0,d1: row g, cols 2c, 2c+1; d2,d3: row g+8
    constexpr int NCOL = NT * 8;
    float* r = red + warp * TOK * NCOL;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        r[g * NCOL + n * 8 + 2 * c] = acc[n][0];
        r[g * NCOL + n * 8 + 2 * c + 1] = acc[n][1];
        r[(g + 8) * NCOL + n * 8 + 2 * c] = acc[n][2];
        r[(g + 8) * NCOL + n * 8 + 2 * c + 1] = acc[n][3];
    }
}

template <int NT>
__device__ __forceinline__ float red_sum(const float* red, int t, int col) {
    constexpr int NCOL = NT * 8;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) s += red[(w * TOK + t) * NCOL + col];
    return s;
}

template <int NT>
__global__ void __launch_bounds__(WARPS * 32)
skinny_router_kernel(const bf16* __restrict__ x, const bf16* __restrict__ w_r, const float* __restrict__ b_r,
                     int64_t n_tok, int D, int M, int K, int32_t* __restrict__ topk_idx,
                     float* __restrict__ topk_gate, float* __restrict__ logits) {
    __shared__ float red[WARPS * TOK * NT * 8];
    const int warp = threadIdx.x >> 5;
    const int fq = D / WARPS;
    const int64_t tiles = cdiv(n_tok, TOK);
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t t0 = tile * TOK;
        warp_tile<NT>(x, t0, n_tok, D, w_r, M, warp * fq, (warp + 1) * fq, red);
        __syncthreads();
        const int i = threadIdx.x;
        if (i < TOK && t0 + i < n_tok) {
            const int64_t t = t0 + i;
            float lg[NT * 8];
#pragma unroll
            for (int m = 0; m < NT * 8; ++m) lg[m] = m < M ? red_sum<NT>(red, i, m) + (b_r ? b_r[m] : 0.f) : 0.f;
            if (logits) {
                for (int m = 0; m < M; ++m) logits[t * M + m] = lg[m];
            }
            // top-k by logit; strict '>' keeps the lower index on equal logits
            uint32_t chosen = 0;
            float first = 0.f, denom = 0.f;
            for (int j = 0; j < K; ++j) {
                int bi = -1;
                float bv = 0.f;
#pragma unroll
                for (int m = 0; m < NT * 8; ++m)
                    if (m < M && !((chosen >> m) & 1u) && (bi < 0 || lg[m] > bv)) { bi = m; bv = lg[m]; }
                chosen |= 1u << bi;
                if (j == 0) first = bv;
                const float e = expf(bv - first);   // softmax restricted to the chosen, renormalised
                denom += e;
                topk_idx[t * K + j] = bi;
                topk_gate[t * K + j] = e;
            }
            for (int j = 0; j < K; ++j) topk_gate[t * K + j] /= denom;
        }
        __syncthreads();
    }
}

template <int NT>
__global__ void __launch_bounds__(WARPS * 32)
skinny_gate_kernel(const bf16* __restrict__ x, const bf16* __restrict__ w_gate, const float* __restrict__ A,
                   const float* __restrict__ b_a, int64_t n_tok, int D, int H, float* __restrict__ beta,
                   float* __restrict__ log_alpha) {
    __shared__ float red[WARPS * TOK * NT * 8];
    const int warp = threadIdx.x >> 5;
    const int fq = D / WARPS;
    const int64_t tiles = cdiv(n_tok, TOK);
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t t0 = tile * TOK;
        warp_tile<NT>(x, t0, n_tok, D, w_gate, 2 * H, warp * fq, (warp + 1) * fq, red);
        __syncthreads();
        for (int i = threadIdx.x; i < TOK * H; i += WARPS * 32) {
            const int tl = i / H, h = i - tl * H;
            const int64_t t = t0 + tl;
            if (t < n_tok) {
                beta[t * H + h] = sigmoidf_(red_sum<NT>(red, tl, h));
                log_alpha[t * H + h] = -expf(A[h]) * softplusf_(red_sum<NT>(red, tl, H + h) + b_a[h]);
            }
        }
        __syncthreads();
    }
}

int grid_for(int64_t n_tok) {
    const int64_t g = cdiv(n_tok, TOK);
    return (int)(g < 148 * 16 ? g : 148 * 16);
}

}  // namespace

bool skinny_ok(int dt, int D, int ncol) {
    return dt == MOM_BF16 && D % (WARPS * 32) == 0 && ncol >= 1 && ncol <= 32;
}

cudaError_t launch_router_skinny(const void* x, const void* w_r, const float* b_r, int64_t n_tok, int D, int M,
                                 int K, int32_t* idx, float* gate, float* logits, cudaStream_t st) {
    const dim3 grid(grid_for(n_tok)), block(WARPS * 32);
    const bf16* xb = (const bf16*)x;
    const bf16* wb = (const bf16*)w_r;
    if (M <= 8)
        skinny_router_kernel<1><<<grid, block, 0, st>>>(xb, wb, b_r, n_tok, D, M, K, idx, gate, logits);
    else if (M <= 16)
        skinny_router_kernel<2><<<grid, block, 0, st>>>(xb, wb, b_r, n_tok, D, M, K, idx, gate, logits);
    else
        skinny_router_kernel<4><<<grid, block, 0, st>>>(xb, wb, b_r, n_tok, D, M, K, idx, gate, logits);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gate_skinny(const void* x, const void* w_gate, const float* A, const float* b_a, int64_t n_tok,
                               int D, int H, float* beta, float* log_alpha, cudaStream_t st) {
    const dim3 grid(grid_for(n_tok)), block(WARPS * 32);
    const bf16* xb = (const bf16*)x;
    const bf16* wb = (const bf16*)w_gate;
    if (2 * H <= 8)
        skinny_gate_kernel<1><<<grid, block, 0, st>>>(xb, wb, A, b_a, n_tok, D, H, beta, log_alpha);
    else if (2 * H <= 16)
        skinny_gate_kernel<2><<<grid, block, 0, st>>>(xb, wb, A, b_a, n_tok, D, H, beta, log_alpha);
    else
        skinny_gate_kernel<4><<<grid, block, 0, st>>>(xb, wb, A, b_a, n_tok, D, H, beta, log_alpha);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
