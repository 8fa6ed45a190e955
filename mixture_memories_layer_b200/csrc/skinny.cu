// Skinny projections that read x once: the router logits (M columns, then
// softmax / top-k / renormalisation: "MoM: Mixture-of-Memories Fixes Linear
// Attention Recall", Router mechanics, step by step) and the per-token gates
// beta = sigmoid(x W_beta^T), log alpha = -exp(A) softplus(x W_a^T + b_a)
// (Gated DeltaNet gating, as MoM's memories use it).
//
// Both are x W^T with at most 32 output columns: HBM-bound on x.  One
// persistent CTA per SM streams 16-token x d_model tiles of x through a ring
// of shared-memory stages with TMA (one producer warp); consumer warp w owns
// stage w and works on every NS-th tile, so there is no cross-warp reduction.
// The products are m16n8k16 bf16 tensor-core MMAs with fp32 accumulation:
// the k order inside an MMA is free as long as x and W use the same one, so
// lane (g, c) feeds the 8 contiguous features 8c..8c+7 of a 32-wide block
// of token rows g and g + 8 (one 16-byte shared load per row) and the same
// 8 features of weight row g (one 16-byte load, L1-resident) -- the first
// four to one MMA, the last four to the next.  The epilogue (top-k, or
// sigmoid / softplus) runs per token from a per-warp scratch.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mom {
namespace {

using namespace sm100;

constexpr int TOK = 16;                      // tokens per tile (the MMA's M)
constexpr int MAX_STAGES = 8;
constexpr size_t RING_BYTES = 200 * 1024;    // x stages + staged W per CTA

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

struct SkinnyArgs {
    const bf16* w;           // [ncol, D] weights
    int64_t n_tok;
    int D, ncol;
    // router
    const float* b_r;
    int M, K;
    int32_t* topk_idx;
    float* topk_gate;
    float* logits;
    // gates
    const float* A;
    const float* b_a;
    int H;
    float* beta;
    float* log_alpha;
    void* err;
};

// Columns [0, NT*8) of one tile: acc[n] holds (row g: cols n*8+2c, +1;
// row g+8: the same cols) after the loop.
// W is staged once per CTA in the same layout as the x tiles: 64-column
// boxes of NT*8 rows x 128 B, 16-byte chunk index XOR (row % 8).
template <int NT>
__device__ __forceinline__ void tile_products(uint32_t stage, uint32_t wsm, int D, int lane, float (&acc)[NT][4]) {
    const int g = lane >> 2, c = lane & 3;
    // two accumulator sets (the two 32-feature halves of each 64-column
    // box) halve the dependent MMA chain; summed at the end
    float acc2[2][NT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int n = 0; n < NT; ++n) acc2[h][n][0] = acc2[h][n][1] = acc2[h][n][2] = acc2[h][n][3] = 0.f;
    const uint32_t r0 = (uint32_t)g * 128, r1 = (uint32_t)(g + 8) * 128;
    const uint32_t sw = (uint32_t)(g & 7);      // rows g, g + 8 (and W rows n*8 + g) share the swizzle phase
#pragma unroll 2
    for (int fb0 = 0; fb0 < D; fb0 += 64) {
        const uint32_t box = stage + (uint32_t)(fb0 >> 6) * (TOK * 128);
        const uint32_t wbox = wsm + (uint32_t)(fb0 >> 6) * (NT * 8 * 128) + r0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t off = (((uint32_t)(4 * h + c)) ^ sw) << 4;
            const uint4 xa = ld_shared_u4(box + r0 + off);
            const uint4 xb = ld_shared_u4(box + r1 + off);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const uint4 wv = ld_shared_u4(wbox + off + n * 8 * 128);
                mma_bf16_16816(acc2[h][n], xa.x, xb.x, xa.y, xb.y, wv.x, wv.y);
                mma_bf16_16816(acc2[h][n], xa.z, xb.z, xa.w, xb.w, wv.z, wv.w);
            }
        }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = acc2[0][n][e] + acc2[1][n][e];
}

template <int NT, bool ROUTER>
__global__ void __launch_bounds__(9 * 32, 1)
skinny_kernel(const __grid_constant__ CUtensorMap tm_x, SkinnyArgs a, int NS) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024_shared(smem_raw);
    const size_t stage_bytes = (size_t)TOK * a.D * 2;
    const size_t w_bytes = (size_t)NT * 8 * a.D * 2;
    unsigned char* wsm_p = sm + NS * stage_bytes;                                  // staged W
    float* scratch = reinterpret_cast<float*>(wsm_p + w_bytes);                   // per warp [TOK][NT*8]
    uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + MAX_STAGES * TOK * NT * 8);   // full[NS], empty[NS]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * MAX_STAGES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles = cdiv(a.n_tok, TOK);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(bars + s), 1);
            mbar_init(smem_u32(bars + MAX_STAGES + s), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const uint32_t wsm = smem_u32(wsm_p);
    const uint32_t ring = smem_u32(sm);
    const int nbox = a.D / 64;
    if (warp < NS) {
        // the consumers stage W while the producer's first tiles are in flight
        for (int i = threadIdx.x; i < NT * 8 * (a.D / 8); i += NS * 32) {
            const int row = i / (a.D / 8), f = (i % (a.D / 8)) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row < a.ncol) v = __ldg(reinterpret_cast<const uint4*>(a.w + (int64_t)row * a.D + f));
            const uint32_t chunk = (uint32_t)((f & 63) >> 3);
            const uint32_t addr = wsm + (uint32_t)(f >> 6) * (NT * 8 * 128) + row * 128 + ((chunk ^ (uint32_t)(row & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NS * 32) : "memory");
    }

    if (warp == NS) {
        // ---------------------------------------------------- producer
        if (lane == 0) {
            int64_t k = 0, last = -1;
            for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++k) {
                const int s = (int)(k % NS);
                const uint32_t ph = (uint32_t)((k / NS) & 1);
                if (!mbar_wait(smem_u32(bars + MAX_STAGES + s), ph ^ 1, abort_flag, a.err, 60)) break;
                const uint32_t full = smem_u32(bars + s);
                mbar_arrive_expect_tx(full, (uint32_t)stage_bytes);
                for (int j = 0; j < nbox; ++j)
                    tma_load_2d(ring + (uint32_t)(s * stage_bytes) + j * (TOK * 128), &tm_x, full, 64 * j,
                                (int)(tile * TOK));
                last = k;
            }
            // copies in flight must land before the CTA exits
            for (int64_t k2 = last - NS + 1 < 0 ? 0 : last - NS + 1; k2 <= last; ++k2)
                mbar_wait_drain(smem_u32(bars + (int)(k2 % NS)), (uint32_t)((k2 / NS) & 1));
        }
        return;
    }
    if (warp > NS) return;
    // -------------------------------------------------------- consumer w
    float* scr = scratch + warp * TOK * NT * 8;
    const int g = lane >> 2, c = lane & 3;
    int64_t k = warp;
    for (int64_t tile = blockIdx.x + (int64_t)warp * gridDim.x; tile < tiles; tile += (int64_t)NS * gridDim.x, k += NS) {
        const int s = warp;
        const uint32_t ph = (uint32_t)((k / NS) & 1);
        if (!mbar_wait(smem_u32(bars + s), ph, abort_flag, a.err, 61)) break;
        float acc[NT][4];
        tile_products<NT>(ring + (uint32_t)(s * stage_bytes), wsm, a.D, lane, acc);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(bars + MAX_STAGES + s));
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            scr[g * NT * 8 + n * 8 + 2 * c] = acc[n][0];
            scr[g * NT * 8 + n * 8 + 2 * c + 1] = acc[n][1];
            scr[(g + 8) * NT * 8 + n * 8 + 2 * c] = acc[n][2];
            scr[(g + 8) * NT * 8 + n * 8 + 2 * c + 1] = acc[n][3];
        }
        __syncwarp();
        const int64_t t0 = tile * TOK;
        if constexpr (ROUTER) {
            if (lane < TOK && t0 + lane < a.n_tok) {
                const int64_t t = t0 + lane;
                const float* row = scr + lane * NT * 8;
                float lg[NT * 8];
#pragma unroll
                for (int m = 0; m < NT * 8; ++m) lg[m] = m < a.M ? row[m] + (a.b_r ? a.b_r[m] : 0.f) : 0.f;
                if (a.logits) {
                    for (int m = 0; m < a.M; ++m) a.logits[t * a.M + m] = lg[m];
                }
                // top-k by logit; strict '>' keeps the lower index on equal logits
                uint32_t chosen = 0;
                float first = 0.f, denom = 0.f;
                for (int j = 0; j < a.K; ++j) {
                    int bi = -1;
                    float bv = 0.f;
#pragma unroll
                    for (int m = 0; m < NT * 8; ++m)
                        if (m < a.M && !((chosen >> m) & 1u) && (bi < 0 || lg[m] > bv)) { bi = m; bv = lg[m]; }
                    chosen |= 1u << bi;
                    if (j == 0) first = bv;
                    const float e = expf(bv - first);   // softmax restricted to the chosen, renormalised
                    denom += e;
                    a.topk_idx[t * a.K + j] = bi;
                    a.topk_gate[t * a.K + j] = e;
                }
                for (int j = 0; j < a.K; ++j) a.topk_gate[t * a.K + j] /= denom;
            }
        } else {
            for (int i = lane; i < TOK * a.H; i += 32) {
                const int tl = i / a.H, h = i - tl * a.H;
                const int64_t t = t0 + tl;
                if (t < a.n_tok) {
                    const float* row = scr + tl * NT * 8;
                    a.beta[t * a.H + h] = sigmoidf_(row[h]);
                    a.log_alpha[t * a.H + h] = -expf(a.A[h]) * softplusf_(row[a.H + h] + a.b_a[h]);
                }
            }
        }
        __syncwarp();
    }
}

int stages_for(int D, int NT) {
    const size_t stage = (size_t)TOK * D * 2, w = (size_t)NT * 8 * D * 2;
    if (w >= RING_BYTES) return 0;
    int ns = (int)((RING_BYTES - w) / stage);
    return ns > MAX_STAGES ? MAX_STAGES : ns;
}

size_t smem_for(int D, int NT) {
    return 1024 + (size_t)stages_for(D, NT) * TOK * D * 2 + (size_t)NT * 8 * D * 2 + (size_t)MAX_STAGES * TOK * NT * 8 * 4 +
           2 * MAX_STAGES * 8 + 16;
}

int nt_for(int ncol) { return ncol <= 8 ? 1 : ncol <= 16 ? 2 : 4; }

template <int NT, bool ROUTER>
cudaError_t launch_skinny(const void* x, const SkinnyArgs& a, cudaStream_t st) {
    CUtensorMap tm;
    if (!make_tma_2d_bf16(&tm, x, (uint64_t)a.n_tok, (uint64_t)a.D, (uint64_t)a.D, 64, TOK)) return cudaErrorInvalidValue;
    const size_t smem = smem_for(a.D, NT);
    cudaError_t e = cudaFuncSetAttribute(skinny_kernel<NT, ROUTER>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int ns = stages_for(a.D, NT);
    int64_t tiles = cdiv(a.n_tok, TOK);
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = cdiv(tiles, ns);         // enough CTAs that every consumer warp gets a tile
    const unsigned grid = (unsigned)(want < sms ? want : sms);
    skinny_kernel<NT, ROUTER><<<grid, (ns + 1) * 32, smem, st>>>(tm, a, ns);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool skinny_ok(int dt, int D, int ncol) {
    return dt == MOM_BF16 && D % 64 == 0 && ncol >= 1 && ncol <= 32 && stages_for(D, nt_for(ncol)) >= 2 &&
           tma_available();
}

cudaError_t launch_router_skinny(const void* x, const void* w_r, const float* b_r, int64_t n_tok, int D, int M,
                                 int K, int32_t* idx, float* gate, float* logits, cudaStream_t st) {
    SkinnyArgs a{};
    a.w = (const bf16*)w_r;
    a.n_tok = n_tok;
    a.D = D;
    a.ncol = M;
    a.b_r = b_r;
    a.M = M;
    a.K = K;
    a.topk_idx = idx;
    a.topk_gate = gate;
    a.logits = logits;
    if (M <= 8) return launch_skinny<1, true>(x, a, st);
    if (M <= 16) return launch_skinny<2, true>(x, a, st);
    return launch_skinny<4, true>(x, a, st);
}

cudaError_t launch_gate_skinny(const void* x, const void* w_gate, const float* A, const float* b_a, int64_t n_tok,
                               int D, int H, float* beta, float* log_alpha, void* err, cudaStream_t st) {
    SkinnyArgs a{};
    a.w = (const bf16*)w_gate;
    a.n_tok = n_tok;
    a.D = D;
    a.ncol = 2 * H;
    a.A = A;
    a.b_a = b_a;
    a.H = H;
    a.beta = beta;
    a.log_alpha = log_alpha;
    a.err = err;
    if (2 * H <= 8) return launch_skinny<1, false>(x, a, st);
    if (2 * H <= 16) return launch_skinny<2, false>(x, a, st);
    return launch_skinny<4, false>(x, a, st);
}

}  // namespace mom
