// Per-memory gates of the routed rows.  Memory m has its own W_beta^m,
// W_a^m, A^m and b_a^m, and routed row r (memory m, token t = perm[r]) gets
//   beta_p[r]      = sigmoid(x_t W_beta^m^T)
//   log_alpha_p[r] = -exp(A^m) softplus(x_t W_a^m^T + b_a^m)
// ("MoM: Linear Sequence Modeling with Mixture-of-Memories", Summary: every
// memory keeps its own recurrent update -- here down to Gated DeltaNet's
// gates, which the shared memory takes from the layer's W_beta, W_a).
//
// Rows come in memory order (the reordering's output), so a 16-row tile
// nearly always lies in one memory.  bf16, d_model % 64 == 0, 2H <= 32: one
// warp per 16-row tile, m16n8k16 tensor-core MMAs (2H output columns: far
// too narrow for tcgen05 tiles) whose A fragments are loaded straight from
// the gathered x rows in global memory -- each x row is read once, by one
// warp, so staging it in shared memory would buy nothing -- and whose B
// fragments come from W^m through L1 (a CTA's tiles are consecutive, so its
// warps share W^m).  The k order inside an MMA is free as long as x and W use
// the same one: lane (g, c) feeds features 8c..8c+7 of each 32-feature half
// block, the first four to one MMA and the last four to the next.  A tile
// that straddles memories is computed once per memory it touches, each row
// keeping its own memory's result.  Other shapes and float32: one warp per
// row on CUDA cores.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace mom {
namespace {

constexpr int MG_TOK = 16;     // rows per tile (the MMA's M)
constexpr int MG_WARPS = 8;    // warps (tiles) per CTA

struct MemGateArgs {
    const void* x;              // [n_tok, D]
    const int32_t* perm;        // [n_rows] token of each routed row (null: row r reads x row r)
    const int32_t* mem_offset;  // [M + 1] first row of each group (a memory, or a (source, memory) group)
    const void* w;              // [n_w, 2H, D]: rows W_beta^m | W_a^m
    const float* A;             // [n_w, H]
    const float* b_a;           // [n_w, H]
    int64_t n_tok, n_rows;
    int D, H, M;
    float* beta;                // [n_rows, H]
    float* la;                  // [n_rows, H]
    void* err;
    const int32_t* gmem;        // [M] weights of each group (null: group m = memory m)
    int n_w;                    // memories in w, A, b_a
};

// the group table and each group's memory (-1: out of range) into shared memory
__device__ __forceinline__ void load_tables(const MemGateArgs& a, int* off, int* wix) {
    for (int i = threadIdx.x; i <= a.M; i += blockDim.x) off[i] = a.mem_offset[i];
    for (int i = threadIdx.x; i < a.M; i += blockDim.x) {
        const int m = a.gmem ? a.gmem[i] : i;
        wix[i] = (m >= 0 && m < a.n_w) ? m : -1;
    }
    __syncthreads();
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// x is read once: keep it out of L1 so that W^m stays there
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

constexpr int MG_G = 2;        // 64-feature blocks per load group

// x features [fb, fb + 64 * MG_G) of the lane's two rows (blocks past D: not loaded)
__device__ __forceinline__ void load_group(const bf16* x0, const bf16* x1, int fb, int D, uint4 (&v)[MG_G][2][2]) {
#pragma unroll
    for (int j = 0; j < MG_G; ++j) {
        if (fb + 64 * j < D) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                v[j][h][0] = ld_stream_u4(x0 + fb + 64 * j + 32 * h);
                v[j][h][1] = ld_stream_u4(x1 + fb + 64 * j + 32 * h);
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) v[j][h][0] = v[j][h][1] = make_uint4(0, 0, 0, 0);
        }
    }
}

// Memory of routed row r (mem_offset in shared memory), or -1 when no memory
// holds it.
__device__ __forceinline__ int memory_of(const int* off, int M, int64_t r) {
    int m = 0;
    while (m < M && r >= off[m + 1]) ++m;
    return (m < M && r >= off[m]) ? m : -1;
}

__device__ __forceinline__ void write_gates(const MemGateArgs& a, int64_t r, int m, int col, float z) {
    if (col < a.H) {
        a.beta[r * a.H + col] = sigmoidf_(z);
    } else if (col < 2 * a.H) {
        const int h = col - a.H;
        a.la[r * a.H + h] = -expf(a.A[m * a.H + h]) * softplusf_(z + a.b_a[m * a.H + h]);
    }
}

template <int NT>
__global__ void __launch_bounds__(MG_WARPS * 32)
mem_gate_mma_kernel(MemGateArgs a) {
    __shared__ int off[MOM_MAX_MEM + 1], wix[MOM_MAX_MEM];
    load_tables(a, off, wix);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int64_t tile = (int64_t)blockIdx.x * MG_WARPS + warp;
    const int64_t r0 = tile * MG_TOK;
    if (r0 >= a.n_rows) return;
    const bf16* x = reinterpret_cast<const bf16*>(a.x);
    const bf16* w = reinterpret_cast<const bf16*>(a.w);
    const int D = a.D, ncol = 2 * a.H;

    // rows g and g + 8 of the tile: token and memory (-1: past the end or invalid)
    int64_t tok[2];
    int mem[2];
    int mlo = INT_MAX, mhi = -1;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int64_t r = r0 + g + 8 * e;
        tok[e] = -1;
        mem[e] = -1;
        if (r < a.n_rows) {
            const int m = memory_of(off, a.M, r);
            const int64_t t = a.perm ? a.perm[r] : r;
            if (m >= 0 && wix[m] >= 0 && t >= 0 && t < a.n_tok) {
                tok[e] = t;
                mem[e] = m;
                mlo = min(mlo, m);
                mhi = max(mhi, m);
            } else {
                if (c == 0) {
                    record_error(a.err, MOM_DEVERR_ROW_INDEX, r);
                    for (int h = 0; h < a.H; ++h) { a.beta[r * a.H + h] = 0.f; a.la[r * a.H + h] = 0.f; }
                }
            }
        }
    }
    mlo = __reduce_min_sync(0xffffffffu, mlo);
    mhi = __reduce_max_sync(0xffffffffu, mhi);

    const bf16* x0 = x + (tok[0] >= 0 ? tok[0] : 0) * D + 8 * c;
    const bf16* x1 = x + (tok[1] >= 0 ? tok[1] : 0) * D + 8 * c;
    for (int m = mlo; m <= mhi; ++m) {
        if (off[m] == off[m + 1] || wix[m] < 0) continue;
        const bf16* wm = w + (size_t)wix[m] * ncol * D + 8 * c;
        // two accumulator sets (the two 32-feature halves of each 64-feature
        // block) halve the dependent MMA chain
        float acc[2][NT][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int n = 0; n < NT; ++n) acc[h][n][0] = acc[h][n][1] = acc[h][n][2] = acc[h][n][3] = 0.f;
        // x in groups of MG_G 64-feature blocks, double-buffered: the next
        // group's loads are issued before this group's products, so each
        // round trip overlaps the previous group's MMAs (loads and MMAs are
        // asm statements, kept in source order)
        uint4 cur[MG_G][2][2], nxt[MG_G][2][2];
        load_group(x0, x1, 0, D, cur);
        for (int fb = 0; fb < D; fb += 64 * MG_G) {
            if (fb + 64 * MG_G < D) load_group(x0, x1, fb + 64 * MG_G, D, nxt);
#pragma unroll
            for (int j = 0; j < MG_G; ++j) {
                if (fb + 64 * j >= D) break;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const int row = n * 8 + g;
                        const uint4 wv = row < ncol
                            ? __ldg(reinterpret_cast<const uint4*>(wm + (size_t)row * D + fb + 64 * j + 32 * h))
                            : make_uint4(0, 0, 0, 0);
                        const uint4 xa = cur[j][h][0], xb = cur[j][h][1];
                        mma_bf16_16816(acc[h][n], xa.x, xb.x, xa.y, xb.y, wv.x, wv.y);
                        mma_bf16_16816(acc[h][n], xa.z, xb.z, xa.w, xb.w, wv.z, wv.w);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < MG_G; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) { cur[j][h][0] = nxt[j][h][0]; cur[j][h][1] = nxt[j][h][1]; }
        }
        // acc[.][n]: (row g: cols n*8 + 2c, +1; row g + 8: the same cols)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int half = e >> 1;
                if (mem[half] != m) continue;
                write_gates(a, r0 + g + 8 * half, wix[m], n * 8 + 2 * c + (e & 1), acc[0][n][e] + acc[1][n][e]);
            }
    }
}

// One warp per routed row: 2H dot products over d_model on CUDA cores.
template <typename T>
__global__ void __launch_bounds__(256)
mem_gate_simt_kernel(MemGateArgs a) {
    __shared__ int off[MOM_MAX_MEM + 1], wix[MOM_MAX_MEM];
    load_tables(a, off, wix);
    const int lane = threadIdx.x & 31, warps = blockDim.x >> 5;
    const T* x = reinterpret_cast<const T*>(a.x);
    const T* w = reinterpret_cast<const T*>(a.w);
    const int D = a.D, ncol = 2 * a.H;
    for (int64_t r = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5); r < a.n_rows; r += (int64_t)gridDim.x * warps) {
        const int m0 = memory_of(off, a.M, r);
        const int m = m0 >= 0 ? wix[m0] : -1;
        const int64_t t = a.perm ? a.perm[r] : r;
        if (m < 0 || t < 0 || t >= a.n_tok) {
            if (lane == 0) record_error(a.err, MOM_DEVERR_ROW_INDEX, r);
            for (int h = lane; h < a.H; h += 32) { a.beta[r * a.H + h] = 0.f; a.la[r * a.H + h] = 0.f; }
            continue;
        }
        const T* xr = x + t * D;
        const T* wm = w + (size_t)m * ncol * D;
        for (int j0 = 0; j0 < ncol; j0 += 8) {
            float z[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) z[i] = 0.f;
            for (int f = lane; f < D; f += 32) {
                const float xv = to_f(xr[f]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (j0 + i < ncol) z[i] = fmaf(xv, to_f(wm[(size_t)(j0 + i) * D + f]), z[i]);
            }
            warp_sum_n<8>(z);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (lane == i && j0 + i < ncol) write_gates(a, r, m, j0 + i, z[i]);
        }
    }
}

}  // namespace

cudaError_t launch_mem_gate_proj(const void* x, const int32_t* perm, const int32_t* mem_offset, const void* w_gate_mem,
                                 const float* A_mem, const float* b_a_mem, int dt, int64_t n_tok, int64_t n_rows, int D,
                                 int H, int M, float* beta, float* log_alpha, void* err, cudaStream_t st,
                                 const int32_t* group_mem, int n_w) {
    if (n_rows == 0) return cudaSuccess;
    MemGateArgs a{x, perm, mem_offset, w_gate_mem, A_mem, b_a_mem, n_tok, n_rows, D, H, M, beta, log_alpha, err,
                  group_mem, group_mem ? n_w : M};
    if (dt == MOM_BF16 && D % 64 == 0 && 2 * H <= 32) {
        const unsigned grid = (unsigned)cdiv(cdiv(n_rows, MG_TOK), MG_WARPS);
        if (2 * H <= 8) mem_gate_mma_kernel<1><<<grid, MG_WARPS * 32, 0, st>>>(a);
        else if (2 * H <= 16) mem_gate_mma_kernel<2><<<grid, MG_WARPS * 32, 0, st>>>(a);
        else mem_gate_mma_kernel<4><<<grid, MG_WARPS * 32, 0, st>>>(a);
    } else {
        const int64_t want = cdiv(n_rows, 8);
        const unsigned grid = (unsigned)(want < 148 * 16 ? want : 148 * 16);
        if (dt == MOM_BF16) mem_gate_simt_kernel<bf16><<<grid, 256, 0, st>>>(a);
        else mem_gate_simt_kernel<float><<<grid, 256, 0, st>>>(a);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
