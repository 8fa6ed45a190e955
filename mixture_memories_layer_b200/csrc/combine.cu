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

// One warp per token row, persistent: the warp reads the token's K row
// indices and gates once, then every lane has its CH 16-byte pieces of the
// shared output and of all K memory rows in flight together before any
// arithmetic.
// 8 consecutive elements as loaded (bf16: one 16-byte vector; f32: two),
// converted to fp32 only at the FMA.
template <typename T> struct Piece;
template <> struct Piece<bf16> {
    uint4 u;
    __device__ __forceinline__ void load(const bf16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ float at(int e) const {
        const uint32_t w = e < 2 ? u.x : e < 4 ? u.y : e < 6 ? u.z : u.w;
        return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
    }
};
template <> struct Piece<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ float at(int e) const {
        const float4& f = e < 4 ? a : b;
        const int k = e & 3;
        return k == 0 ? f.x : k == 1 ? f.y : k == 2 ? f.z : f.w;
    }
};

template <typename T, int KMAX, int CH>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ o_sh, const T* __restrict__ o_p, const int32_t* __restrict__ row_of,
               const float* __restrict__ gate, int64_t n_tok, int K, int HD, T* __restrict__ out, void* ws) {
    const int lane = threadIdx.x & 31;
    const int64_t n_rows = n_tok * K;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < n_tok; t += warps) {
        for (int c0 = 0; c0 < HD; c0 += 8 * 32 * CH) {
            Piece<T> sh[CH];
#pragma unroll
            for (int q = 0; q < CH; ++q) {
                const int c = c0 + 8 * (lane + 32 * q);
                if (c < HD) sh[q].load(o_sh + t * HD + c);
            }
            float acc[CH][8];
            bool first = true;
            for (int j0 = 0; j0 < K; j0 += KMAX) {       // one pass when K <= KMAX
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
                            if (lane == 0 && c0 == 0) record_error(ws, MOM_DEVERR_ROW_INDEX, t);
                            r[j] = -1;
                        }
                    }
                }
                Piece<T> v[KMAX][CH];
#pragma unroll
                for (int q = 0; q < CH; ++q) {
                    const int c = c0 + 8 * (lane + 32 * q);
#pragma unroll
                    for (int j = 0; j < KMAX; ++j)
                        if (r[j] >= 0 && c < HD) v[j][q].load(o_p + r[j] * HD + c);
                }
#pragma unroll
                for (int q = 0; q < CH; ++q) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float a = first ? sh[q].at(e) : acc[q][e];
#pragma unroll
                        for (int j = 0; j < KMAX; ++j)
                            if (r[j] >= 0) a = fmaf(g[j], v[j][q].at(e), a);
                        acc[q][e] = a;
                    }
                }
                first = false;
            }
#pragma unroll
            for (int q = 0; q < CH; ++q) {
                const int c = c0 + 8 * (lane + 32 * q);
                if (c < HD) store_vec<8>(out + t * HD + c, acc[q]);
            }
        }
    }
}

// The Gated DeltaNet block's gated output norm fused into the combine (the
// block's form is a reading: the pages print nothing of it): per head of d
// channels of token t, with o the combined output above,
//   out = o / sqrt(mean(o^2) + eps) * w_norm * SiLU(g[t])
// A head is d/8 consecutive lanes of one 256-column piece (d divides 256).
// With K = 0 (o_p, row_of and gate unused) o is o_sh: the norm and gate of
// an output combined elsewhere (the decode step's).
template <int KMAX, int CH>
__global__ void __launch_bounds__(256, 2)
combine_norm_gate_kernel(const bf16* __restrict__ o_sh, const bf16* __restrict__ o_p,
                         const int32_t* __restrict__ row_of, const float* __restrict__ gate,
                         const bf16* __restrict__ g, const float* __restrict__ w_norm, float eps, int64_t n_tok,
                         int K, int HD, int d, bf16* __restrict__ out, void* ws) {
    const int lane = threadIdx.x & 31;
    const int64_t n_rows = n_tok * K;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const float inv_d = 1.f / (float)d;
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < n_tok; t += warps) {
        for (int c0 = 0; c0 < HD; c0 += 8 * 32 * CH) {
            Piece<bf16> sh[CH], gp[CH];
#pragma unroll
            for (int q = 0; q < CH; ++q) {
                const int c = c0 + 8 * (lane + 32 * q);
                sh[q].u = gp[q].u = make_uint4(0u, 0u, 0u, 0u);
                if (c < HD) {
                    sh[q].load(o_sh + t * HD + c);
                    gp[q].load(g + t * HD + c);
                }
            }
            float acc[CH][8];
            bool first = true;
            for (int j0 = 0; j0 < K; j0 += KMAX) {
                int64_t r[KMAX];
                float gt[KMAX];
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    r[j] = -1;
                    gt[j] = 0.f;
                    if (j0 + j < K) {
                        r[j] = __ldg(row_of + t * K + j0 + j);
                        gt[j] = __ldg(gate + t * K + j0 + j);
                        if (r[j] < 0 || r[j] >= n_rows) {
                            if (lane == 0 && c0 == 0) record_error(ws, MOM_DEVERR_ROW_INDEX, t);
                            r[j] = -1;
                        }
                    }
                }
                Piece<bf16> v[KMAX][CH];
#pragma unroll
                for (int q = 0; q < CH; ++q) {
                    const int c = c0 + 8 * (lane + 32 * q);
#pragma unroll
                    for (int j = 0; j < KMAX; ++j)
                        if (r[j] >= 0 && c < HD) v[j][q].load(o_p + r[j] * HD + c);
                }
#pragma unroll
                for (int q = 0; q < CH; ++q) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float a = first ? sh[q].at(e) : acc[q][e];
#pragma unroll
                        for (int j = 0; j < KMAX; ++j)
                            if (r[j] >= 0) a = fmaf(gt[j], v[j][q].at(e), a);
                        acc[q][e] = a;
                    }
                }
                first = false;
            }
            if (first) {                                  // top_k = 0: o = o_sh
#pragma unroll
                for (int q = 0; q < CH; ++q)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[q][e] = sh[q].at(e);
            }
#pragma unroll
            for (int q = 0; q < CH; ++q) {
                const int c = c0 + 8 * (lane + 32 * q);
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(acc[q][e], acc[q][e], ss);
                if (c >= HD) ss = 0.f;
                for (int o = d >> 4; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float rs = rsqrtf(ss * inv_d + eps);
                if (c < HD) {
                    const float4* wn = reinterpret_cast<const float4*>(w_norm + c % d);
                    const float4 w0 = __ldg(wn), w1 = __ldg(wn + 1);
                    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        // SiLU by the fast exponential and division (the result is rounded to bf16)
                        const float ge = gp[q].at(e);
                        y[e] = acc[q][e] * rs * wv[e] * __fdividef(ge, 1.f + __expf(-ge));
                    }
                    store_vec<8>(out + t * HD + c, y);
                }
            }
        }
    }
}

cudaError_t launch_combine_norm_gate(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                                     const void* g, const float* w_norm, float eps, int64_t n_tok, int K, int H,
                                     int d, void* out, void* ws, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    const int HD = H * d;
    int64_t grid = cdiv(n_tok, 8);
    if (grid > 148 * 8) grid = 148 * 8;
    const bf16 *a = (const bf16*)o_sh, *b = (const bf16*)o_p, *gg = (const bf16*)g;
    if (K <= 2)
        combine_norm_gate_kernel<2, 2><<<(unsigned)grid, 256, 0, st>>>(a, b, row_of, gate, gg, w_norm, eps, n_tok, K,
                                                                       HD, d, (bf16*)out, ws);
    else
        combine_norm_gate_kernel<4, 2><<<(unsigned)grid, 256, 0, st>>>(a, b, row_of, gate, gg, w_norm, eps, n_tok, K,
                                                                       HD, d, (bf16*)out, ws);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_combine(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                           int64_t n_tok, int K, int H, int d, int dt, void* out, void* ws, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    const int HD = H * d;
    int64_t g = cdiv(n_tok, 8);                 // 8 warps (tokens) per CTA
    if (g > 148 * 8) g = 148 * 8;
    const dim3 grid((unsigned)g), block(256);
    if (dt == MOM_BF16) {
        if (K <= 2)
            combine_kernel<bf16, 2, 4><<<grid, block, 0, st>>>((const bf16*)o_sh, (const bf16*)o_p, row_of, gate, n_tok, K, HD, (bf16*)out, ws);
        else
            combine_kernel<bf16, 4, 2><<<grid, block, 0, st>>>((const bf16*)o_sh, (const bf16*)o_p, row_of, gate, n_tok, K, HD, (bf16*)out, ws);
    } else {
        if (K <= 2)
            combine_kernel<float, 2, 2><<<grid, block, 0, st>>>((const float*)o_sh, (const float*)o_p, row_of, gate, n_tok, K, HD, (float*)out, ws);
        else
            combine_kernel<float, 4, 1><<<grid, block, 0, st>>>((const float*)o_sh, (const float*)o_p, row_of, gate, n_tok, K, HD, (float*)out, ws);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
