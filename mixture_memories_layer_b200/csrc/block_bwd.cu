// The reverse pass of the Gated DeltaNet block around the memories (the
// forward: conv.cu, the combine's gated norm in combine.cu, the output
// projection on the tensor cores).  Training is the pages' main workload
// ("MoM: Linear Sequence Modeling with Mixture-of-Memories", Key points);
// the block's form is a reading (the pages print none of it).
//
//   norm_gate_bwd : per head of the combined output o (recomputed from
//                   o_sh and the routed rows), with r = 1/sqrt(mean(o^2)+eps),
//                   n = o r, s = SiLU(g), dn = dy w_norm s:
//                     do = r (dn - n mean(dn n)),  dg = dy n w_norm SiLU'(g),
//                     dw_norm += dy n s  (summed over tokens and heads)
//   conv_bwd_fused: for out = [l2norm] SiLU(a), a = conv(z): da from d out
//                   (a recomputed from the raw rows, the norm's adjoint per
//                   head, then SiLU's), then dz[t] = sum_j w[W-1-j] da[t+j]
//                   over the rows t+j of t's segment (the convolution run
//                   backwards in time) and dw[g][W-1-j] += da[t] z[t-j]
// Streaming elementwise work, one warp per (row, 256 channels) or per
// (32 rows, 256 channels); the filter gradients are summed per warp task in
// registers and added atomically.
#include "common.cuh"
#include "kernels.h"

namespace mom {
namespace {

__device__ __forceinline__ float bfv(const uint4& u, int e) {
    const uint32_t w = e < 2 ? u.x : e < 4 ? u.y : e < 6 ? u.z : u.w;
    return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

__device__ __forceinline__ float silu_grad(float g) {
    const float s = sigmoidf_(g);
    return s * (1.f + g * (1.f - s));
}

// ------------------------------------------------------------- norm gate --
template <int KMAX>
__global__ void __launch_bounds__(256)
norm_gate_bwd_kernel(const bf16* __restrict__ o_sh, const bf16* __restrict__ o_p, const int32_t* __restrict__ row_of,
                     const float* __restrict__ gate, const bf16* __restrict__ g, const float* __restrict__ w_norm,
                     float eps, const bf16* __restrict__ dy, int64_t n_tok, int K, int HD, int d,
                     bf16* __restrict__ d_o, float* __restrict__ dg, int64_t ldg, float* __restrict__ dw_norm,
                     void* ws) {
    extern __shared__ float dw_s[];                       // [d]
    const int lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < d; i += blockDim.x) dw_s[i] = 0.f;
    __syncthreads();
    const int64_t n_rows = n_tok * K;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const float inv_d = 1.f / (float)d;
    float wacc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) wacc[e] = 0.f;
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < n_tok; t += warps) {
        for (int c0 = 0; c0 < HD; c0 += 256) {           // uniform over the warp
            // one 256-column piece per pass (heads of d <= 256 channels lie inside it)
            const int c = c0 + 8 * lane;
            const bool on = c < HD;
            float o[8], gy[8], gg[8];
            uint4 u = make_uint4(0u, 0u, 0u, 0u), ug = u, uy = u;
            if (on) {
                u = __ldg(reinterpret_cast<const uint4*>(o_sh + t * HD + c));
                ug = __ldg(reinterpret_cast<const uint4*>(g + t * HD + c));
                uy = __ldg(reinterpret_cast<const uint4*>(dy + t * HD + c));
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) { o[e] = bfv(u, e); gg[e] = bfv(ug, e); gy[e] = bfv(uy, e); }
            for (int j0 = 0; j0 < K; j0 += KMAX) {
                int64_t r[KMAX];
                float gt[KMAX];
                uint4 v[KMAX];
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    r[j] = -1;
                    gt[j] = 0.f;
                    if (j0 + j < K) {
                        r[j] = __ldg(row_of + t * K + j0 + j);
                        gt[j] = __ldg(gate + t * K + j0 + j);
                        if (r[j] < 0 || r[j] >= n_rows) {
                            if (lane == 0 && c == 0) record_error(ws, MOM_DEVERR_ROW_INDEX, t);
                            r[j] = -1;
                        }
                    }
                    v[j] = (on && r[j] >= 0) ? __ldg(reinterpret_cast<const uint4*>(o_p + r[j] * HD + c))
                                             : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = fmaf(gt[j], bfv(v[j], e), o[e]);
            }
            // per head (d/8 lanes): r, then mean(dn n)
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(o[e], o[e], ss);
            for (int sh = d >> 4; sh >= 1; sh >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, sh);
            const float rr = rsqrtf(ss * inv_d + eps);
            const int cd = on ? c % d : 0;
            float wn[8], n[8], dn[8], dnn = 0.f;
            const float4* wp = reinterpret_cast<const float4*>(w_norm + cd);
            const float4 w0 = __ldg(wp), w1 = __ldg(wp + 1);
            wn[0] = w0.x; wn[1] = w0.y; wn[2] = w0.z; wn[3] = w0.w; wn[4] = w1.x; wn[5] = w1.y; wn[6] = w1.z; wn[7] = w1.w;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                n[e] = o[e] * rr;
                const float s = gg[e] * sigmoidf_(gg[e]);
                dn[e] = gy[e] * wn[e] * s;
                dnn = fmaf(dn[e], n[e], dnn);
                wacc[e] = fmaf(gy[e], n[e] * s, wacc[e]);
            }
            for (int sh = d >> 4; sh >= 1; sh >>= 1) dnn += __shfl_xor_sync(0xffffffffu, dnn, sh);
            const float mean = dnn * inv_d;
            if (on) {
                float dov[8], dgv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    dov[e] = rr * (dn[e] - n[e] * mean);
                    dgv[e] = gy[e] * n[e] * wn[e] * silu_grad(gg[e]);
                }
                store_vec<8>(d_o + t * HD + c, dov);
                store_vec<8>(dg + t * ldg + c, dgv);
            }
        }
    }
    // the norm weight's gradient: this lane's channels, summed over the CTA, then added
    if (8 * lane < HD) {
        const int cd = (8 * lane) % d;
#pragma unroll
        for (int e = 0; e < 8; ++e) atomicAdd(&dw_s[cd + e], wacc[e]);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < d; i += blockDim.x) atomicAdd(dw_norm + i, dw_s[i]);
}

// ------------------------------------------------------------ convolution --
constexpr int MAXP = 8, RANGE = 32;
struct ConvBwdBatch {
    ConvBwdArgs pr[MAXP];
    int64_t base_rng[MAXP + 1];   // work items before each problem (one per 32 rows x 256 channels)
    int n, C, d;
    void* err;
};

// segment of row r (seg_cu[n_seg] > r >= seg_cu[0]): the last s with seg_cu[s] <= r
__device__ __forceinline__ int seg_of(const int32_t* seg_cu, int n_seg, int64_t r) {
    int lo = 0, hi = n_seg;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(seg_cu + mid) <= r) lo = mid; else hi = mid;
    }
    return lo;
}

// The convolution's adjoint: a warp's 32-row range (x 256 channels)
// recomputes da for its rows and the W-1 rows after them (a ring in
// registers), so da never goes to memory: per element z (2 B) and d out
// (4 B) in, dz (4 B) out.  (As a row pass writing da and a tap pass reading
// it back, twice the bytes, the two took 1.04 ms on the 380M block's five
// convolutions against 0.86 ms fused.)
template <int W>
__global__ void __launch_bounds__(256, 2) conv_bwd_fused_kernel(const __grid_constant__ ConvBwdBatch B) {
    const int lane = threadIdx.x & 31;
    const int nblk = (B.C + 255) / 256;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    int pi = 0;
    for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < B.base_rng[B.n]; it += nw) {
        while (it >= B.base_rng[pi + 1]) ++pi;
        const ConvBwdArgs& a = B.pr[pi];
        const int64_t r_beg = __ldg(a.seg_cu), r_end = __ldg(a.seg_cu + a.n_seg);
        if (r_beg < 0 || r_end < r_beg || r_end > a.n_rows) {
            if (lane == 0 && it == B.base_rng[pi]) record_error(B.err, MOM_DEVERR_SEGMENT, pi);
            continue;
        }
        const int64_t local = it - B.base_rng[pi];
        const int64_t ra = r_beg + (local / nblk) * RANGE;
        if (ra >= r_end) continue;
        const int64_t rb = ra + RANGE < r_end ? ra + RANGE : r_end;
        const int c = (int)(local % nblk) * 256 + 8 * lane;
        const bool on = c < B.C;
        const bf16* z = reinterpret_cast<const bf16*>(a.z);
        float wv[W][8], dwa[W][8];
#pragma unroll
        for (int t = 0; t < W; ++t)
#pragma unroll
            for (int e = 0; e < 8; ++e) dwa[t][e] = 0.f;
        int grp = -1;
        bool okg = false;
        auto flush = [&]() {
            if (on && okg) {
#pragma unroll
                for (int t = 0; t < W; ++t)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (dwa[t][e] != 0.f) atomicAdd(a.dw + ((int64_t)grp * W + t) * B.C + c + e, dwa[t][e]);
            }
#pragma unroll
            for (int t = 0; t < W; ++t)
#pragma unroll
                for (int e = 0; e < 8; ++e) dwa[t][e] = 0.f;
        };
        // da of row r of the segment [s_beg, s_end) (0 past its end); warp-uniform r
        auto da_row = [&](int64_t r, int64_t s_beg, int64_t s_end, float (&out)[8]) {
            const bool in = r < s_end;
            float acc[8], dy[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) { acc[e] = 0.f; dy[e] = 0.f; }
            if (in && on) {
#pragma unroll
                for (int j = 0; j < W; ++j) {
                    if (r - j >= s_beg) {
                        const uint4 v = __ldg(reinterpret_cast<const uint4*>(z + (r - j) * B.C + c));
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wv[W - 1 - j][e], bfv(v, e), acc[e]);
                    }
                }
                load_vec<8>(a.dout + r * B.C + c, dy);
            }
            float cv[8], ss = 0.f, cdy = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                cv[e] = acc[e] * sigmoidf_(acc[e]);
                ss = fmaf(cv[e], cv[e], ss);
                cdy = fmaf(cv[e], dy[e], cdy);
            }
            if (a.l2) {                                   // uniform over the warp
                for (int sh = B.d >> 4; sh >= 1; sh >>= 1) {
                    ss += __shfl_xor_sync(0xffffffffu, ss, sh);
                    cdy += __shfl_xor_sync(0xffffffffu, cdy, sh);
                }
                const float inv = 1.f / sqrtf(ss + 1e-6f), k3 = cdy * inv * inv * inv;
#pragma unroll
                for (int e = 0; e < 8; ++e) out[e] = (in && okg) ? (dy[e] * inv - cv[e] * k3) * silu_grad(acc[e]) : 0.f;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) out[e] = (in && okg) ? dy[e] * silu_grad(acc[e]) : 0.f;
            }
        };
        int64_t t = ra;
        while (t < rb) {
            const int s = seg_of(a.seg_cu, a.n_seg, t);
            const int64_t s_beg = __ldg(a.seg_cu + s), s_end = __ldg(a.seg_cu + s + 1);
            const int g2 = s / a.seg_per_group;
            if (g2 != grp) {
                flush();
                grp = g2;
                okg = grp < a.n_groups;
                if (!okg && lane == 0) record_error(B.err, MOM_DEVERR_SEGMENT, s);
#pragma unroll
                for (int tp = 0; tp < W; ++tp) {
                    if (on && okg) {
                        const float* wp = a.w + ((int64_t)grp * W + tp) * B.C + c;
                        const float4 w0 = __ldg(reinterpret_cast<const float4*>(wp));
                        const float4 w1 = __ldg(reinterpret_cast<const float4*>(wp) + 1);
                        wv[tp][0] = w0.x; wv[tp][1] = w0.y; wv[tp][2] = w0.z; wv[tp][3] = w0.w;
                        wv[tp][4] = w1.x; wv[tp][5] = w1.y; wv[tp][6] = w1.z; wv[tp][7] = w1.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) wv[tp][e] = 0.f;
                    }
                }
            }
            const int64_t t_stop = rb < s_end ? rb : s_end;
            float ring[W][8];                             // da of rows t .. t+W-1
#pragma unroll
            for (int j = 0; j + 1 < W; ++j) da_row(t + j, s_beg, s_end, ring[j]);
            for (; t < t_stop; ++t) {
                da_row(t + W - 1, s_beg, s_end, ring[W - 1]);
                if (on) {
                    float dz[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) dz[e] = 0.f;
#pragma unroll
                    for (int j = 0; j < W; ++j)
#pragma unroll
                        for (int e = 0; e < 8; ++e) dz[e] = fmaf(wv[W - 1 - j][e], ring[j][e], dz[e]);
#pragma unroll
                    for (int j = 0; j < W; ++j) {
                        if (t - j >= s_beg) {
                            const uint4 v = __ldg(reinterpret_cast<const uint4*>(z + (t - j) * B.C + c));
#pragma unroll
                            for (int e = 0; e < 8; ++e) dwa[W - 1 - j][e] = fmaf(ring[0][e], bfv(v, e), dwa[W - 1 - j][e]);
                        }
                    }
                    float* dst = a.dz + t * a.ldz + a.col0 + c;
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[e] = dz[e];
                }
#pragma unroll
                for (int j = 0; j + 1 < W; ++j)
#pragma unroll
                    for (int e = 0; e < 8; ++e) ring[j][e] = ring[j + 1][e];
            }
        }
        flush();
    }
}

__global__ void convert_kernel(const void* __restrict__ src, int src_dt, void* __restrict__ dst, int dst_dt, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = src_dt == MOM_BF16 ? __bfloat162float(reinterpret_cast<const bf16*>(src)[i])
                                           : reinterpret_cast<const float*>(src)[i];
        if (dst_dt == MOM_BF16) reinterpret_cast<bf16*>(dst)[i] = __float2bfloat16_rn(v);
        else reinterpret_cast<float*>(dst)[i] = v;
    }
}

}  // namespace

cudaError_t launch_norm_gate_bwd(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                                 const void* g, const float* w_norm, float eps, const void* dy, int64_t n_tok, int K,
                                 int H, int d, void* d_o, float* dg, int64_t ldg, float* dw_norm, void* ws,
                                 cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(dw_norm, 0, (size_t)d * 4, st);
    if (e != cudaSuccess || n_tok == 0) return e;
    const int HD = H * d;
    int64_t grid = cdiv(n_tok, 8);
    if (grid > 148 * 4) grid = 148 * 4;
    const size_t smem = (size_t)d * 4;
    const bf16 *a = (const bf16*)o_sh, *b = (const bf16*)o_p, *gg = (const bf16*)g, *yy = (const bf16*)dy;
    if (K <= 2)
        norm_gate_bwd_kernel<2><<<(unsigned)grid, 256, smem, st>>>(a, b, row_of, gate, gg, w_norm, eps, yy, n_tok, K,
                                                                   HD, d, (bf16*)d_o, dg, ldg, dw_norm, ws);
    else
        norm_gate_bwd_kernel<4><<<(unsigned)grid, 256, smem, st>>>(a, b, row_of, gate, gg, w_norm, eps, yy, n_tok, K,
                                                                   HD, d, (bf16*)d_o, dg, ldg, dw_norm, ws);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_conv_bwd(const ConvBwdArgs* problems, int n, int C, int W, int d, void* err, cudaStream_t st) {
    if (n < 1 || n > MAXP) return cudaErrorInvalidValue;
    ConvBwdBatch b{};
    b.n = n;
    b.C = C;
    b.d = d;
    b.err = err;
    const int nblk = (C + 255) / 256;
    b.base_rng[0] = 0;
    for (int i = 0; i < n; ++i) {
        const ConvBwdArgs& q = problems[i];
        b.pr[i] = q;
        b.base_rng[i + 1] = b.base_rng[i] + cdiv(q.n_rows, RANGE) * nblk;
        cudaError_t e = cudaMemsetAsync(q.dw, 0, (size_t)q.n_groups * W * C * 4, st);
        if (e != cudaSuccess) return e;
    }
    if (b.base_rng[n] == 0) return cudaSuccess;
    auto grid_of = [](int64_t items) {
        int64_t g = cdiv(items, 8);
        return (unsigned)(g > 148 * 16 ? 148 * 16 : g < 1 ? 1 : g);
    };
    switch (W) {
        case 1: conv_bwd_fused_kernel<1><<<grid_of(b.base_rng[n]), 256, 0, st>>>(b); break;
        case 2: conv_bwd_fused_kernel<2><<<grid_of(b.base_rng[n]), 256, 0, st>>>(b); break;
        case 3: conv_bwd_fused_kernel<3><<<grid_of(b.base_rng[n]), 256, 0, st>>>(b); break;
        case 4: conv_bwd_fused_kernel<4><<<grid_of(b.base_rng[n]), 256, 0, st>>>(b); break;
        default: return cudaErrorInvalidValue;
    }
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_convert(const void* src, int src_dt, void* dst, int dst_dt, int64_t n, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    int64_t grid = cdiv(n, 256);
    if (grid > 148 * 16) grid = 148 * 16;
    convert_kernel<<<(unsigned)grid, 256, 0, st>>>(src, src_dt, dst, dst_dt, n);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
