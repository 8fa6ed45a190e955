// State pass of one recurrent decode step, with the combine fused in
// (constant cost per token: the authors' MoM blog post, introduction and
// inference-efficiency section; "MoM: Linear Sequence Modeling with
// Mixture-of-Memories", Summary).
//
// For sequence b and head h the CTA walks the top_k routed slots and the
// shared slot.  Each slot's state rows are read once, updated in place and
// written once:
//   y = S k, z = S q (one pass over S), u = beta (v - alpha y),
//   S' = alpha S + u k^T, o = scale (alpha z + u (k . q)),
// (with the scalar-gated linear rule u = beta v: no delta correction; with
// per-memory gates a routed slot takes its memory's own beta and alpha)
//   out += w_slot * o   (w = router gate, 1 for the shared memory).
// The state stream (read + write of (k+1) * d * d floats per sequence and
// head) is the whole cost, so the kernel is written for HBM bandwidth:
// 16-byte loads, every load of a slot issued before its reductions.
#include "common.cuh"
#include "kernels.h"

namespace mom {

static constexpr int RPW = 4, WPB = 8;

template <typename T, int D>
__global__ void __launch_bounds__(WPB * 32)
decode_state_kernel(DecodeArgs a) {
    constexpr int E = D / 32;
    constexpr int TILES = D / (RPW * WPB);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = blockIdx.x / TILES, tile = blockIdx.x % TILES, h = blockIdx.y;
    const int H = a.H, M = a.M, K = a.K;
    const int row0 = (tile * WPB + warp) * RPW;
    const T* q = reinterpret_cast<const T*>(a.q);

    float qq[E];
    load_vec<E>(q + ((int64_t)b * H + h) * D + lane * E, qq);
    const float be_tok = a.beta[(int64_t)b * H + h];
    const float la_tok = a.log_alpha[(int64_t)b * H + h];
    const bool delta = a.rule == MOM_RULE_GATED_DELTA;

    float out_acc[RPW];
#pragma unroll
    for (int i = 0; i < RPW; ++i) out_acc[i] = 0.f;

    for (int j = 0; j <= K; ++j) {
        int m;
        int64_t r;
        float w;
        const T *kb, *vb;
        if (j < K) {
            m = a.idx[(int64_t)b * K + j];
            r = a.row_of[(int64_t)b * K + j];
            w = a.gate[(int64_t)b * K + j];
            kb = reinterpret_cast<const T*>(a.k_p);
            vb = reinterpret_cast<const T*>(a.v_p);
            if (m < 0 || m >= M || r < 0 || r >= (int64_t)a.B * K) {
                if (threadIdx.x == 0 && tile == 0) record_error(a.ws, MOM_DEVERR_MEM_INDEX, b);
                continue;
            }
        } else {
            m = M;
            r = b;
            w = 1.f;
            kb = reinterpret_cast<const T*>(a.k_sh);
            vb = reinterpret_cast<const T*>(a.v_sh);
        }
        // the slot's gates: its memory's own for a routed slot when given
        const bool own = j < K && a.beta_p;
        const float be = own ? a.beta_p[r * H + h] : be_tok;
        const float al = expf(own ? a.log_alpha_p[r * H + h] : la_tok);
        const float dl = delta ? al : 0.f;
        float* Sp = a.state + ((((int64_t)b * (M + 1) + m) * H + h) * D + row0) * D + lane * E;
        float S[RPW][E];
#pragma unroll
        for (int i = 0; i < RPW; ++i) load_vec<E>(Sp + (size_t)i * D, S[i]);
        float kk[E], vv[RPW];
        load_vec<E>(kb + (r * H + h) * D + lane * E, kk);
#pragma unroll
        for (int i = 0; i < RPW; ++i) vv[i] = to_f(vb[(r * H + h) * D + row0 + i]);

        float red[2 * RPW + 1];
        red[2 * RPW] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) red[2 * RPW] = fmaf(kk[e], qq[e], red[2 * RPW]);
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            float y = 0.f, z = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) { y = fmaf(S[i][e], kk[e], y); z = fmaf(S[i][e], qq[e], z); }
            red[2 * i] = y;
            red[2 * i + 1] = z;
        }
        warp_sum_n<2 * RPW + 1>(red);
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const float u = be * (vv[i] - dl * red[2 * i]);
#pragma unroll
            for (int e = 0; e < E; ++e) S[i][e] = fmaf(al, S[i][e], u * kk[e]);
            out_acc[i] = fmaf(w, a.scale * fmaf(al, red[2 * i + 1], u * red[2 * RPW]), out_acc[i]);
            store_vec<E>(Sp + (size_t)i * D, S[i]);
        }
    }
    T* out = reinterpret_cast<T*>(a.out);
    float mine = 0.f;
#pragma unroll
    for (int i = 0; i < RPW; ++i) if (lane == i) mine = out_acc[i];
    if (lane < RPW) out[((int64_t)b * H + h) * D + row0 + lane] = from_f<T>(mine);
}

template <typename T, int D>
static cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
    dim3 grid((unsigned)a.B * (D / (RPW * WPB)), a.H);
    decode_state_kernel<T, D><<<grid, WPB * 32, 0, st>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_decode_state(const DecodeArgs& a, int dt, cudaStream_t st) {
    if (a.B == 0) return cudaSuccess;
    if (dt == MOM_BF16) {
        switch (a.d) {
            case 64: return launch_t<bf16, 64>(a, st);
            case 128: return launch_t<bf16, 128>(a, st);
            case 256: return launch_t<bf16, 256>(a, st);
        }
    } else {
        switch (a.d) {
            case 64: return launch_t<float, 64>(a, st);
            case 128: return launch_t<float, 128>(a, st);
            case 256: return launch_t<float, 256>(a, st);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace mom
