// Gated DeltaNet recurrence, token by token, on CUDA cores.
//
//   S_r = alpha_r S_{r-1} (I - beta_r k_r k_r^T) + beta_r v_r k_r^T,  o_r = S_r (scale q_r)
//
// or, with the scalar-gated linear rule, S_r = alpha_r S_{r-1} + beta_r v_r k_r^T
// (u_i = beta v_i below: the delta correction -alpha y_i drops out).
//
// (the authors' MoM blog post, experiments section: every memory uses Gated
// DeltaNet's gate and update rule).  Each row i of S (one d_v index) evolves
// on its own given k, beta and alpha:
//   y_i = S_i . k,  z_i = S_i . q,  u_i = beta (v_i - alpha y_i),
//   S_i <- alpha S_i + u_i k,       o_i = alpha z_i + u_i (k . q)
// so one warp owns RPW rows, each lane D/32 contiguous columns of them, and
// only warp reductions couple the lanes.  This is the exact float32 path
// (float32 mode: chunk size 1) and the fallback for shapes the tensor-core
// chunk kernel does not take.
#include "common.cuh"
#include "kernels.h"

namespace mom {

static constexpr int RPW = 4;     // state rows per warp
static constexpr int WPB = 4;     // warps per CTA

template <typename T, int D>
__global__ void __launch_bounds__(WPB * 32)
gdn_recurrent_kernel(GdnArgs a) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int TILES = D / (RPW * WPB);
    const int seg = blockIdx.x / TILES, h = blockIdx.y, H = a.H;
    const int tile = blockIdx.x % TILES;
    const int row0 = (tile * WPB + warp) * RPW;
    const T* q = reinterpret_cast<const T*>(a.q);
    const T* k = reinterpret_cast<const T*>(a.k);
    const T* v = reinterpret_cast<const T*>(a.v);
    T* o = reinterpret_cast<T*>(a.o);

    int64_t r0 = a.seg_cu[seg], r1 = a.seg_cu[seg + 1];
    if (r0 < 0 || r1 < r0 || r1 > a.n_rows) {
        if (threadIdx.x == 0 && tile == 0 && h == 0) record_error(a.ws, MOM_DEVERR_SEGMENT, seg);
        r1 = r0;   // process nothing; still write h_final = h0
    }

    float S[RPW][E];
    const size_t sbase = ((size_t)seg * H + h) * D * D;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        if (a.h0) load_vec<E>(a.h0 + sbase + (size_t)(row0 + i) * D + lane * E, S[i]);
        else {
#pragma unroll
            for (int e = 0; e < E; ++e) S[i][e] = 0.f;
        }
    }

    for (int64_t r = r0; r < r1; ++r) {
        int64_t qr = a.qidx ? (int64_t)a.qidx[r] : r;
        if (qr < 0 || qr >= a.n_q_rows) {
            if (lane == 0 && warp == 0 && tile == 0) record_error(a.ws, MOM_DEVERR_ROW_INDEX, r);
            continue;
        }
        float kk[E], qq[E], vv[RPW];
        load_vec<E>(k + (r * H + h) * D + lane * E, kk);
        load_vec<E>(q + (qr * H + h) * D + lane * E, qq);
#pragma unroll
        for (int i = 0; i < RPW; ++i) vv[i] = to_f(v[(r * H + h) * D + row0 + i]);
        const int64_t gr = a.gates_by_row ? r : qr;
        const float b = a.beta[gr * H + h];
        const float al = expf(a.log_alpha[gr * H + h]);

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
        const float kq = red[2 * RPW];
        float my_o = 0.f;
        const float dl = a.rule == MOM_RULE_GATED_DELTA ? al : 0.f;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const float u = b * (vv[i] - dl * red[2 * i]);
#pragma unroll
            for (int e = 0; e < E; ++e) S[i][e] = fmaf(al, S[i][e], u * kk[e]);
            const float oi = a.scale * fmaf(al, red[2 * i + 1], u * kq);
            if (lane == i) my_o = oi;
        }
        if (lane < RPW) o[(r * H + h) * D + row0 + lane] = from_f<T>(my_o);
    }

    if (a.h_final) {
#pragma unroll
        for (int i = 0; i < RPW; ++i) store_vec<E>(a.h_final + sbase + (size_t)(row0 + i) * D + lane * E, S[i]);
    }
}

template <typename T, int D>
static cudaError_t launch_t(const GdnArgs& a, cudaStream_t st) {
    dim3 grid((unsigned)a.n_seg * (D / (RPW * WPB)), a.H);
    gdn_recurrent_kernel<T, D><<<grid, WPB * 32, 0, st>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gdn_recurrent(const GdnArgs& a, int dt, cudaStream_t st) {
    if (!(a.phase & GDN_STATE)) return cudaSuccess;   // token-serial: nothing to prepare
    if (a.n_seg == 0) return cudaSuccess;
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
