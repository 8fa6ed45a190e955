// Grouped projections on CUDA cores: every output tile is one head (DH
// columns) of one projection, so the per-head L2 norm of q and k is fused in
// the epilogue (the whole head row lives in one warp).  Used in float32 mode,
// where tf32 tensor cores would miss a 1e-4 tolerance, and for shapes the
// tcgen05 path does not take.
//
// Problems ("MoM: Linear Sequence Modeling with Mixture-of-Memories",
// Summary: a shared query and each memory's own key/value projections):
//   shared : all tokens x [W_q | W_k_sh | W_v_sh]          -> q, k_sh, v_sh
//   memory m: reordered rows mem_offset[m].. (token perm_token[r])
//             x [W_k^m | W_v^m]                             -> k_p, v_p
// Tiles never straddle two memories; the number of routed tiles is read from
// mem_offset on the device, and CTAs past the last tile exit.
#include "common.cuh"
#include "kernels.h"

namespace mom {

static constexpr int BM = 64, BK = 32, NT = 256;

template <typename T, int DH>
__global__ void __launch_bounds__(NT)
proj_simt_kernel(ProjArgs a, int64_t sh_tiles) {
    constexpr int NJ = DH / 32;        // columns per thread
    __shared__ float As[BK][BM + 1];
    __shared__ float Bs[BK][DH + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, D = a.D;
    const T* x = reinterpret_cast<const T*>(a.x);

    // ---- which tile is this CTA? ----
    int64_t bid = blockIdx.x;
    int64_t r_begin, r_end;
    int cb, part, m = -1;
    const T* W;
    T* out;
    bool norm;
    float* nout;
    if (bid < sh_tiles) {
        const int nb = 3 * H;
        cb = (int)(bid % nb);
        r_begin = (bid / nb) * BM;
        r_end = (r_begin + BM < a.n_tok ? r_begin + BM : a.n_tok);
        part = cb / H;
        W = reinterpret_cast<const T*>(a.w_shared) + (size_t)cb * DH * D;
        out = reinterpret_cast<T*>(part == 0 ? a.q : part == 1 ? a.k_sh : a.v_sh);
        norm = part < 2;
        nout = part == 0 ? a.q_norm : part == 1 ? a.k_sh_norm : nullptr;
    } else {
        const int nb = 2 * H;
        int64_t local = bid - sh_tiles;
        cb = (int)(local % nb);
        int64_t rt = local / nb;
        const int64_t n_rows = a.routed_rows();
        for (int g = 0; g < a.groups(); ++g) {
            int64_t lo = a.mem_offset[g], hi = a.mem_offset[g + 1];
            const int gm = a.group_mem ? a.group_mem[g] : g;
            if (lo < 0 || hi < lo || hi > n_rows || gm < 0 || gm >= a.M) {   // corrupted table: touch nothing
                if (cb == 0) record_error(a.ws, MOM_DEVERR_SEGMENT, g);
                return;
            }
            int64_t nt = cdiv(hi - lo, BM);
            if (rt < nt) { m = gm; r_begin = lo + rt * BM; r_end = (r_begin + BM < hi ? r_begin + BM : hi); break; }
            rt -= nt;
        }
        if (m < 0) return;
        part = cb / H;
        W = reinterpret_cast<const T*>(a.w_kv) + ((size_t)m * 2 * H * DH + (size_t)cb * DH) * D;
        out = reinterpret_cast<T*>(part == 0 ? a.k_p : a.v_p);
        norm = part == 0;
        nout = part == 0 ? a.k_p_norm : nullptr;
    }
    const int h = cb % H;

    // source token of each of this tile's rows (for the A loads)
    const int lrow = tid >> 2, kq = (tid & 3) * 8;
    int64_t src = -1;
    {
        int64_t r = r_begin + lrow;
        if (r < r_end) {
            src = (m < 0 || !a.perm_token) ? r : (int64_t)a.perm_token[r];
            if (src < 0 || src >= a.n_tok) { record_error(a.ws, MOM_DEVERR_ROW_INDEX, r); src = -1; }
        }
    }

    float acc[8][NJ];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < D; k0 += BK) {
        float v8[8];
        if (src >= 0) load_vec<8>(x + src * D + k0 + kq, v8);
        else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v8[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) As[kq + e][lrow] = v8[e];
#pragma unroll
        for (int c = 0; c < DH / 64; ++c) {
            const int n = lrow + 64 * c;
            load_vec<8>(W + (size_t)n * D + k0 + kq, v8);
#pragma unroll
            for (int e = 0; e < 8; ++e) Bs[kq + e][n] = v8[e];
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < BK; ++kk) {
            float av[8], bv[NJ];
#pragma unroll
            for (int i = 0; i < 8; ++i) av[i] = As[kk][warp + 8 * i];
#pragma unroll
            for (int j = 0; j < NJ; ++j) bv[j] = Bs[kk][lane + 32 * j];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < NJ; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = r_begin + warp + 8 * i;
        float sc = 1.f;
        if (norm) {
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < NJ; ++j) ss = fmaf(acc[i][j], acc[i][j], ss);
            ss = warp_sum(ss);
            sc = rsqrtf(ss + 1e-6f);
            if (nout && lane == 0 && r < r_end) nout[r * H + h] = sqrtf(ss + 1e-6f);
        }
        if (r < r_end) {
            T* o = out + (r * H + h) * DH;
#pragma unroll
            for (int j = 0; j < NJ; ++j) o[lane + 32 * j] = from_f<T>(acc[i][j] * sc);
        }
    }
}

template <typename T, int DH>
static cudaError_t launch_t(const ProjArgs& a, cudaStream_t st) {
    const int64_t sh_tiles = (a.parts & PROJ_SHARED) ? cdiv(a.n_tok, BM) * 3 * a.H : 0;
    const int64_t rt_tiles = (a.parts & PROJ_ROUTED) ? (cdiv(a.routed_rows(), BM) + a.groups()) * 2 * a.H : 0;
    const int64_t grid = sh_tiles + rt_tiles;
    if (grid == 0) return cudaSuccess;
    proj_simt_kernel<T, DH><<<(unsigned)grid, NT, 0, st>>>(a, sh_tiles);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_proj_simt(const ProjArgs& a, int dt, cudaStream_t st) {
    if (a.n_tok == 0) return cudaSuccess;
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
