// Chunked Gated DeltaNet on the tcgen05 tensor cores: bf16 operands, fp32
// state carried across chunks in TMEM.
//
// The recurrence of every memory (the authors' MoM blog post, experiments
// section: Gated DeltaNet's gate and update rule)
//   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t
// is evaluated in chunks of C = 64 rows.  With gamma_r the running sum of
// log alpha inside the chunk, S the state at the chunk start, and
// Tb = (I + L)^-1 diag(beta), L_rs = beta_r e^(gamma_r - gamma_s) k_r.k_s (s < r):
//   U^T = Y Tb^T,   Y = V^T - (S K^T) diag(e^gamma)                 (d_v x C)
//   o_r = e^(gamma_r) S q_r + sum_{s<=r} e^(gamma_r-gamma_s) (q_r.k_s) u_s
//   S'  = e^(gamma_C) S + sum_s e^(gamma_C-gamma_s) u_s k_s^T
// where u_r = beta_r (v_r - alpha_r S_{r-1} k_r) are the delta-rule
// corrections.  U enters both the output and the next state only through
// products with state-independent matrices, so the serial walk never forms
// it: with P_rs = e^(gamma_r-gamma_s) q_r.k_s (s <= r),
//   O = e^gamma S Q^T + Y (P Tb)^T,   S' = e^(gamma_C) S + Y Tb^T diag(e^(gamma_C-gamma)) K.
// Every product keeps the d_v rows of S as the MMA's M dimension (128 TMEM
// lanes): every walk MMA is M = 128.
//
// Three launches per call, in two stream-ordered phases (the prep of
// every chunk does not depend on the state):
//   schedule: chunk offsets of every segment (device-side, no host sync)
//   prep    : per (chunk, head): G = [K;Q] K^T on the tensor cores; the
//             decay matrix by running products of alpha; T = (I + L)^-1 by
//             16 x 16 blocks (diagonal blocks by forward substitution in
//             fp32, off-diagonal block products on tf32 tensor cores); then
//             on the tensor cores Wk = Tb^T diag(e^(gamma_C-gamma)) K and
//             Q' = P Tb, stored as one bf16 image per (chunk, head)
//   state   : per (segment, head, 128-row d_v tile), the serial walk over the
//             segment's chunks with the state resident in TMEM (T = rho S,
//             fp32) and its bf16 copy in TMEM as the A operand of Z = T K^T
//             and X = T q~^T; per chunk Y = V^T - Z diag(e^gamma / rho), then
//             X += Y Q'^T and T <- 2^-e T + (rho' Y) Wk.  The chunk decay is
//             the MMA's power-of-two accumulator scale plus a change of the
//             running scalar rho.  Roles: one producer warp (TMA and bulk
//             loads, chunk gates), three q~ warps (q rows, through the index
//             when given, scaled in place), one MMA warp (Z in two d_k
//             halves, then X), eight math warps (the last to finish Y issues
//             the output and state-update MMAs).
// The scalar-gated linear rule S_t = alpha_t S_{t-1} + beta_t v_t k_t^T runs
// the same kernels with L = 0 (so T = I, U = diag(beta) V) and Y = V^T.
// Rows past a segment's end are masked (zero gates, zeroed or masked rows),
// so a ragged tail chunk needs no padding.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mom {
namespace {

using namespace sm100;

constexpr int C = 64;                 // chunk length
constexpr int DVT = 128;              // d_v rows per state CTA (TMEM lanes)
constexpr int IMG = C * C * 2;        // one swizzled 64x64 bf16 tile
constexpr int GB = C + 4;             // floats per chunk-gate record

struct GdnTc {
    const bf16* q;
    const int32_t* qidx;
    const bf16* k;
    const bf16* v;
    const float* beta;
    const float* la;
    const int32_t* seg_cu;
    int n_seg;
    int64_t n_rows, n_q_rows;
    int H;
    float scale;
    const float* h0;
    float* h_final;
    bf16* o;
    int32_t* chunk_cu;
    int4* chunk_info;     // per chunk: segment, first row, rows (<= C)
    unsigned char* img;
    void* err;
    int delta;            // 1: the Gated DeltaNet rule; 0: the scalar-gated linear rule (L = 0, Y = V^T)
    int gates_by_row;     // 1: beta / la [n_rows, H], one per row of k / v (per-memory gates)
};

// ------------------------------------------------------------- schedule --
__global__ void __launch_bounds__(1024)
gdn_schedule_kernel(const int32_t* __restrict__ seg_cu, int n_seg, int64_t n_rows, int32_t* __restrict__ chunk_cu,
                    int4* __restrict__ chunk_info, void* err) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) { carry = 0; chunk_cu[0] = 0; }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < n_seg; base += 1024) {
        const int s = base + threadIdx.x;
        int32_t cnt = 0;
        if (s < n_seg) {
            const int64_t a = seg_cu[s], b = seg_cu[s + 1];
            if (a < 0 || b < a || b > n_rows) record_error(err, MOM_DEVERR_SEGMENT, s);
            else cnt = (int32_t)((b - a + C - 1) / C);
        }
        int32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int32_t w = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int32_t t = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += t;
            }
            warp_tot[lane] = w;
        }
        __syncthreads();
        if (s < n_seg) chunk_cu[s + 1] = carry + (warp ? warp_tot[warp - 1] : 0) + incl;
        __syncthreads();
        if (threadIdx.x == 0) carry += warp_tot[31];
        __syncthreads();
    }
    // every chunk's segment, first row and length (chunk_cu is visible to the CTA after the barrier)
    for (int s = threadIdx.x; s < n_seg; s += 1024) {
        const int c0 = chunk_cu[s], c1 = chunk_cu[s + 1];
        const int a = seg_cu[s], b = seg_cu[s + 1];
        for (int c = c0; c < c1; ++c) {
            const int r0 = a + (c - c0) * C;
            chunk_info[c] = make_int4(s, r0, b - r0 < C ? b - r0 : C, 0);
        }
    }
}

// Gates of one chunk, by one full warp (lane l holds rows 2l and 2l+1):
// beta (0 past n) and log alpha (0 past n), loaded from global memory
// (through the row index when given, unless the gates are per row).
__device__ __forceinline__ void chunk_gates_load(const GdnTc& p, int64_t r0, int n, int h, int lane, float (&b)[2],
                                                 float (&l)[2]) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int s = 2 * lane + e;
        b[e] = 0.f;
        l[e] = 0.f;
        if (s < n) {
            const int64_t r = r0 + s;
            const int64_t qr = (p.qidx && !p.gates_by_row) ? (int64_t)p.qidx[r] : r;
            // per-row gates leave the index unread here: pull its line into L1
            // for the q-row gather, which looks it up next
            if (p.gates_by_row && p.qidx) asm volatile("prefetch.global.L1 [%0];" ::"l"(p.qidx + r));
            if (qr >= 0 && qr < (p.gates_by_row ? p.n_rows : p.n_q_rows)) {
                b[e] = p.beta[qr * p.H + h];
                l[e] = p.la[qr * p.H + h];
            } else {
                record_error(p.err, MOM_DEVERR_ROW_INDEX, r);
            }
        }
    }
}

// gamma, the running sum of log alpha from the chunk start, of the loaded
// gates; returns gamma of the last valid row.  Both the prep and the state
// kernel derive their factors from this one scan, so they agree bit for bit.
__device__ __forceinline__ float chunk_gates_scan(const float (&l)[2], int n, int lane, float (&g)[2]) {
    const float pair = l[0] + l[1];
    float incl = pair;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    g[0] = incl - pair + l[0];
    g[1] = incl;
    const int last = n - 1;
    return __shfl_sync(0xffffffffu, (last & 1) ? g[1] : g[0], last >> 1);
}

__device__ __forceinline__ float chunk_scan(const GdnTc& p, int64_t r0, int n, int h, int lane, float (&b)[2],
                                            float (&g)[2]) {
    float l[2];
    chunk_gates_load(p, r0, n, h, lane, b, l);
    return chunk_gates_scan(l, n, lane, g);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t* v) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, float* v) {
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]) : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h2);
}

// Gathering 64 rows x D of a bf16 [rows, H, D] array through an index into
// 128-byte-swizzled 64-column slabs, by NT threads (thread t: items t, t +
// NT, ...; item = (row, 16-byte column chunk)), in two steps: the source
// rows of a thread's items (-1 past n or for a bad index: zero-filled), then
// the copies.  All index loads of a step are in flight together -- between
// the copies' asm statements they would each wait a full round trip -- and a
// caller can issue the first step a chunk ahead.
template <int NT>
struct GatherRows {
    static constexpr int ITEMS = (C * 8 + NT - 1) / NT;
    int32_t src[ITEMS];   // row indices fit: qidx is int32, and n_rows < 2^31 / C

    __device__ __forceinline__ void rows(const GdnTc& p, int64_t r0, int n, int t) {
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int idx = t + i * NT, row = idx >> 3;
            src[i] = -1;
            if (idx < C * 8 && row < n) {
                const int64_t r = r0 + row;
                const int64_t qr = p.qidx ? (int64_t)__ldg(p.qidx + r) : r;
                src[i] = (qr >= 0 && qr < p.n_q_rows) ? (int32_t)qr : -1;
            }
        }
    }

    template <int D>
    __device__ __forceinline__ void copy(const GdnTc& p, const bf16* base, int h, uint32_t dst, uint32_t slab_stride,
                                         int t) const {
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int idx = t + i * NT;
            if (idx < C * 8) {
                const int row = idx >> 3, c8 = idx & 7;
                const bf16* s = base + ((int64_t)(src[i] >= 0 ? src[i] : 0) * p.H + h) * D + c8 * 8;
                const uint32_t d0 = dst + row * 128 + ((c8 ^ (row & 7)) << 4);
#pragma unroll
                for (int j = 0; j < D / 64; ++j) cp_async_16(d0 + j * slab_stride, s + j * 64, src[i] >= 0 ? 16u : 0u);
            }
        }
    }
};

// ----------------------------------------------------------------- prep --
// The prep computes, per (chunk, head), everything the serial walk needs
// that does not depend on the state, in the form the walk's two products
// take it:
//   Wk = Tb^T diag(e^(gamma_C - gamma)) K     (C x d_k): the state update is
//        T <- 2^-e T + (rho' Y) Wk, with Y = V^T - Z~ and rho' the next
//        running scale (U^T diag(dec) K = Y Tb^T diag(dec) K);
//   Q' = P Tb                                  (C x C):  the output is
//        X += Y Q'^T  (U^T P^T = Y Tb^T P^T).
// Both leave as one contiguous bf16 image per (chunk, head): Wk rows j of
// the d_k columns (64 chunk positions each, 128-byte swizzled, K-major for
// the walk's state update), then Q' rows r (the same format).

// fp32 64 x 64 work tile in two 32-row halves of 32 x 64 floats (8 KB each,
// no padding), the column index XOR-ed with the row: a warp walking one
// column over 32 rows, or one row over 32 columns, touches 32 banks.
struct Tile {
    float* lo;
    float* hi;
    __device__ __forceinline__ float& at(int r, int s) const {
        return (r < 32 ? lo : hi)[(r & 31) * 64 + (s ^ (r & 31))];
    }
};

constexpr int PREP_THREADS = 256;      // 8 warps per (chunk, head)

// 2^x by the hardware approximation (an error of a few units in the last
// place of fp32; results below 2^-126 flush to 0): the prep's decay factors,
// which are rounded to bf16 afterwards.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Writes NCH 16-byte chunks (8 fp32 values each, rounded to bf16) of row r,
// starting at chunk c8_0, into a 128-byte-swizzled 64-column image.
template <int NCH>
__device__ __forceinline__ void image_chunks(unsigned char* __restrict__ img, int r, int c8_0, const float* v) {
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        const float* w = v + 8 * k;
        const int c8 = c8_0 + k;
        *reinterpret_cast<uint4*>(img + r * 128 + ((c8 ^ (r & 7)) << 4)) =
            make_uint4(pack_bf16(w[0], w[1]), pack_bf16(w[2], w[3]), pack_bf16(w[4], w[5]), pack_bf16(w[6], w[7]));
    }
}

// Writes 64 fp32 values of row r as bf16 into a 128-byte-swizzled 64 x 64
// shared-memory image.
__device__ __forceinline__ void image_row(unsigned char* __restrict__ img, int r, const float (&v)[64]) {
    image_chunks<8>(img, r, 0, v);
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// d (16 x 8, fp32) += A (16 x 8) * B (8 x 8): one m16n8k8 tf32 tensor-core
// product with fp32 accumulation; a(i, k) and b(k, j) fetch the operands.
template <class FA, class FB>
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], FA a, FB b, int lane) {
    const int g = lane >> 2, c = lane & 3;
    const uint32_t a0 = to_tf32(a(g, c)), a1 = to_tf32(a(g + 8, c));
    const uint32_t a2 = to_tf32(a(g, c + 4)), a3 = to_tf32(a(g + 8, c + 4));
    const uint32_t b0 = to_tf32(b(c, g)), b1 = to_tf32(b(c + 4, g));
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One level of the blocked inverse: the 16 x 16 blocks at distance LEV below
// the diagonal, T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj (i = j + LEV), from the
// blocks closer to the diagonal.  The 16 x 16 block products run on the
// tensor cores (tf32 operands, fp32 accumulation; T is rounded to bf16 for
// its use anyway): a task is one 8-column half of one block, spread over
// the warps.
template <int LEV>
__device__ __forceinline__ void offdiag_level(const Tile& Lm, const Tile& Tm, float* Mb, int tid) {
    constexpr int NB = 4 - LEV;
    constexpr int NW = PREP_THREADS / 32;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    // M_q = sum_kb L[bi][bj+kb] T[bj+kb][bj]        (bi = LEV + q, bj = q)
    for (int task = warp; task < 2 * NB; task += NW) {
        const int q = task >> 1, nh = task & 1;
        const int bi = LEV + q, bj = q;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kb = 0; kb < LEV; ++kb)
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int k0 = 16 * (bj + kb) + 8 * ks;
                mma_tf32_16x8x8(d, [&](int i, int k) { return Lm.at(16 * bi + i, k0 + k); },
                                [&](int k, int j) { return Tm.at(k0 + k, 16 * bj + 8 * nh + j); }, lane);
            }
        float* m = Mb + q * 256;
        m[g * 16 + 8 * nh + 2 * c] = d[0];
        m[g * 16 + 8 * nh + 2 * c + 1] = d[1];
        m[(g + 8) * 16 + 8 * nh + 2 * c] = d[2];
        m[(g + 8) * 16 + 8 * nh + 2 * c + 1] = d[3];
    }
    __syncthreads();
    // T[bi][bj] = -T[bi][bi] M_q
    for (int task = warp; task < 2 * NB; task += NW) {
        const int q = task >> 1, nh = task & 1;
        const int bi = LEV + q, bj = q;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const float* mq = Mb + q * 256 + (8 * ks) * 16 + 8 * nh;
            mma_tf32_16x8x8(d, [&](int i, int k) { return Tm.at(16 * bi + i, 16 * bi + 8 * ks + k); },
                            [&](int k, int j) { return mq[k * 16 + j]; }, lane);
        }
        const int r0 = 16 * bi, c0 = 16 * bj + 8 * nh;
        Tm.at(r0 + g, c0 + 2 * c) = -d[0];
        Tm.at(r0 + g, c0 + 2 * c + 1) = -d[1];
        Tm.at(r0 + g + 8, c0 + 2 * c) = -d[2];
        Tm.at(r0 + g + 8, c0 + 2 * c + 1) = -d[3];
    }
    __syncthreads();
}

template <int D>
struct PrepLayout {
    static constexpr int SLABS = D / 64;
    // per 64-column slab: K rows 0..63 | q rows 64..127 (16 KB)
    static constexpr int KQ = 0;
    static constexpr int KQ_BYTES = SLABS * 16384;
    // the four 8 KB halves of the fp32 tiles T and L: in the q halves of the
    // slabs once G has read them (the K halves stay for the Wk product), the
    // rest after the slabs.  After the solve the bf16 images take their
    // place: Tb over L's first half, TD over L's second, P over T's first.
    static constexpr int EXTRA = SLABS >= 4 ? 0 : (4 - SLABS) * 8192;
    static constexpr int MB = KQ_BYTES + EXTRA;               // fp32 3 x [16][16] block products
    static constexpr int GBB = MB + 3 * 256 * 4;              // beta, gamma log2(e) [64]
    static constexpr int BARS = GBB + 2 * C * 4;              // land, G done, products done (x2)
    static constexpr int MISC = BARS + 32;
    static constexpr size_t BYTES = 1024 + MISC + 16;
    static constexpr int OUT = D * 128 + IMG;                 // output image bytes: Wk rows, then Q'
    // TMEM: G, then one 128-column-of-d_k half of Wk^T and Q' per round
    static constexpr uint32_t TMEM_COLS = 128;
    // output staging (every region dead by then): the round-1 Wk half and Q',
    // then (d = 256) the second round's Wk half
    static constexpr int ST_W1 = D == 256 ? 24576 : 0;
    static constexpr int ST_Q = D == 256 ? 40960 : 16384;
    static_assert(D == 256 || D == 128, "head dimension");
    static __device__ __forceinline__ int tile_half(int w) {
        return w < SLABS ? KQ + w * 16384 + 8192 : KQ_BYTES + (w - SLABS) * 8192;
    }
};

template <int D>
__global__ void __launch_bounds__(PREP_THREADS, 3)
gdn_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q, GdnTc p) {
    using Lay = PrepLayout<D>;
    constexpr int SLABS = D / 64, HALVES = SLABS / 2;
    constexpr float LOG2E_ = 1.4426950408889634f;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024_shared(smem_raw);
    const Tile Tm{reinterpret_cast<float*>(sm + Lay::tile_half(0)), reinterpret_cast<float*>(sm + Lay::tile_half(1))};
    const Tile Lm{reinterpret_cast<float*>(sm + Lay::tile_half(2)), reinterpret_cast<float*>(sm + Lay::tile_half(3))};
    float* Mb = reinterpret_cast<float*>(sm + Lay::MB);
    float* gbeta = reinterpret_cast<float*>(sm + Lay::GBB);
    float* g2 = gbeta + C;                                // gamma * log2(e)
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::BARS);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Lay::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    const uint32_t land = smem_u32(bars), mma_bar = smem_u32(bars + 1);
    const uint32_t mma2_bar = smem_u32(bars + 2), mma3_bar = smem_u32(bars + 3);
    const uint32_t kq = smem_u32(sm + Lay::KQ);
    unsigned char* pimg = sm + Lay::tile_half(0);
    unsigned char* tbimg = sm + Lay::tile_half(2);
    unsigned char* tdimg = sm + Lay::tile_half(3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.x, h = blockIdx.y;
    if (g >= p.chunk_cu[p.n_seg]) return;                 // uniform over the CTA
    const int4 info = p.chunk_info[g];
    const int64_t r0 = info.y;
    const int n = info.z;
    // TMEM lane quarter of this warp and the 32-column half of a 64-column
    // accumulator it reads (warps w and w + 4 share the lanes)
    const int quarter = warp & 3, colh = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    const int rho = 32 * quarter + lane;                  // this thread's TMEM lane

    // Everything the chunk reads is requested at once: K (and contiguous q)
    // by TMA, indexed q rows by warps 2-7, the gates by warp 0.  Rows past n
    // hold other data or zeros and are zeroed below.
    if (tid == 0) {
        mbar_init(land, 1);
        mbar_init(mma_bar, 1);
        mbar_init(mma2_bar, 1);
        mbar_init(mma3_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        mbar_arrive_expect_tx(land, SLABS * 8192 * (p.qidx ? 1 : 2));
#pragma unroll
        for (int j = 0; j < SLABS; ++j) {
            tma_load_2d(kq + j * 16384, &tm_k, land, h * D + 64 * j, (int)r0);
            if (!p.qidx) tma_load_2d(kq + j * 16384 + 8192, &tm_q, land, h * D + 64 * j, (int)r0);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tslot), Lay::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0) {
        float b[2], gg[2];
        chunk_scan(p, r0, n, h, lane, b, gg);
        gbeta[2 * lane] = b[0]; gbeta[2 * lane + 1] = b[1];
        g2[2 * lane] = gg[0] * LOG2E_; g2[2 * lane + 1] = gg[1] * LOG2E_;
    } else if (p.qidx && warp >= 2) {
        GatherRows<PREP_THREADS - 64> g;
        g.rows(p, r0, n, tid - 64);
        g.copy<D>(p, p.q, h, kq + 8192, 16384, tid - 64);
        cp_async_commit();
        cp_async_wait<0>();
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    // G = [K; q] K^T : M = 128, N = 64, K = D
    mbar_wait(land, 0, abort_flag, p.err, 10);
    __syncthreads();
    bool ok = *abort_flag == 0;                           // uniform after the barrier
    if (!ok) mbar_wait_drain(land, 0);                    // copies in flight land before we leave
    if (ok && n < C) {
        // rows past n belong to other segments (or were never written): zero
        // them, so that no product below can meet a non-finite value there
        for (int idx = tid; idx < (C - n) * 8 * SLABS * 2; idx += PREP_THREADS) {
            const int row = n + idx / (16 * SLABS), rest = idx % (16 * SLABS);
            const uint32_t dst = kq + (rest >> 4) * 16384 + ((rest >> 3) & 1) * 8192 + row * 128 + (rest & 7) * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(dst), "r"(0u) : "memory");
        }
        fence_proxy_async_smem();
    }
    __syncthreads();
    if (ok && tid == 0) {
        tc_fence_after();
        constexpr uint32_t ID = idesc_bf16_f32(128, 64);
#pragma unroll
        for (int j = 0; j < SLABS; ++j)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a = kq + j * 16384 + kk * 32;
                umma_f16(tmem, desc_kmajor_sw128(a), desc_kmajor_sw128(a), ID, (j | kk) != 0);
            }
        umma_commit(mma_bar);
    }
    if (ok) {
        if (!mbar_wait(mma_bar, 0, abort_flag, p.err, 11)) mbar_wait_drain(mma_bar, 0);   // q bytes free again
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abort_flag) {
        if (warp == 1) tmem_dealloc(tmem, Lay::TMEM_COLS);
        return;
    }
    // L = beta_r e^(gamma_r - gamma_s) k_r.k_s (s < r < n) into the L tile
    // from TMEM lanes 0..63 (the K rows of G), 32 columns per thread -- the
    // quadrant above the diagonal (warp 4) is never read -- while the warps
    // of lanes 64..127 (the q rows) form P = e^(gamma_r - gamma_s) q_r.k_s
    // (s <= r < n) in registers, written out once T's bytes are free.
    uint32_t pk[16];
    if (quarter < 2 && warp != 4) {
        uint32_t gv[32];
        tmem_ld_x32(tmem + lane_base + 32 * colh, gv);
        tmem_ld_wait();
        const int r = rho;
        // beta is 0 past n; without the delta correction L = 0 (T = I)
        const float g2r = g2[r], br = p.delta ? gbeta[r] : 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int s = 32 * colh + e;
            Lm.at(r, s) = s < r ? br * ex2_approx(g2r - g2[s]) * __uint_as_float(gv[e]) : 0.f;
        }
    } else if (quarter >= 2) {
        uint32_t gv[32];
        tmem_ld_x32(tmem + lane_base + 32 * colh, gv);
        tmem_ld_wait();
        const int r = rho - 64;
        const float g2r = g2[r];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const int s = 32 * colh + e;
            const float p0 = (s <= r && r < n) ? ex2_approx(g2r - g2[s]) * __uint_as_float(gv[e]) : 0.f;
            const float p1 = (s + 1 <= r && r < n) ? ex2_approx(g2r - g2[s + 1]) * __uint_as_float(gv[e + 1]) : 0.f;
            pk[e / 2] = pack_bf16(p0, p1);
        }
    }
    // T = (I + L)^-1 in 16 x 16 blocks.  Diagonal blocks: forward
    // substitution, one column per thread, by the two warps whose L quadrants
    // hold them (warp 0: blocks 0 and 1, warp 5: blocks 2 and 3), as soon as
    // their own rows are written.
    if (warp == 0 || warp == 5) {
        __syncwarp();
        const int bk = (warp == 5 ? 2 : 0) + (lane >> 4), cc = lane & 15, base = 16 * bk;
        float t[16];
#pragma unroll
        for (int rl = 0; rl < 16; ++rl) t[rl] = rl == cc ? 1.f : 0.f;
#pragma unroll
        for (int rl = 1; rl < 16; ++rl) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int sl = 0; sl < rl; ++sl) {
                const float l = Lm.at(base + rl, base + sl);
                if (sl & 1) a1 = fmaf(l, t[sl], a1); else a0 = fmaf(l, t[sl], a0);
            }
            if (rl > cc) t[rl] = -(a0 + a1);
        }
#pragma unroll
        for (int rl = 0; rl < 16; ++rl) Tm.at(base + rl, base + cc) = t[rl];
    }
    __syncthreads();
    // Off-diagonal blocks by distance from the diagonal:
    //   T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj      (i > j)
    offdiag_level<1>(Lm, Tm, Mb, tid);
    offdiag_level<2>(Lm, Tm, Mb, tid);
    offdiag_level<3>(Lm, Tm, Mb, tid);
    // Tb = T diag(beta) and diag(e^(gamma_C - gamma)) Tb over L's bytes: row
    // r, 16 columns per thread (rows past n are zero, beta being 0 there)
    {
        const int r = tid & 63, q4 = tid >> 6;
        const float dec = ex2_approx(g2[n - 1] - g2[r]);
        float v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int s = 16 * q4 + e;
            v[e] = s <= r ? Tm.at(r, s) * gbeta[s] : 0.f;
        }
        image_chunks<2>(tbimg, r, 2 * q4, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] *= dec;
        image_chunks<2>(tdimg, r, 2 * q4, v);
    }
    // P over T's first half once T is read
    __syncthreads();
    if (quarter >= 2) {
        const int r = rho - 64;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int c8 = 4 * colh + k;
            *reinterpret_cast<uint4*>(pimg + r * 128 + ((c8 ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // Products on the tensor cores, D[j, t] over s:
    //   Wk^T = K^T TD: A = K^T (MN-major view of two K slabs), B = TD (MN-major)
    //   Q'  = P Tb:   A = P (K-major; rows 64..127 read the next 8 KB and are
    //                 discarded), B = Tb (MN-major)
    constexpr uint32_t IDW = idesc_bf16_f32(128, 64, 1, 1);
    constexpr uint32_t IDQ = idesc_bf16_f32(128, 64, 0, 1);
    auto issue_wk = [&](int half) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem, desc_mnmajor_sw128(kq + 2 * half * 16384 + kk * 2048, 16384),
                     desc_mnmajor_sw128(smem_u32(tdimg) + kk * 2048, 8192), IDW, kk != 0);
    };
    // one Wk^T half (TMEM lanes j, columns 0..63) into rows j of the staged image
    auto read_wk = [&](int half, unsigned char* st) {
        uint32_t w[32];
        tmem_ld_x32(tmem + lane_base + 32 * colh, w);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(w[e]);
        image_chunks<4>(st, rho, 4 * colh, v);
        (void)half;
    };
    // round 1: the last Wk half and Q'
    if (tid == 0) {
        tc_fence_after();
        issue_wk(HALVES - 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + 64, desc_kmajor_sw128(smem_u32(pimg) + kk * 32),
                     desc_mnmajor_sw128(smem_u32(tbimg) + kk * 2048, 8192), IDQ, kk != 0);
        umma_commit(mma2_bar);
    }
    if (!mbar_wait(mma2_bar, 0, abort_flag, p.err, 12)) mbar_wait_drain(mma2_bar, 0);
    tc_fence_after();
    __syncthreads();
    bool fail = *abort_flag != 0;
    unsigned char* img = p.img + ((size_t)g * p.H + h) * (size_t)Lay::OUT;
    if (!fail) {
        read_wk(HALVES - 1, sm + Lay::ST_W1);
        if (quarter < 2) {
            uint32_t w[32];
            tmem_ld_x32(tmem + lane_base + 64 + 32 * colh, w);
            tmem_ld_wait();
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(w[e]);
            image_chunks<4>(sm + Lay::ST_Q, rho, 4 * colh, v);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (!fail && tid == 0) {
        if (HALVES == 2) {
            bulk_store(img + 16384, smem_u32(sm + Lay::ST_W1), 16384);
            bulk_store(img + D * 128, smem_u32(sm + Lay::ST_Q), IMG);
            // round 2: the first Wk half, over the same TMEM columns (read out above)
            tc_fence_after();
            issue_wk(0);
            umma_commit(mma3_bar);
        } else {
            bulk_store(img, smem_u32(sm + Lay::ST_W1), Lay::OUT);
        }
        bulk_commit();
    }
    if (HALVES == 2 && !fail) {
        if (!mbar_wait(mma3_bar, 0, abort_flag, p.err, 13)) mbar_wait_drain(mma3_bar, 0);
        tc_fence_after();
        __syncthreads();
        fail = *abort_flag != 0;
        if (!fail) {
            read_wk(0, sm + Lay::KQ);                     // K slab 0 and T's first half: both dead now
            fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncthreads();
        if (!fail && tid == 0) {
            bulk_store(img, smem_u32(sm + Lay::KQ), 16384);
            bulk_commit();
        }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::TMEM_COLS);
    }
    if (tid == 0) bulk_wait_read0();                      // the shared sources stay until they are read
}

// ---------------------------------------------------------------- state --
enum Bar {
    GB_FULL = 0, GB_FREE = 2, K_FULL = 4, Q_FULL = 6, KQ_FREE = 8,
    W_FULL = 10, W_FREE, V_FULL, V_FREE, SBF_LO, SBF_HI, Z_FULL, S_FULL, O_FULL, XO_FREE, DONE,
    DRAIN0, NBARS = DRAIN0 + 8          // one per math warp (NMATH)
};

constexpr int NMATH = 8;              // math warps 0..7
constexpr int W_PROD = 8;             // producer warp (TMA, gates, tail zeroing)
constexpr int NGATHER = 3;            // q~ warps 9..11 (q rows, possibly through the index, scaled in place)
constexpr int W_MMA = 12;             // MMA warp
constexpr int STATE_THREADS = 13 * 32;
static_assert(NMATH == 8, "one drain barrier per math warp");
constexpr float LOG2E = 1.4426950408889634f;

// Gate record of one chunk.  TMEM holds T = rho S with rho = 2^lr a running
// scalar kept in [2^-1/2, 2^1/2]: the chunk decay a = e^gamma_last is applied
// as the MMA's power-of-two accumulator scale 2^-e plus a change of rho.
constexpr int G_EGR = 0;              // e^gamma_s / rho_c   (0 past n)
constexpr int G_N = C;                // n (int bits)
constexpr int G_SCL = C + 1;          // e (int bits): T <- 2^-e T + ...; -1: the old T is dropped (a < 2^-15.5)
constexpr int G_LR = C + 2;           // lr_{c+1}

template <int D>
struct StateLayout {
    static constexpr int SLABS = D / 64;
    // [K; q~] of a chunk: per 64-column slab, the 64 key rows then the 64
    // scaled query rows (8 KB each)
    static constexpr int KQSZ = SLABS * 16384;
    static constexpr int KQ0 = 0;                             // 2 x [K; q~]
    static constexpr int VB = KQ0 + 2 * KQSZ;                 // [64 x 128] bf16: two 64-column slabs
    static constexpr int IMGB = D * 128 + IMG;                // one prep image: Wk (d_k rows x 64), then Q'
    static constexpr int WB = VB + 2 * 8192;                  // prep image
    static constexpr int STG = WB + IMGB;                     // 2 x 8 x [32 rows x 32 d_v] bf16: per-warp output staging
    static constexpr int GBB = STG + 2 * 16384;               // 2 gate records
    static constexpr int BARS = GBB + 2 * GB * 4;
    static constexpr int MISC = BARS + NBARS * 8;
    static constexpr size_t BYTES = 1024 + MISC + 16;
};

// Arrival on a math-warp hand-off counter (acquire-release, CTA scope);
// true for the warp that completes the round of NMATH arrivals.
__device__ __forceinline__ bool last_arrival(uint32_t counter) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(counter) : "memory");
    return old % NMATH == NMATH - 1;
}

// TMEM column of K-step kk (16 chunk positions) of Y (off = 0) or rho' Y
// (off = 16): math warp half hf keeps both inside its own 32 Z columns.
__device__ __forceinline__ uint32_t y_col(int kk, int off) { return 32 * (kk >> 1) + 8 * (kk & 1) + off; }

template <int D>
__global__ void __launch_bounds__(STATE_THREADS, 1)
gdn_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_o, GdnTc p) {
    using Lay = StateLayout<D>;
    constexpr int SLABS = D / 64, NDV = D / DVT, HALF = D / 2;
    // TMEM columns: T = rho S (fp32), its bf16 copy (the A operand of Z and
    // X), Z (then Y and rho' Y, bf16, each math warp over the Z columns it
    // has read), X (then X + O)
    constexpr uint32_t T_S = 0, T_SB = D, T_ZU = D + D / 2, T_XO = T_ZU + 64;
    constexpr uint32_t TMEM_COLS = 512;
    constexpr int IMGB = Lay::IMGB;
    static_assert(T_XO + 64 <= TMEM_COLS, "TMEM budget");
    static_assert(Lay::BYTES <= 232448, "shared memory budget");

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024_shared(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::BARS);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Lay::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    // arrival counter of the math warps' hand-off: the last warp to finish Y
    // issues the output and state-update MMAs itself
    const uint32_t cnt_y = smem_u32(tslot + 2);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    const uint32_t kq0 = smem_u32(sm + Lay::KQ0), vb = smem_u32(sm + Lay::VB);
    const uint32_t wimg = smem_u32(sm + Lay::WB), pimg = wimg + D * 128, stg0 = smem_u32(sm + Lay::STG);
    float* gbuf = reinterpret_cast<float*>(sm + Lay::GBB);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x;
    const int seg = unit / (p.H * NDV);
    const int h = (unit / NDV) % p.H;
    const int dv0 = (unit % NDV) * DVT;
    const int c_base = p.chunk_cu[seg];
    const int nc = p.chunk_cu[seg + 1] - c_base;
    const int64_t rs0 = nc > 0 ? (int64_t)p.seg_cu[seg] : 0;
    const int64_t rs1 = nc > 0 ? (int64_t)p.seg_cu[seg + 1] : 0;

    if (threadIdx.x == 0) {
        int counts[NBARS];
        for (int i = 0; i < NBARS; ++i) counts[i] = 1;
        counts[GB_FREE] = counts[GB_FREE + 1] = NMATH;
        counts[V_FREE] = counts[SBF_LO] = counts[SBF_HI] = counts[XO_FREE] = NMATH;
        counts[Q_FULL] = counts[Q_FULL + 1] = NGATHER;
        for (int i = 0; i < NBARS; ++i) mbar_init(bar(i), counts[i]);
        *abort_flag = 0;
        tslot[2] = 0;
        fence_barrier_init();
    }
    if (warp == W_MMA) {
        tmem_alloc(smem_u32(tslot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp < NMATH) {
        // ---------------------------------------------------- math warps
        // warp (qd, hf): TMEM lanes / d_v rows 32 qd .. 32 qd + 31, chunk
        // positions (and state columns) of half hf
        const int qd = warp & 3, hf = warp >> 2;
        const int i = 32 * qd + lane;                 // d_v row inside the tile
        const uint32_t lb = (uint32_t)(32 * qd) << 16;
        const int sh = 32 * hf;
        const size_t hoff = (((size_t)seg * p.H + h) * D + dv0 + i) * D;
        // initial state: rho = 1, T = h0 (or zeros) and its bf16 copy
        for (int blk = 0; blk < HALF / 64; ++blk) {
            const int col = hf * HALF + 64 * blk;
            uint32_t w0[32], w1[32], pk[32];
#pragma unroll
            for (int e = 0; e < 64; e += 4) {
                const float4 f = p.h0 ? *reinterpret_cast<const float4*>(p.h0 + hoff + col + e)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                uint32_t* w = e < 32 ? w0 : w1;
                const int ee = e & 31;
                w[ee] = __float_as_uint(f.x); w[ee + 1] = __float_as_uint(f.y);
                w[ee + 2] = __float_as_uint(f.z); w[ee + 3] = __float_as_uint(f.w);
            }
            if (nc == 0) {
                if (p.h_final) {
                    float* out = p.h_final + hoff + col;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        *reinterpret_cast<float4*>(out + e) = make_float4(__uint_as_float(w0[e]), __uint_as_float(w0[e + 1]),
                                                                          __uint_as_float(w0[e + 2]), __uint_as_float(w0[e + 3]));
                        *reinterpret_cast<float4*>(out + 32 + e) = make_float4(__uint_as_float(w1[e]), __uint_as_float(w1[e + 1]),
                                                                               __uint_as_float(w1[e + 2]), __uint_as_float(w1[e + 3]));
                    }
                }
                continue;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                pk[e] = pack_bf16(__uint_as_float(w0[2 * e]), __uint_as_float(w0[2 * e + 1]));
                pk[16 + e] = pack_bf16(__uint_as_float(w1[2 * e]), __uint_as_float(w1[2 * e + 1]));
            }
            tmem_st_x32(tmem + lb + T_S + col, w0);
            tmem_st_x32(tmem + lb + T_S + col + 32, w1);
            tmem_st_x32(tmem + lb + T_SB + col / 2, pk);
        }
        if (nc > 0) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(SBF_LO));
                mbar_arrive(bar(SBF_HI));
            }
        }
        bool issued = false;                          // this warp's lane 0 issued MMAs
        // this thread's element of V^T: V[s][i] sits in slab i / 64, 16-byte chunk (i % 64) / 8 of row s
        const uint32_t v_slab = vb + (uint32_t)(i >> 6) * 8192 + (uint32_t)(i & 7) * 2;
        const uint32_t v_chunk = (uint32_t)((i & 63) >> 3);
        for (int c = 0; c < nc; ++c) {
            const int b = c & 1;
            const float* gb = gbuf + b * GB;
            const uint32_t ph = c & 1;
            if (!mbar_wait(bar(GB_FULL + b), (c >> 1) & 1, abort_flag, p.err, 21)) break;
            const int n = __float_as_int(gb[G_N]);
            const int64_t r0 = rs0 + (int64_t)c * C;
            // ---- Y = V^T - Z~,  Z~ = (T K^T) diag(e^gamma / rho), and rho' Y
            if (!mbar_wait(bar(V_FULL), ph, abort_flag, p.err, 22)) break;
            uint32_t vv[16];                          // V[s][i] for the 32 positions, bf16 pairs
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const int s = sh + e;
                unsigned short r0s, r1s;
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(r0s) : "r"(v_slab + s * 128 + ((v_chunk ^ (uint32_t)(s & 7)) << 4)));
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(r1s) : "r"(v_slab + (s + 1) * 128 + ((v_chunk ^ (uint32_t)((s + 1) & 7)) << 4)));
                vv[e / 2] = (uint32_t)r0s | ((uint32_t)r1s << 16);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(V_FREE));
            if (!mbar_wait(bar(Z_FULL), ph, abort_flag, p.err, 23)) break;
            tc_fence_after();
            {
                uint32_t z[32];
                tmem_ld_x32(tmem + lb + T_ZU + sh, z);
                float eg[32];
#pragma unroll
                for (int e = 0; e < 32; e += 4) ld_shared_v4(smem_u32(gb + G_EGR + sh + e), eg + e);
                const float rho1 = exp2f(gb[G_LR]);
                tmem_ld_wait();
                uint32_t py[16], pr[16];
                // positions past n hold other rows' keys and values: Y is 0 there
                // (a select, so that nothing read there can reach the products);
                // without the delta correction Y = V^T
                const float zs = p.delta ? -1.f : 0.f;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float y0 = sh + e < n
                        ? fmaf(zs * __uint_as_float(z[e]), eg[e], __uint_as_float(vv[e / 2] << 16)) : 0.f;
                    const float y1 = sh + e + 1 < n
                        ? fmaf(zs * __uint_as_float(z[e + 1]), eg[e + 1], __uint_as_float(vv[e / 2] & 0xFFFF0000u)) : 0.f;
                    py[e / 2] = pack_bf16(y0, y1);
                    pr[e / 2] = pack_bf16(rho1 * y0, rho1 * y1);
                }
                // over this warp's own Z columns, read above
                tmem_st_x16(tmem + lb + T_ZU + sh, py);
                tmem_st_x16(tmem + lb + T_ZU + sh + 16, pr);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && last_arrival(cnt_y)) {
                // T = 2^-e T + (rho' Y) Wk first (the serial chain waits for it), then
                // X += Y Q'^T; one thread issues and commits both
                constexpr uint32_t ID64 = idesc_bf16_f32(128, 64);
                constexpr uint32_t IDS = idesc_bf16_f32(128, D);     // B = Wk, K-major, N = d_k
                if (mbar_wait(bar(W_FULL), ph, abort_flag, p.err, 48)) {
                    tc_fence_after();
                    const int e = __float_as_int(gb[G_SCL]);
                    umma_f16_ts_scaled(tmem + T_S, tmem + T_ZU + y_col(0, 16), desc_kmajor_sw128(wimg), IDS,
                                       e >= 0 ? 1u : 0u, e >= 0 ? e : 0);
#pragma unroll
                    for (int kk = 1; kk < 4; ++kk)
                        umma_f16_ts(tmem + T_S, tmem + T_ZU + y_col(kk, 16), desc_kmajor_sw128(wimg + kk * 32), IDS, 1);
                    umma_commit(bar(S_FULL));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ts(tmem + T_XO, tmem + T_ZU + y_col(kk, 0), desc_kmajor_sw128(pimg + kk * 32), ID64, 1);
                    umma_commit(bar(O_FULL));
                    umma_commit(bar(W_FREE));
                    issued = true;
                }
            }
            // ---- after the state update the bf16 copy of the new T in two d_k halves
            // (the next Z | X product starts on the first); between them the output,
            // read out of TMEM (the next product overwrites X); then the output stored
            const bool last = c + 1 == nc;
            auto readback_half = [&](int part) {
                for (int blk = 0; blk < HALF / 64; ++blk) {
                    const int col = part * HALF + hf * (HALF / 2) + 32 * blk;
                    uint32_t s0[32], pk[16];
                    tmem_ld_x32(tmem + lb + T_S + col, s0);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(__uint_as_float(s0[2 * e]), __uint_as_float(s0[2 * e + 1]));
                    tmem_st_x16(tmem + lb + T_SB + col / 2, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(part ? SBF_HI : SBF_LO));
            };
            if (!mbar_wait(bar(S_FULL), ph, abort_flag, p.err, 25)) break;
            tc_fence_after();
            if (!last) readback_half(0);
            if (!mbar_wait(bar(O_FULL), ph, abort_flag, p.err, 26)) break;
            tc_fence_after();
            uint32_t xo[32];
            tmem_ld_x32(tmem + lb + T_XO + sh, xo);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(XO_FREE));
            if (!last) {
                readback_half(1);
            } else if (p.h_final) {
                // the final state S = T / rho
                const float inv = exp2f(-gb[G_LR]);
                for (int blk = 0; blk < HALF / 32; ++blk) {
                    const int col = hf * HALF + 32 * blk;
                    uint32_t sv[32];
                    tmem_ld_x32(tmem + lb + T_S + col, sv);
                    tmem_ld_wait();
                    float* out = p.h_final + hoff + col;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4*>(out + e) =
                            make_float4(inv * __uint_as_float(sv[e]), inv * __uint_as_float(sv[e + 1]),
                                        inv * __uint_as_float(sv[e + 2]), inv * __uint_as_float(sv[e + 3]));
                }
            }
            // ---- output o_r = scale (S e^gamma_r q_r + sum_s P_rs u_s), rows r < n: this
            // warp's [32 rows x 32 d_v] piece, staged row-major (two staging buffers,
            // by chunk parity), leaves by one TMA store
            {
                const uint32_t piece = stg0 + b * 16384 + warp * 2048;
                const uint32_t stg = piece + lane * 2;
                if (lane == 0) bulk_wait_read1();     // the store from two chunks ago has read this buffer
                __syncwarp();
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const uint32_t pr = pack_bf16(p.scale * __uint_as_float(xo[e]), p.scale * __uint_as_float(xo[e + 1]));
                    asm volatile("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
                                 "st.shared.b16 [%0], lo;\n\tst.shared.b16 [%1], hi;\n\t}"
                                 ::"r"(stg + e * 64), "r"(stg + (e + 1) * 64), "r"(pr) : "memory");
                }
                if (sh + 32 <= n) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tm_o, piece, h * D + dv0 + 32 * qd, (int)(r0 + sh));
                        bulk_commit();
                    }
                } else {
                    // ragged last chunk: only rows < n belong to this segment
                    bf16* orow = p.o + (r0 + sh) * (int64_t)p.H * D + (int64_t)h * D + dv0 + i;
                    const int64_t rstride = (int64_t)p.H * D;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (sh + e < n) orow[e * rstride] = __float2bfloat16_rn(p.scale * __uint_as_float(xo[e]));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(GB_FREE + b));
        }
        if (lane == 0) {
            bulk_wait0();
            // MMAs this lane issued complete before TMEM is freed (already so unless
            // the walk aborted): a commit to this warp's own barrier, whose only
            // phase completes when they have
            if (issued) {
                umma_commit(bar(DRAIN0 + warp));
                mbar_wait_drain(bar(DRAIN0 + warp), 0);
            }
        }
    } else if (warp == W_PROD) {
        // ------------------------------------------ producer: gates + loads
        // Waits only for buffers to be free, never for a copy to land (the
        // consumers wait on the copies' transaction barriers): every load is
        // issued as early as its buffer allows.  The gates of chunk c + 1 are
        // loaded while chunk c's are scanned.
        bool ok = true;
        int last_k[2] = {-1, -1}, last_w = -1, last_v = -1;
        float lr = 0.f;                               // log2 rho at the chunk start
        float bt[2], la[2];
        chunk_gates_load(p, rs0, (int)(rs1 - rs0 < C ? rs1 - rs0 : C), h, lane, bt, la);
        for (int c = 0; c < nc && ok; ++c) {
            const int b = c & 1;
            const uint32_t ph = c & 1, pb = (c >> 1) & 1;
            const int64_t r0 = rs0 + (int64_t)c * C;
            const int64_t rem = rs1 - r0;
            const int n = (int)(rem < C ? rem : C);
            const unsigned char* img = p.img + ((size_t)(c_base + c) * p.H + h) * (size_t)IMGB;
            // K tile of this chunk
            const uint32_t kb = kq0 + b * Lay::KQSZ;
            if (!mbar_wait(bar(KQ_FREE + b), pb ^ 1, abort_flag, p.err, 31)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(K_FULL + b), SLABS * 8192);
#pragma unroll
                for (int j = 0; j < SLABS; ++j) tma_load_2d(kb + j * 16384, &tm_k, bar(K_FULL + b), h * D + 64 * j, (int)r0);
            }
            last_k[b] = c;
            // gates
            if (!mbar_wait(bar(GB_FREE + b), pb ^ 1, abort_flag, p.err, 30)) { ok = false; break; }
            {
                float gg[2];
                const float gl = chunk_gates_scan(la, n, lane, gg);
                const float t = lr - gl * LOG2E;      // >= -1/2
                int e = (int)floorf(t + 0.5f);
                float lr1 = t - (float)e;
                if (e > 15) { e = -1; lr1 = 0.f; }
                float* gb = gbuf + b * GB;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int s = 2 * lane + k;
                    gb[G_EGR + s] = s < n ? exp2f(gg[k] * LOG2E - lr) : 0.f;
                }
                if (lane == 0) {
                    gb[G_N] = __int_as_float(n);
                    gb[G_SCL] = __int_as_float(e);
                    gb[G_LR] = lr1;
                }
                lr = lr1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(GB_FULL + b));
            if (c + 1 < nc) {
                const int64_t rem1 = rs1 - (r0 + C);
                chunk_gates_load(p, r0 + C, (int)(rem1 < C ? rem1 : C), h, lane, bt, la);
            }
            // V tile (this CTA's d_v rows)
            if (!mbar_wait(bar(V_FREE), ph ^ 1, abort_flag, p.err, 32)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(V_FULL), 16384);
                tma_load_2d(vb, &tm_v, bar(V_FULL), h * D + dv0, (int)r0);
                tma_load_2d(vb + 8192, &tm_v, bar(V_FULL), h * D + dv0 + 64, (int)r0);
            }
            last_v = c;
            // Wk and Q' images of this chunk
            if (!mbar_wait(bar(W_FREE), ph ^ 1, abort_flag, p.err, 36)) { ok = false; break; }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(W_FULL), IMGB);
                bulk_load(wimg, img, IMGB, bar(W_FULL));
            }
            last_w = c;
        }
        if (!ok && lane == 0) {
            // copies still in flight must land before the CTA exits
            for (int b = 0; b < 2; ++b)
                if (last_k[b] >= 0) mbar_wait_drain(bar(K_FULL + b), (last_k[b] >> 1) & 1);
            if (last_w >= 0) mbar_wait_drain(bar(W_FULL), last_w & 1);
            if (last_v >= 0) mbar_wait_drain(bar(V_FULL), last_v & 1);
        }
    } else if (warp < W_MMA) {
        // ------------------- q~ warps: q rows (through the index when given),
        // then scaled in place by e^gamma_r / rho (the output's state term)
        const int t = threadIdx.x - (W_PROD + 1) * 32;
        // the source rows of chunk c + 1 are looked up while chunk c is scaled
        GatherRows<NGATHER * 32> g;
        g.rows(p, rs0, (int)(rs1 - rs0 < C ? rs1 - rs0 : C), t);
        for (int c = 0; c < nc; ++c) {
            const int b = c & 1;
            const uint32_t pb = (c >> 1) & 1;
            const uint32_t qb = kq0 + b * Lay::KQSZ + 8192;
            const int64_t r0 = rs0 + (int64_t)c * C;
            if (!mbar_wait(bar(KQ_FREE + b), pb ^ 1, abort_flag, p.err, 38)) break;
            g.copy<D>(p, p.q, h, qb, 16384, t);
            cp_async_commit();
            if (c + 1 < nc) {
                const int64_t rem1 = rs1 - (r0 + C);
                g.rows(p, r0 + C, (int)(rem1 < C ? rem1 : C), t);
            }
            const bool gates = mbar_wait(bar(GB_FULL + b), pb, abort_flag, p.err, 39);
            cp_async_wait<0>();
            if (!gates) break;
            const float* gb = gbuf + b * GB;
            // the same (row, chunk) assignment as the gather: each thread scales what it fetched
            for (int idx = t; idx < C * 8; idx += NGATHER * 32) {
                const int row = idx >> 3, c8 = idx & 7;
                const float f = gb[G_EGR + row];
                const uint32_t d0 = qb + row * 128 + ((c8 ^ (row & 7)) << 4);
#pragma unroll
                for (int j = 0; j < SLABS; ++j) {
                    uint32_t w[4];
                    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(d0 + j * 16384));
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
                        w[e] = pack_bf16(lo * f, hi * f);
                    }
                    st_shared_v4(d0 + j * 16384, w);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Q_FULL + b));
        }
        cp_async_wait<0>();
    } else if (lane == 0) {
        // ------------------------------------------------------ MMA issuer
        // [Z | X] = T [K; q~]^T, one N = 128 product (per 64-column slab the
        // key rows then the scaled query rows); A = the bf16 copy of T in TMEM:
        // the first d_k half as soon as its copy is ready, then the second
        constexpr uint32_t ID128 = idesc_bf16_f32(128, 128);
        for (int c = 0; c < nc; ++c) {
            const int b = c & 1;
            const uint32_t ph = c & 1, pb = (c >> 1) & 1;
            const uint32_t kq = kq0 + b * Lay::KQSZ;
            if (!mbar_wait(bar(K_FULL + b), pb, abort_flag, p.err, 40)) break;
            if (!mbar_wait(bar(Q_FULL + b), pb, abort_flag, p.err, 41)) break;
            if (!mbar_wait(bar(SBF_LO), ph, abort_flag, p.err, 42)) break;
            if (!mbar_wait(bar(XO_FREE), ph ^ 1, abort_flag, p.err, 43)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
                umma_f16_ts(tmem + T_ZU, tmem + T_SB + 8 * kk, desc_kmajor_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32),
                            ID128, kk != 0);
            if (!mbar_wait(bar(SBF_HI), ph, abort_flag, p.err, 44)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = D / 32; kk < D / 16; ++kk)
                umma_f16_ts(tmem + T_ZU, tmem + T_SB + 8 * kk, desc_kmajor_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32),
                            ID128, 1);
            umma_commit(bar(Z_FULL));
            umma_commit(bar(KQ_FREE + b));
        }
        umma_commit(bar(DONE));
        mbar_wait_drain(bar(DONE), 0);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

int64_t max_chunks(int64_t n_rows, int n_seg) { return n_rows / C + n_seg; }

template <int D>
cudaError_t launch_d(const GdnTc& t, int64_t mchunks, int phase, cudaStream_t st) {
    static unsigned long long optin_prep = 0, optin_state = 0;
    cudaError_t e = smem_optin((const void*)gdn_prep_kernel<D>, (int)PrepLayout<D>::BYTES, &optin_prep);
    if (e != cudaSuccess) return e;
    e = smem_optin((const void*)gdn_state_kernel<D>, (int)StateLayout<D>::BYTES, &optin_state);
    if (e != cudaSuccess) return e;
    const int HD = t.H * D;
    CUtensorMap tm_k, tm_v, tm_q;
    if (!make_tma_2d_bf16(&tm_k, t.k, (uint64_t)t.n_rows, HD, HD, 64, C)) return cudaErrorInvalidValue;
    if (!make_tma_2d_bf16(&tm_v, t.v, (uint64_t)t.n_rows, HD, HD, 64, C)) return cudaErrorInvalidValue;
    if (!make_tma_2d_bf16(&tm_q, t.q, (uint64_t)t.n_q_rows, HD, HD, 64, C)) return cudaErrorInvalidValue;
    int launched = 0;
    if (phase & GDN_PREP) {
        gdn_schedule_kernel<<<1, 1024, 0, st>>>(t.seg_cu, t.n_seg, t.n_rows, t.chunk_cu, t.chunk_info, t.err);
        ++launched;
        if (mchunks > 0) {
            dim3 pg((unsigned)mchunks, t.H);
            gdn_prep_kernel<D><<<pg, PREP_THREADS, PrepLayout<D>::BYTES, st>>>(tm_k, tm_q, t);
            ++launched;
        }
    }
    if (phase & GDN_STATE) {
        CUtensorMap tm_o;
        if (!make_tma_2d_bf16_plain(&tm_o, t.o, (uint64_t)t.n_rows, HD, HD, 32, 32)) return cudaErrorInvalidValue;
        gdn_state_kernel<D><<<(unsigned)((int64_t)t.n_seg * t.H * (D / DVT)), STATE_THREADS, StateLayout<D>::BYTES,
                              st>>>(tm_k, tm_v, tm_o, t);
        ++launched;
    }
    count_launches(launched);
    return cudaGetLastError();
}

}  // namespace

bool gdn_tc_supported(const GdnArgs& a, int dt) {
    if (dt != MOM_BF16 || (a.d != 128 && a.d != 256)) return false;
    if (a.n_rows <= 0 || a.n_q_rows <= 0 || a.n_rows >= ((int64_t)1 << 31) / C) return false;
    return device_is_sm100() && tma_available();
}

static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t gdn_tc_ws_bytes(int64_t n_rows, int n_seg, int H, int d) {
    const size_t mc = (size_t)max_chunks(n_rows, n_seg);
    return up256(((size_t)n_seg + 1) * 4) + up256(mc * sizeof(int4)) + mc * H * ((size_t)d * 128 + IMG);
}

cudaError_t launch_gdn_tc(const GdnArgs& a, cudaStream_t st) {
    if (a.ws_bytes < MOM_WS_HEADER_BYTES + gdn_tc_ws_bytes(a.n_rows, a.n_seg, a.H, a.d)) return cudaErrorInvalidValue;
    GdnTc t;
    t.q = reinterpret_cast<const bf16*>(a.q);
    t.qidx = a.qidx;
    t.k = reinterpret_cast<const bf16*>(a.k);
    t.v = reinterpret_cast<const bf16*>(a.v);
    t.beta = a.beta;
    t.la = a.log_alpha;
    t.seg_cu = a.seg_cu;
    t.n_seg = a.n_seg;
    t.n_rows = a.n_rows;
    t.n_q_rows = a.n_q_rows;
    t.H = a.H;
    t.scale = a.scale;
    t.h0 = a.h0;
    t.h_final = a.h_final;
    t.o = reinterpret_cast<bf16*>(a.o);
    unsigned char* base = reinterpret_cast<unsigned char*>(a.ws) + MOM_WS_HEADER_BYTES;
    const int64_t mc = max_chunks(a.n_rows, a.n_seg);
    t.chunk_cu = reinterpret_cast<int32_t*>(base);
    base += up256(((size_t)a.n_seg + 1) * 4);
    t.chunk_info = reinterpret_cast<int4*>(base);
    base += up256((size_t)mc * sizeof(int4));
    t.img = base;
    t.err = a.ws;
    t.delta = a.rule == MOM_RULE_GATED_DELTA ? 1 : 0;
    t.gates_by_row = a.gates_by_row;
    return a.d == 256 ? launch_d<256>(t, mc, a.phase, st) : launch_d<128>(t, mc, a.phase, st);
}

}  // namespace mom
