// Chunked Gated DeltaNet on the tcgen05 tensor cores: bf16 operands, fp32
// state carried across chunks in TMEM.
//
// The recurrence of every memory (the authors' MoM blog post, experiments
// section: Gated DeltaNet's gate and update rule)
//   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t
// is evaluated in chunks of C = 64 rows.  With gamma_r the running sum of
// log alpha inside the chunk and S the state at the chunk start:
//   T   = (I + L)^-1,  L_rs = beta_r e^(gamma_r - gamma_s) k_r.k_s  (s < r)
//   Y^T = [beta_s (v_s - e^(gamma_s) S k_s)]_s         (d_v x C)
//   U^T = Y^T T^T                                      (u_r: the delta-rule corrections)
//   o_r = e^(gamma_r) S q_r + sum_{s<=r} e^(gamma_r-gamma_s) (q_r.k_s) u_s
//   S'  = e^(gamma_C) S + sum_s e^(gamma_C-gamma_s) u_s k_s^T
// All products are written so that the d_v rows of S are the MMA's M
// dimension (128 TMEM lanes): every MMA is M = 128.
//
// Three launches:
//   schedule: chunk offsets of every segment (device-side, no host sync)
//   prep    : per (chunk, head), independent of the state: G = [K;Q] K^T on
//             the tensor cores, then T (forward substitution, fp32) and the
//             causal decayed P = (Q K^T) o [e^(gamma_r-gamma_s)]_{s<=r}, both
//             stored as pre-swizzled bf16 64x64 tiles
//   state   : per (segment, head, 128-row d_v tile), the serial walk over the
//             segment's chunks with warp-specialised roles (producers,
//             one MMA thread, eight math warps), the state in TMEM.
// Rows past a segment's end are zero-filled on load and masked in every
// elementwise step, so a ragged tail chunk needs no padding.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mom {
namespace {

using namespace sm100;

constexpr int C = 64;                 // chunk length
constexpr int DVT = 128;              // d_v rows per state CTA (TMEM lanes)
constexpr int IMG = C * C * 2;        // one swizzled 64x64 bf16 tile
constexpr int GB = 2 * C + 4;         // beta[64], gamma[64], n, e^gamma_last, gamma_last, pad

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
    unsigned char* img;
    void* err;
};

// ------------------------------------------------------------- schedule --
__global__ void __launch_bounds__(1024)
gdn_schedule_kernel(const int32_t* __restrict__ seg_cu, int n_seg, int64_t n_rows, int32_t* __restrict__ chunk_cu,
                    void* err) {
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
}

// Gates of one chunk, computed by one full warp: beta (0 past n), the running
// sum gamma of log alpha, and e^gamma of the last valid row.  Both the prep
// and the state kernel call this, so they agree bit for bit.
__device__ __forceinline__ void chunk_gates(const GdnTc& p, int64_t r0, int n, int h, float* gb, int lane) {
    float b[2], l[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int s = 2 * lane + e;
        b[e] = 0.f;
        l[e] = 0.f;
        if (s < n) {
            const int64_t r = r0 + s;
            const int64_t qr = p.qidx ? (int64_t)p.qidx[r] : r;
            if (qr >= 0 && qr < p.n_q_rows) {
                b[e] = p.beta[qr * p.H + h];
                l[e] = p.la[qr * p.H + h];
            } else {
                record_error(p.err, MOM_DEVERR_ROW_INDEX, r);
            }
        }
    }
    const float pair = l[0] + l[1];
    float incl = pair;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    const float g0 = incl - pair + l[0], g1 = incl;
    gb[2 * lane] = b[0];
    gb[2 * lane + 1] = b[1];
    gb[C + 2 * lane] = g0;
    gb[C + 2 * lane + 1] = g1;
    const int last = n - 1;
    const float gl = __shfl_sync(0xffffffffu, (last & 1) ? g1 : g0, last >> 1);
    if (lane == 0) {
        gb[2 * C] = __int_as_float(n);
        gb[2 * C + 1] = expf(gl);
        gb[2 * C + 2] = gl;
    }
}

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
    return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// ----------------------------------------------------------------- prep --
template <int D>
constexpr size_t prep_smem() { return 1024 + (size_t)(D / 64) * 16384 + C * C * 4 + GB * 4 + 64; }

template <int D>
__global__ void __launch_bounds__(128)
gdn_prep_kernel(GdnTc p) {
    constexpr int SLABS = D / 64;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align1024(smem_raw);
    unsigned char* kq = smem;                              // slab j: K rows 0..63 | Q rows 64..127, 128 B each
    float* Lm = reinterpret_cast<float*>(smem + SLABS * 16384);
    float* gb = Lm + C * C;
    uint64_t* bar = reinterpret_cast<uint64_t*>(gb + GB);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.x, h = blockIdx.y;
    if (g >= p.chunk_cu[p.n_seg]) return;                 // uniform over the CTA
    int lo = 0, hi = p.n_seg;                              // segment s with chunk_cu[s] <= g < chunk_cu[s+1]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.chunk_cu[mid] <= g) lo = mid; else hi = mid;
    }
    const int seg = lo;
    const int64_t r0 = p.seg_cu[seg] + (int64_t)(g - p.chunk_cu[seg]) * C;
    const int64_t rem = p.seg_cu[seg + 1] - r0;
    const int n = (int)(rem < C ? rem : C);

    if (tid == 0) {
        mbar_init(smem_u32(bar), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    // K rows -> slab rows 0..63, Q rows (through qidx) -> 64..127; rows past n are zero
    {
        const int c8 = tid & 7;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int row = (tid >> 3) + 16 * i;
            const int rr = row & 63;
            const bool isq = row >= 64;
            int64_t src_row = -1;
            if (rr < n) {
                const int64_t r = r0 + rr;
                if (!isq) {
                    src_row = r;
                } else {
                    const int64_t qr = p.qidx ? (int64_t)p.qidx[r] : r;
                    src_row = (qr >= 0 && qr < p.n_q_rows) ? qr : -1;
                }
            }
            const bf16* src = (isq ? p.q : p.k) + ((src_row >= 0 ? src_row : 0) * p.H + h) * D + c8 * 8;
            const uint32_t dst = smem_u32(kq) + row * 128 + ((c8 ^ (row & 7)) << 4);
#pragma unroll
            for (int j = 0; j < SLABS; ++j) cp_async_16(dst + j * 16384, src + j * 64, src_row >= 0 ? 16u : 0u);
        }
        cp_async_commit();
    }
    if (warp == 0) chunk_gates(p, r0, n, h, gb, lane);
    if (warp == 1) {
        tmem_alloc(smem_u32(tslot), 64);
        tmem_relinquish();
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    // G = [K; Q] K^T : M = 128, N = 64, K = D
    if (tid == 0) {
        constexpr uint32_t ID = idesc_bf16_f32(128, 64);
#pragma unroll
        for (int j = 0; j < SLABS; ++j)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a = smem_u32(kq + j * 16384) + kk * 32;
                umma_f16(tmem, desc_kmajor_sw128(a), desc_kmajor_sw128(a), ID, (j | kk) != 0);
            }
        umma_commit(smem_u32(bar));
    }
    __syncwarp();
    mbar_wait(smem_u32(bar), 0, abort_flag, p.err, 10);
    tc_fence_after();
    uint32_t ga[32], gc[32];
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    tmem_ld_x32(taddr, ga);
    tmem_ld_x32(taddr + 32, gc);
    tmem_ld_wait();

    unsigned char* img = p.img + ((size_t)g * p.H + h) * 2 * IMG;
    const int r = tid & 63;
    const float gr = gb[C + r], br = gb[r];
    if (tid < 64) {
        // L row r (strictly lower, rows and columns past n are zero)
#pragma unroll
        for (int s = 0; s < C; ++s) {
            float val = 0.f;
            if (s < r && r < n) {
                const float G = __uint_as_float(s < 32 ? ga[s] : gc[s - 32]);
                val = br * expf(gr - gb[C + s]) * G;
            }
            Lm[r * C + s] = val;
        }
    } else {
        // P row r = causal, decayed q_r . k_s, bf16, swizzled image
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            uint32_t w[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                float pv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int s = c8 * 8 + e2 * 2 + e;
                    pv[e] = 0.f;
                    if (s <= r && r < n) {
                        const float G = __uint_as_float(s < 32 ? ga[s] : gc[s - 32]);
                        pv[e] = expf(gr - gb[C + s]) * G;
                    }
                }
                __nv_bfloat162 h2 = __floats2bfloat162_rn(pv[0], pv[1]);
                w[e2] = *reinterpret_cast<uint32_t*>(&h2);
            }
            *reinterpret_cast<uint4*>(img + IMG + r * 128 + ((c8 ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
    // T = (I + L)^-1 by forward substitution, one column per thread
    if (tid < 64) {
        const int j = tid;
        float t[C];
#pragma unroll
        for (int rr = 0; rr < C; ++rr) t[rr] = rr == j ? 1.f : 0.f;
#pragma unroll
        for (int rr = 1; rr < C; ++rr) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            const float* Lr = Lm + rr * C;
#pragma unroll
            for (int s = 0; s < rr; ++s) {
                const float x = Lr[s] * t[s];
                if ((s & 3) == 0) a0 += x; else if ((s & 3) == 1) a1 += x; else if ((s & 3) == 2) a2 += x; else a3 += x;
            }
            if (rr > j) t[rr] = -((a0 + a1) + (a2 + a3));
        }
#pragma unroll
        for (int rr = 0; rr < C; ++rr)
            *reinterpret_cast<bf16*>(img + sw128_offset(rr, j)) = __float2bfloat16_rn(t[rr]);
    }
}

// ---------------------------------------------------------------- state --
enum Bar {
    GB_FULL = 0, GB_FREE = 2, K_FULL = 4, K_FREE = 6,
    Q_FULL = 8, Q_FREE, V_FULL, V_FREE, T_FULL, T_FREE, P_FULL, P_FREE,
    SBF_READY, Z_FULL, X_FULL, Y_FULL, U_FULL, U_READY, S_FULL, O_FULL, XO_FREE, DONE, NBARS
};

constexpr int NMATH = 8, NPROD = 4;                  // warps
constexpr int STATE_THREADS = (NMATH + NPROD + 1) * 32;

template <int D>
struct StateLayout {
    static constexpr int SLABS = D / 64;
    static constexpr int S_BF = 0;                            // [128 x D] bf16, SLABS slabs of 16 KB
    static constexpr int K0 = S_BF + SLABS * 16384;           // 2 x [64 x D] bf16
    static constexpr int KSZ = SLABS * 8192;
    static constexpr int QB = K0 + 2 * KSZ;                   // [64 x D] bf16
    static constexpr int VB = QB + KSZ;                       // [64 x 128] bf16, plain rows of 256 B
    static constexpr int TB = VB + C * DVT * 2;               // T image
    static constexpr int PB = TB + IMG;                       // P image
    static constexpr int YB = PB + IMG;                       // [128 x 64] bf16: Y, then U^T
    static constexpr int UB = YB + 16384;                     // [128 x 64] bf16: decayed U^T
    static constexpr int GBB = UB + 16384;                    // 2 x GB floats
    static constexpr int BARS = GBB + 2 * GB * 4;
    static constexpr int MISC = BARS + NBARS * 8;
    static constexpr size_t BYTES = 1024 + MISC + 16;
};

template <int D>
__global__ void __launch_bounds__(STATE_THREADS, 1)
gdn_state_kernel(GdnTc p) {
    using Lay = StateLayout<D>;
    constexpr int SLABS = D / 64, NDV = D / DVT;
    constexpr uint32_t T_S = 0, T_ZU = D, T_X = D + 64, T_O = D + 128;
    constexpr uint32_t TMEM_COLS = 512;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::BARS);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Lay::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    auto bar = [&](int i) { return smem_u32(bars + i); };
    const uint32_t s_bf = smem_u32(sm + Lay::S_BF), kb0 = smem_u32(sm + Lay::K0), qb = smem_u32(sm + Lay::QB);
    const uint32_t timg = smem_u32(sm + Lay::TB), pimg = smem_u32(sm + Lay::PB);
    const uint32_t yb = smem_u32(sm + Lay::YB), ub = smem_u32(sm + Lay::UB);
    const bf16* vbuf = reinterpret_cast<const bf16*>(sm + Lay::VB);
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
        const int counts[NBARS] = {1, 1, NMATH, NMATH, NPROD, NPROD, 1, 1,
                                   NPROD, 1, NPROD, NMATH, 1, 1, 1, 1,
                                   NMATH, 1, 1, NMATH, 1, NMATH, 1, 1, NMATH, 1};
        for (int i = 0; i < NBARS; ++i) mbar_init(bar(i), counts[i]);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == NMATH + NPROD) {
        tmem_alloc(smem_u32(tslot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp < NMATH) {
        // ---------------------------------------------------- math warps
        const int qd = warp & 3, hf = warp >> 2;
        const int i = 32 * qd + lane;                 // d_v row inside the tile
        const uint32_t lb = (uint32_t)(32 * qd) << 16;
        constexpr int HALF = D / 2;
        bool ok = true;
        // initial state: h0 (or zeros) -> TMEM (pre-scaled by chunk 0's decay) and bf16 -> s_bf
        {
            float sc = 1.f;
            if (nc > 0) {
                ok = mbar_wait(bar(GB_FULL), 0, abort_flag, p.err, 20);
                sc = gbuf[2 * C + 1];
            }
            const float* hrow = p.h0 ? p.h0 + (((size_t)seg * p.H + h) * D + dv0 + i) * D : nullptr;
            for (int blk = 0; blk < HALF / 32 && ok; ++blk) {
                const int col = hf * HALF + 32 * blk;
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    float4 f = hrow ? *reinterpret_cast<const float4*>(hrow + col + e) : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[e] = f.x; v[e + 1] = f.y; v[e + 2] = f.z; v[e + 3] = f.w;
                }
                if (nc == 0) {
                    if (p.h_final) {
                        float* out = p.h_final + (((size_t)seg * p.H + h) * D + dv0 + i) * D + col;
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(out + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                    }
                    continue;
                }
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(v[e] * sc);
                tmem_st_x32(tmem + lb + T_S + col, w);
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[c8 * 8 + 2 * e2], v[c8 * 8 + 2 * e2 + 1]);
                        pk[e2] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    const int cc = (col & 63) / 8 + c8;
                    const uint32_t dst = s_bf + (col >> 6) * 16384 + i * 128 + ((cc ^ (i & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                                 "r"(pk[2]), "r"(pk[3]) : "memory");
                }
            }
            if (nc > 0) {
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(SBF_READY));
            }
        }
        for (int c = 0; c < nc && ok; ++c) {
            const int b = c & 1;
            const float* gb = gbuf + b * GB;
            const uint32_t ph = c & 1;
            if (!mbar_wait(bar(GB_FULL + b), (c >> 1) & 1, abort_flag, p.err, 21)) break;
            const int n = __float_as_int(gb[2 * C]);
            const int64_t r0 = rs0 + (int64_t)c * C;
            // ---- Y^T = beta_s (v_s - e^gamma_s S k_s)
            if (!mbar_wait(bar(Z_FULL), ph, abort_flag, p.err, 22)) break;
            tc_fence_after();
            uint32_t z[32];
            tmem_ld_x32(tmem + lb + T_ZU + hf * 32, z);
            tmem_ld_wait();
            if (!mbar_wait(bar(V_FULL), ph, abort_flag, p.err, 23)) break;
            {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float y[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int s = hf * 32 + e + u;
                        y[u] = 0.f;
                        if (s < n)
                            y[u] = gb[s] * (__bfloat162float(vbuf[s * DVT + i]) -
                                            expf(gb[C + s]) * __uint_as_float(z[e + u]));
                    }
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(y[0], y[1]);
                    pk[e / 2] = *reinterpret_cast<uint32_t*>(&h2);
                }
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    const int cc = hf * 4 + c8;
                    const uint32_t dst = yb + i * 128 + ((cc ^ (i & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(pk[4 * c8]),
                                 "r"(pk[4 * c8 + 1]), "r"(pk[4 * c8 + 2]), "r"(pk[4 * c8 + 3]) : "memory");
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) { mbar_arrive(bar(Y_FULL)); mbar_arrive(bar(V_FREE)); }
            // ---- U^T (for the output) and decayed U^T (for the state)
            if (!mbar_wait(bar(U_FULL), ph, abort_flag, p.err, 24)) break;
            tc_fence_after();
            uint32_t u[32];
            tmem_ld_x32(tmem + lb + T_ZU + hf * 32, u);
            tmem_ld_wait();
            {
                const float gC = gb[2 * C + 2];
                uint32_t pu[16], pd[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float a[2], dcy[2];
#pragma unroll
                    for (int w2 = 0; w2 < 2; ++w2) {
                        const int s = hf * 32 + e + w2;
                        a[w2] = 0.f;
                        dcy[w2] = 0.f;
                        if (s < n) {
                            a[w2] = __uint_as_float(u[e + w2]);
                            dcy[w2] = a[w2] * expf(gC - gb[C + s]);
                        }
                    }
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(a[0], a[1]);
                    pu[e / 2] = *reinterpret_cast<uint32_t*>(&h2);
                    __nv_bfloat162 d2 = __floats2bfloat162_rn(dcy[0], dcy[1]);
                    pd[e / 2] = *reinterpret_cast<uint32_t*>(&d2);
                }
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    const int cc = hf * 4 + c8;
                    const uint32_t off = i * 128 + ((cc ^ (i & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(yb + off), "r"(pu[4 * c8]),
                                 "r"(pu[4 * c8 + 1]), "r"(pu[4 * c8 + 2]), "r"(pu[4 * c8 + 3]) : "memory");
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(ub + off), "r"(pd[4 * c8]),
                                 "r"(pd[4 * c8 + 1]), "r"(pd[4 * c8 + 2]), "r"(pd[4 * c8 + 3]) : "memory");
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(U_READY));
            // ---- state read-back: bf16 copy for the next chunk, pre-scaled fp32 in TMEM
            if (!mbar_wait(bar(S_FULL), ph, abort_flag, p.err, 25)) break;
            tc_fence_after();
            const bool last = c + 1 == nc;
            float sc = 1.f;
            if (!last) {
                if (!mbar_wait(bar(GB_FULL + (b ^ 1)), ((c + 1) >> 1) & 1, abort_flag, p.err, 26)) break;
                sc = gbuf[(b ^ 1) * GB + 2 * C + 1];
            }
            for (int blk = 0; blk < HALF / 32; ++blk) {
                const int col = hf * HALF + 32 * blk;
                uint32_t sv[32];
                tmem_ld_x32(tmem + lb + T_S + col, sv);
                tmem_ld_wait();
                if (last) {
                    if (p.h_final) {
                        float* out = p.h_final + (((size_t)seg * p.H + h) * D + dv0 + i) * D + col;
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(out + e) =
                                make_float4(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1]),
                                            __uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]));
                    }
                    continue;
                }
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(sv[c8 * 8 + 2 * e2]),
                                                                  __uint_as_float(sv[c8 * 8 + 2 * e2 + 1]));
                        pk[e2] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    const int cc = (col & 63) / 8 + c8;
                    const uint32_t dst = s_bf + (col >> 6) * 16384 + i * 128 + ((cc ^ (i & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                                 "r"(pk[2]), "r"(pk[3]) : "memory");
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[e] = __float_as_uint(__uint_as_float(sv[e]) * sc);
                tmem_st_x32(tmem + lb + T_S + col, sv);
            }
            if (!last) {
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(SBF_READY));
            }
            // ---- output o_r = scale (e^gamma_r S q_r + sum_s P_rs u_s)
            if (!mbar_wait(bar(O_FULL), ph, abort_flag, p.err, 27)) break;
            tc_fence_after();
            uint32_t xr[32], orr[32];
            tmem_ld_x32(tmem + lb + T_X + hf * 32, xr);
            tmem_ld_x32(tmem + lb + T_O + hf * 32, orr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int r = hf * 32 + e;
                if (r < n) {
                    const float val = p.scale * fmaf(expf(gb[C + r]), __uint_as_float(xr[e]), __uint_as_float(orr[e]));
                    p.o[((r0 + r) * p.H + h) * D + dv0 + i] = __float2bfloat16_rn(val);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) { mbar_arrive(bar(XO_FREE)); mbar_arrive(bar(GB_FREE + b)); }
        }
    } else if (warp < NMATH + NPROD) {
        // ------------------------------------------------------ producers
        const int pw = warp - NMATH;
        const int pt = threadIdx.x - NMATH * 32;   // 0..127
        bool ok = true;
        int last_t = -1, last_p = -1;   // chunks whose T / P tiles were last requested
        for (int c = 0; c < nc && ok; ++c) {
            const int b = c & 1;
            const uint32_t ph = c & 1;
            const int64_t r0 = rs0 + (int64_t)c * C;
            const int64_t rem = rs1 - r0;
            const int n = (int)(rem < C ? rem : C);
            if (pw == 0) {
                if (!mbar_wait(bar(GB_FREE + b), ((c >> 1) & 1) ^ 1, abort_flag, p.err, 30)) { ok = false; break; }
                chunk_gates(p, r0, n, h, gbuf + b * GB, lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(GB_FULL + b));
            }
            const int c8 = pt & 7;
            // K rows (zero past n)
            if (!mbar_wait(bar(K_FREE + b), ((c >> 1) & 1) ^ 1, abort_flag, p.err, 31)) { ok = false; break; }
            {
                const uint32_t kb = kb0 + b * Lay::KSZ;
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const int row = (pt >> 3) + 16 * i4;
                    const bool valid = row < n;
                    const bf16* src = p.k + ((r0 + (valid ? row : 0)) * p.H + h) * D + c8 * 8;
                    const uint32_t dst = kb + row * 128 + ((c8 ^ (row & 7)) << 4);
#pragma unroll
                    for (int j = 0; j < SLABS; ++j) cp_async_16(dst + j * 8192, src + j * 64, valid ? 16u : 0u);
                }
                cp_async_commit();
            }
            // Q rows through qidx
            if (!mbar_wait(bar(Q_FREE), ph ^ 1, abort_flag, p.err, 32)) { ok = false; break; }
            {
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const int row = (pt >> 3) + 16 * i4;
                    int64_t qr = -1;
                    if (row < n) {
                        const int64_t r = r0 + row;
                        qr = p.qidx ? (int64_t)p.qidx[r] : r;
                        if (qr < 0 || qr >= p.n_q_rows) qr = -1;
                    }
                    const bf16* src = p.q + ((qr >= 0 ? qr : 0) * p.H + h) * D + c8 * 8;
                    const uint32_t dst = qb + row * 128 + ((c8 ^ (row & 7)) << 4);
#pragma unroll
                    for (int j = 0; j < SLABS; ++j) cp_async_16(dst + j * 8192, src + j * 64, qr >= 0 ? 16u : 0u);
                }
                cp_async_commit();
            }
            // V rows, this CTA's 128 d_v columns, plain layout
            if (!mbar_wait(bar(V_FREE), ph ^ 1, abort_flag, p.err, 33)) { ok = false; break; }
            {
                const int c16 = pt & 15;
                const uint32_t vb = smem_u32(vbuf);
#pragma unroll
                for (int i8 = 0; i8 < 8; ++i8) {
                    const int row = (pt >> 4) + 8 * i8;
                    const bool valid = row < n;
                    const bf16* src = p.v + ((r0 + (valid ? row : 0)) * p.H + h) * D + dv0 + c16 * 8;
                    cp_async_16(vb + row * (DVT * 2) + c16 * 16, src, valid ? 16u : 0u);
                }
                cp_async_commit();
            }
            cp_async_wait<2>();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(K_FULL + b));
            cp_async_wait<1>();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Q_FULL));
            cp_async_wait<0>();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(V_FULL));
            if (pt == 0) {
                const unsigned char* img = p.img + ((size_t)(c_base + c) * p.H + h) * 2 * IMG;
                if (!mbar_wait(bar(T_FREE), ph ^ 1, abort_flag, p.err, 34)) { ok = false; break; }
                mbar_arrive_expect_tx(bar(T_FULL), IMG);
                bulk_load(timg, img, IMG, bar(T_FULL));
                last_t = c;
                if (!mbar_wait(bar(P_FREE), ph ^ 1, abort_flag, p.err, 35)) { ok = false; break; }
                mbar_arrive_expect_tx(bar(P_FULL), IMG);
                bulk_load(pimg, img + IMG, IMG, bar(P_FULL));
                last_p = c;
            }
        }
        cp_async_wait<0>();
        if (!ok && pt == 0) {
            // bulk copies still in flight must land before the CTA exits
            if (last_t >= 0) mbar_wait_drain(bar(T_FULL), last_t & 1);
            if (last_p >= 0) mbar_wait_drain(bar(P_FULL), last_p & 1);
        }
    } else if (lane == 0) {
        // ------------------------------------------------------ MMA issuer
        constexpr uint32_t ID64 = idesc_bf16_f32(128, 64);
        constexpr uint32_t IDS = idesc_bf16_f32(128, D, 0, 1);
        for (int c = 0; c < nc; ++c) {
            const int b = c & 1;
            const uint32_t ph = c & 1;
            const uint32_t kb = kb0 + b * Lay::KSZ;
            if (!mbar_wait(bar(K_FULL + b), (c >> 1) & 1, abort_flag, p.err, 40)) break;
            if (!mbar_wait(bar(Q_FULL), ph, abort_flag, p.err, 41)) break;
            if (!mbar_wait(bar(SBF_READY), ph, abort_flag, p.err, 42)) break;
            if (!mbar_wait(bar(XO_FREE), ph ^ 1, abort_flag, p.err, 43)) break;
            tc_fence_after();
            // Z = S K^T and X = S Q^T (K = D)
#pragma unroll
            for (int j = 0; j < SLABS; ++j)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + T_ZU, desc_kmajor_sw128(s_bf + j * 16384 + kk * 32),
                             desc_kmajor_sw128(kb + j * 8192 + kk * 32), ID64, (j | kk) != 0);
            umma_commit(bar(Z_FULL));
#pragma unroll
            for (int j = 0; j < SLABS; ++j)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + T_X, desc_kmajor_sw128(s_bf + j * 16384 + kk * 32),
                             desc_kmajor_sw128(qb + j * 8192 + kk * 32), ID64, (j | kk) != 0);
            umma_commit(bar(X_FULL));
            umma_commit(bar(Q_FREE));
            // U^T = Y^T T^T (K = C)
            if (!mbar_wait(bar(Y_FULL), ph, abort_flag, p.err, 44)) break;
            if (!mbar_wait(bar(T_FULL), ph, abort_flag, p.err, 45)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + T_ZU, desc_kmajor_sw128(yb + kk * 32), desc_kmajor_sw128(timg + kk * 32), ID64,
                         kk != 0);
            umma_commit(bar(U_FULL));
            umma_commit(bar(T_FREE));
            // S += (decayed U^T) K  (B = K tile, MN-major) ; O = U^T P^T
            if (!mbar_wait(bar(U_READY), ph, abort_flag, p.err, 46)) break;
            if (!mbar_wait(bar(P_FULL), ph, abort_flag, p.err, 47)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + T_S, desc_kmajor_sw128(ub + kk * 32), desc_mnmajor_sw128(kb + kk * 2048, 8192), IDS,
                         1);
            umma_commit(bar(S_FULL));
            umma_commit(bar(K_FREE + b));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + T_O, desc_kmajor_sw128(yb + kk * 32), desc_kmajor_sw128(pimg + kk * 32), ID64,
                         kk != 0);
            umma_commit(bar(O_FULL));
            umma_commit(bar(P_FREE));
        }
        umma_commit(bar(DONE));
        mbar_wait_drain(bar(DONE), 0);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == NMATH + NPROD) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

bool device_is_sm100() {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    return major == 10;
}

int64_t max_chunks(int64_t n_rows, int n_seg) { return n_rows / C + n_seg; }

template <int D>
cudaError_t launch_d(const GdnTc& t, int64_t mchunks, cudaStream_t st) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(gdn_prep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)prep_smem<D>());
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gdn_state_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)StateLayout<D>::BYTES);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    gdn_schedule_kernel<<<1, 1024, 0, st>>>(t.seg_cu, t.n_seg, t.n_rows, t.chunk_cu, t.err);
    if (mchunks > 0) {
        dim3 pg((unsigned)mchunks, t.H);
        gdn_prep_kernel<D><<<pg, 128, prep_smem<D>(), st>>>(t);
    }
    gdn_state_kernel<D><<<(unsigned)((int64_t)t.n_seg * t.H * (D / DVT)), STATE_THREADS, StateLayout<D>::BYTES, st>>>(t);
    count_launches(mchunks > 0 ? 3 : 2);
    return cudaGetLastError();
}

}  // namespace

bool gdn_tc_supported(const GdnArgs& a, int dt) {
    if (dt != MOM_BF16 || (a.d != 128 && a.d != 256)) return false;
    if (a.n_rows >= ((int64_t)1 << 31) / C) return false;
    return device_is_sm100();
}

size_t gdn_tc_ws_bytes(int64_t n_rows, int n_seg, int H, int d) {
    (void)d;
    const size_t cu = (((size_t)n_seg + 1) * 4 + 255) & ~(size_t)255;
    return cu + (size_t)max_chunks(n_rows, n_seg) * H * 2 * IMG;
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
    t.chunk_cu = reinterpret_cast<int32_t*>(base);
    t.img = base + ((((size_t)a.n_seg + 1) * 4 + 255) & ~(size_t)255);
    t.err = a.ws;
    const int64_t mc = max_chunks(a.n_rows, a.n_seg);
    return a.d == 256 ? launch_d<256>(t, mc, st) : launch_d<128>(t, mc, st);
}

}  // namespace mom
