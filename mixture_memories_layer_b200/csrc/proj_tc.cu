// Grouped projections on the tcgen05 tensor cores (bf16 in, fp32 accumulate).
//
// ("MoM: Linear Sequence Modeling with Mixture-of-Memories", Summary: a
// shared query and each memory's own key/value projections.)  Two groups of
// problems share one persistent launch:
//   shared : every token x [W_q | W_k_sh | W_v_sh]^T      -> q, k_sh, v_sh
//   memory m: reordered rows mem_offset[m] .. mem_offset[m+1] (token
//             perm_token[r]) x [W_k^m | W_v^m]^T           -> k_p, v_p
// Output tiles are 128 rows x 256 columns; a tile never straddles two
// memories or two projections, and holds whole heads, so the per-head L2
// norm of q and k is applied in the epilogue straight from TMEM.  In the
// Gated DeltaNet block's form the outputs stay unnormalised (the short
// convolution comes first) and the shared problem has a fourth part, the
// output gate x W_g^T; the same kernel also runs one plain product
// y = x W^T (the block's output projection).
//
// Roles (416 threads, one CTA per SM, persistent over tiles):
//   warps 0-3  producers: A rows gathered with 16-byte cp.async into the
//              128-byte-swizzled K-major layout (rows come from perm_token,
//              so a tile of routed rows is a gather), each thread's arrival
//              on the stage barrier triggered by the copies' completion;
//              thread 0 also issues the TMA load of the weight tile (B,
//              K-major, 128-byte swizzle)
//   warp 12    MMA issuer: 4 x tcgen05.mma (M=128, N=256, K=16) per 64-wide
//              K step into one of two TMEM accumulators (2 x 256 columns)
//   warps 4-11 epilogue: TMEM -> registers -> (L2 norm) -> bf16 -> global,
//              two warps per TMEM lane quarter (one per column half),
//              overlapping the next tile's main loop
// Every wait is bounded (sm100.cuh); on a timeout the CTA records
// MOM_DEVERR_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mom {
namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BN * BK * 2;   // 32 KB
constexpr int NPROD = 128, NEPI = 256;     // 4 producer warps, 8 epilogue warps
constexpr int W_MMA = (NPROD + NEPI) / 32;  // MMA warp
constexpr int THREADS = NPROD + NEPI + 32;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
constexpr int STAGE_PIECE = 32 * 128;               // one warp's 32 rows x 64 columns, bf16, 128-byte swizzle
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + (size_t)(NEPI / 32) * STAGE_PIECE + 256;
constexpr uint32_t TMEM_COLS = 2 * BN;

struct TcParams {
    const bf16* x;
    const int32_t* perm;
    const int32_t* mem_offset;       // routed group offsets [n_groups + 1]
    const int32_t* group_mem;        // memory of each group (null: group g = memory g)
    bf16 *q, *k_sh, *v_sh, *k_p, *v_p, *g;
    int64_t n_tok, n_routed;
    int sh_parts, part_w;   // shared problem: parts (q, k_sh, v_sh[, g]) of part_w columns each
    int raw;                // 1: no L2 norm in the epilogue
    int D, H, d, M, K, n_groups;
    float *q_norm, *k_sh_norm, *k_p_norm;     // optional per-(row, head) lengths
    int sh_ct, rt_ct;       // column tiles per row tile (shared / routed)
    int64_t sh_tiles;       // shared tiles
    int64_t n_tiles;        // shared + an upper bound of routed tiles
    void* ws;
};

struct Tile {
    int64_t r0, r1;  // row range [r0, r1)
    int ct;          // column tile
    int m;           // memory, -1 for the shared group
};

// Tile t of the launch (identical answer in every role).  Routed tiles past
// the real count (the grid is sized by an upper bound) return false.
__device__ __forceinline__ bool tile_at(const TcParams& p, int64_t t, Tile& T) {
    if (t < p.sh_tiles) {
        const int64_t rt = t / p.sh_ct;
        T.ct = (int)(t % p.sh_ct);
        T.r0 = rt * BM;
        T.r1 = T.r0 + BM < p.n_tok ? T.r0 + BM : p.n_tok;
        T.m = -1;
        return true;
    }
    const int64_t local = t - p.sh_tiles;
    int64_t rt = local / p.rt_ct;
    T.ct = (int)(local % p.rt_ct);
    for (int g = 0; g < p.n_groups; ++g) {
        const int64_t lo = p.mem_offset[g], hi = p.mem_offset[g + 1];
        if (lo < 0 || hi < lo || hi > p.n_routed) return false;
        const int64_t nt = (hi - lo + BM - 1) / BM;
        if (rt < nt) {
            const int m = p.group_mem ? p.group_mem[g] : g;
            if (m < 0 || m >= p.M) return false;
            T.m = m;
            T.r0 = lo + rt * BM;
            T.r1 = T.r0 + BM < hi ? T.r0 + BM : hi;
            return true;
        }
        rt -= nt;
    }
    return false;
}

struct OutMaps {
    CUtensorMap q, k_sh, v_sh, k_p, v_p, g;   // [rows, columns] bf16, boxes of 32 rows x 64 columns
};

__global__ void __launch_bounds__(THREADS, 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap tm_sh, const __grid_constant__ CUtensorMap tm_kv,
               const __grid_constant__ OutMaps om, TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align1024_shared(smem_raw);
    unsigned char* sA = smem;
    unsigned char* sB = smem + STAGES * A_BYTES;
    unsigned char* sOut = sB + STAGES * B_BYTES;                       // per epilogue warp staging piece
    uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + (NEPI / 32) * STAGE_PIECE);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);


    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
    const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);
    const uint32_t done_bar = smem_u32(bars + 2 * STAGES + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, NPROD + 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull0 + 8 * a, 1);
            mbar_init(tempty0 + 8 * a, NEPI);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == W_MMA) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int KB = p.D / BK;

    if (warp < 4) {
        // ------------------------------------------------------ producers
        const int tid = threadIdx.x;
        const int c = tid & 7, rsub = tid >> 3;   // 8 lanes per 128-byte row, 16 rows per pass
        uint32_t it = 0;
        bool ok = true;
        // the next valid tile of this CTA at or after t
        auto next_tile = [&](int64_t t, Tile& T) {
            while (t < p.n_tiles && !tile_at(p, t, T)) t += gridDim.x;
            return t;
        };
        // token behind each of this thread's 8 rows (-1: zero-fill)
        auto row_tokens = [&](const Tile& T, int64_t (&tok)[8]) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t row = T.r0 + rsub + 16 * i;
                tok[i] = row < T.r1 ? ((T.m < 0 || !p.perm) ? row : (int64_t)p.perm[row]) : -1;
            }
        };
        Tile T;
        int64_t t = next_tile(blockIdx.x, T);
        int64_t tok[8];
        if (t < p.n_tiles) row_tokens(T, tok);
        while (t < p.n_tiles && ok) {
            // the next tile and its (gathered) row tokens are fetched half-way
            // through this tile, so the loads are in flight while it is issued
            Tile Tn;
            int64_t tn = p.n_tiles, ntok[8];
            const bf16* src[8];
            uint32_t nbytes[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int64_t tk = tok[i];
                if (tk >= p.n_tok || (tk < 0 && T.r0 + rsub + 16 * i < T.r1)) {
                    if (c == 0) record_error(p.ws, MOM_DEVERR_ROW_INDEX, T.r0 + rsub + 16 * i);
                    tk = -1;
                }
                src[i] = p.x + (tk >= 0 ? tk : 0) * p.D + c * 8;
                nbytes[i] = tk >= 0 ? 16u : 0u;   // rows past the tile are zero-filled
            }
            const CUtensorMap* tm = T.m < 0 ? &tm_sh : &tm_kv;
            const int wrow = (T.m < 0 ? 0 : T.m * 2 * p.H * p.d) + T.ct * BN;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                if (!mbar_wait(empty0 + 8 * s, ph ^ 1, abort_flag, p.ws, 1)) { ok = false; break; }
                if (tid == 0) {
                    mbar_arrive_expect_tx(full0 + 8 * s, B_BYTES);
                    tma_load_2d(smem_u32(sB + s * B_BYTES), tm, full0 + 8 * s, kb * BK, wrow);
                }
                const uint32_t dstA = smem_u32(sA + s * A_BYTES);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = rsub + 16 * i;
                    cp_async_16(dstA + r * 128 + ((c ^ (r & 7)) << 4), src[i] + kb * BK, nbytes[i]);
                }
                // the barrier receives this thread's arrival when its copies land
                cp_async_arrive_noinc(full0 + 8 * s);
                if (kb == KB / 2) {
                    tn = next_tile(t + gridDim.x, Tn);
                    if (tn < p.n_tiles) row_tokens(Tn, ntok);
                }
            }
            t = tn;
            T = Tn;
#pragma unroll
            for (int i = 0; i < 8; ++i) tok[i] = ntok[i];
        }
        cp_async_wait<0>();
        if (!ok && tid == 0) {
            // weight tiles still in flight must land before the CTA exits
            for (uint32_t j = it >= STAGES ? it - STAGES : 0; j < it; ++j)
                mbar_wait_drain(full0 + 8 * (j % STAGES), (j / STAGES) & 1);
        }
    } else if (warp < W_MMA) {
        // ------------------------------------------------------- epilogue
        // warp 4 + e: TMEM lanes 32 (e % 4) .. + 31, columns [128 (e / 4), + 128)
        const int e = warp - 4, qd = e & 3, hf = e >> 2;
        const int row_local = 32 * qd + lane;
        const int Hd = p.H * p.d;
        constexpr int HALF = BN / 2;
        uint32_t tc = 0;
        for (int64_t t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
            Tile T;
            if (!tile_at(p, t, T)) continue;
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            if (!mbar_wait(tfull0 + 8 * acc, aph, abort_flag, p.ws, 2)) break;
            tc_fence_after();
            const int64_t row = T.r0 + row_local;
            const bool live = row < T.r1;
            const int col0 = T.ct * BN;
            const int pw = T.m < 0 ? p.part_w : Hd;          // columns of the tile's output part
            const int part_i = col0 / pw, cc0 = col0 % pw;
            bf16* base;
            bool norm;
            float* nout;
            if (T.m < 0) {
                base = part_i == 0 ? p.q : part_i == 1 ? p.k_sh : part_i == 2 ? p.v_sh : p.g;
                norm = !p.raw && p.sh_parts >= 3 && part_i < 2;
                nout = !norm ? nullptr : part_i == 0 ? p.q_norm : p.k_sh_norm;
            } else {
                base = part_i == 0 ? p.k_p : p.v_p;
                norm = !p.raw && part_i == 0;
                nout = norm ? p.k_p_norm : nullptr;
            }
            const CUtensorMap* omap =
                T.m < 0 ? (part_i == 0 ? &om.q : part_i == 1 ? &om.k_sh : part_i == 2 ? &om.v_sh : &om.g)
                        : (part_i == 0 ? &om.k_p : &om.v_p);
            // a piece goes out by TMA only when all 32 of its rows belong to this tile
            const bool full_piece = T.r0 + 32 * qd + 32 <= T.r1;
            bf16* orow = base + (live ? row : 0) * (int64_t)pw + cc0 + hf * HALF;
            const uint32_t taddr = tmem_base + ((uint32_t)(32 * qd) << 16) + acc * BN + hf * HALF;
            const uint32_t piece = smem_u32(sOut + e * STAGE_PIECE);
            const int gw = p.d < HALF ? p.d : HALF;          // head-group width inside this half
            float sc_full = 1.f;
            if (norm && p.d > HALF) {
                // a head spans both halves: each thread sums the whole row (TMEM reads are cheap)
                float ss = 0.f;
                uint32_t r[32];
                const uint32_t trow = taddr - hf * HALF;
                for (int cc = 0; cc < BN; cc += 32) {
                    tmem_ld_x32(trow + cc, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ss);
                }
                sc_full = rsqrtf(ss + 1e-6f);
                if (nout && live && hf == 0) nout[row * p.H + cc0 / p.d] = sqrtf(ss + 1e-6f);
            }
            float scg[HALF / 64 * 2];                        // per 32-column block scale
#pragma unroll
            for (int j = 0; j < HALF / 32; ++j) scg[j] = sc_full;
            if (norm && p.d <= HALF) {
                for (int g = 0; g < HALF; g += gw) {
                    float ss = 0.f;
                    uint32_t r[32];
                    for (int cc = 0; cc < gw; cc += 32) {
                        tmem_ld_x32(taddr + g + cc, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ss);
                    }
                    const float sc = rsqrtf(ss + 1e-6f);
                    if (nout && live) nout[row * p.H + (cc0 + hf * HALF + g) / p.d] = sqrtf(ss + 1e-6f);
#pragma unroll
                    for (int j = 0; j < HALF / 32; ++j)
                        if (j * 32 >= g && j * 32 < g + gw) scg[j] = sc;
                }
            }
            // 64-column pieces: registers -> swizzled staging -> TMA store
#pragma unroll
            for (int pc = 0; pc < HALF / 64; ++pc) {
                if (lane == 0) bulk_wait_read0();            // the previous piece has left shared memory
                __syncwarp();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int j = pc * 2 + hh;
                    uint32_t r[32];
                    tmem_ld_x32(taddr + 32 * j, r);
                    tmem_ld_wait();
                    const float sc = scg[j];
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[2 * i]) * sc,
                                                                  __uint_as_float(r[2 * i + 1]) * sc);
                        w[i] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    if (full_piece) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            const int ch = hh * 4 + c4;
                            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};"
                                         ::"r"(piece + lane * 128 + ((ch ^ (lane & 7)) << 4)),
                                           "r"(w[4 * c4]), "r"(w[4 * c4 + 1]), "r"(w[4 * c4 + 2]), "r"(w[4 * c4 + 3])
                                         : "memory");
                        }
                    } else if (live) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * j);
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) dst[c4] = make_uint4(w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
                    }
                }
                if (full_piece) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(omap, piece, cc0 + hf * HALF + 64 * pc, (int)(T.r0 + 32 * qd));
                        bulk_commit();
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tempty0 + 8 * acc);
            ++tc;
        }
        if (lane == 0) bulk_wait0();
    } else if (lane == 0) {
        // ------------------------------------------------------ MMA issuer
        uint32_t it = 0, tc = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x) {
            Tile T;
            if (!tile_at(p, t, T)) continue;
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1, abort_flag, p.ws, 3)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * BN;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                if (!mbar_wait(full0 + 8 * s, ph, abort_flag, p.ws, 4)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a0 = smem_u32(sA + s * A_BYTES), b0 = smem_u32(sB + s * B_BYTES);
#pragma unroll
                for (int j = 0; j < BK / 16; ++j)
                    umma_f16(d_tmem, desc_kmajor_sw128(a0 + 32 * j), desc_kmajor_sw128(b0 + 32 * j), IDESC,
                             (kb | j) != 0);
                umma_commit(empty0 + 8 * s);
            }
            if (!ok) break;
            umma_commit(tfull0 + 8 * acc);
            ++tc;
        }
        // every MMA this CTA issued has finished before TMEM is released
        umma_commit(done_bar);
        mbar_wait_drain(done_bar, 0);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace

bool proj_tc_supported(const ProjArgs& a, int dt) {
    if (dt != MOM_BF16 || a.n_tok <= 0) return false;
    if (a.plain_n > 0 ? a.plain_n % BN != 0 : (a.H * a.d) % BN != 0) return false;
    if (a.D % BK != 0) return false;
    return device_is_sm100() && tma_available();
}

cudaError_t launch_proj_tc(const ProjArgs& a, cudaStream_t st) {
    const int Hd = a.H * a.d;
    const bool plain = a.plain_n > 0;
    const bool sh = a.parts & PROJ_SHARED, rt = !plain && (a.parts & PROJ_ROUTED) && a.routed_rows() > 0;
    if (!sh && !rt) return cudaSuccess;
    const int sh_parts = plain ? 1 : a.g ? 4 : 3, part_w = plain ? a.plain_n : Hd;
    // maps of a problem that does not run are copies of one that does (never used)
    CUtensorMap tm_sh, tm_kv;
    if (sh && !make_tma_2d_bf16(&tm_sh, a.w_shared, (uint64_t)sh_parts * part_w, a.D, a.D, 64, BN))
        return cudaErrorInvalidValue;
    if (rt && !make_tma_2d_bf16(&tm_kv, a.w_kv, (uint64_t)a.M * 2 * Hd, a.D, a.D, 64, BN)) return cudaErrorInvalidValue;
    if (!sh) tm_sh = tm_kv;
    if (!rt) tm_kv = tm_sh;
    OutMaps om;
    const uint64_t nrp = (uint64_t)a.routed_rows();
    if (sh && !make_tma_2d_bf16(&om.q, a.q, a.n_tok, part_w, part_w, 64, 32)) return cudaErrorInvalidValue;
    if (sh && !plain && (!make_tma_2d_bf16(&om.k_sh, a.k_sh, a.n_tok, Hd, Hd, 64, 32) ||
                         !make_tma_2d_bf16(&om.v_sh, a.v_sh, a.n_tok, Hd, Hd, 64, 32)))
        return cudaErrorInvalidValue;
    if (sh && a.g && !plain && !make_tma_2d_bf16(&om.g, a.g, a.n_tok, Hd, Hd, 64, 32)) return cudaErrorInvalidValue;
    if (sh && plain) om.k_sh = om.v_sh = om.q;
    if (rt && (!make_tma_2d_bf16(&om.k_p, a.k_p, nrp, Hd, Hd, 64, 32) || !make_tma_2d_bf16(&om.v_p, a.v_p, nrp, Hd, Hd, 64, 32)))
        return cudaErrorInvalidValue;
    if (!sh) om.q = om.k_sh = om.v_sh = om.k_p;
    if (!rt) om.k_p = om.v_p = om.q;
    if (!(sh && a.g && !plain)) om.g = om.q;
    TcParams p;
    p.x = reinterpret_cast<const bf16*>(a.x);
    p.perm = a.perm_token;
    p.mem_offset = a.mem_offset;
    p.group_mem = a.group_mem;
    p.q_norm = a.q_norm;
    p.k_sh_norm = a.k_sh_norm;
    p.k_p_norm = a.k_p_norm;
    p.q = reinterpret_cast<bf16*>(a.q);
    p.k_sh = reinterpret_cast<bf16*>(a.k_sh);
    p.v_sh = reinterpret_cast<bf16*>(a.v_sh);
    p.k_p = reinterpret_cast<bf16*>(a.k_p);
    p.v_p = reinterpret_cast<bf16*>(a.v_p);
    p.g = reinterpret_cast<bf16*>(a.g);
    p.sh_parts = sh_parts;
    p.part_w = part_w;
    p.raw = a.raw || plain;
    p.n_tok = a.n_tok;
    p.n_routed = nrp;
    p.n_groups = a.groups();
    p.D = a.D; p.H = a.H; p.d = a.d; p.M = a.M; p.K = a.K;
    p.sh_ct = sh_parts * part_w / BN;
    p.rt_ct = 2 * Hd / BN;
    p.sh_tiles = sh ? cdiv(a.n_tok, BM) * p.sh_ct : 0;
    p.n_tiles = p.sh_tiles + (rt ? (cdiv((int64_t)nrp, BM) + p.n_groups) * p.rt_ct : 0);
    p.ws = a.ws;

    static unsigned long long optin_done = 0;
    cudaError_t e = smem_optin((const void*)proj_tc_kernel, (int)SMEM_BYTES, &optin_done);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = p.n_tiles < sms ? p.n_tiles : sms;
    proj_tc_kernel<<<(unsigned)grid, THREADS, SMEM_BYTES, st>>>(tm_sh, tm_kv, om, p);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
