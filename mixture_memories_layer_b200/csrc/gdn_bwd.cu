// Reverse pass of a memory's recurrence over each segment, for both update
// rules (the first GPU path of the layer's backward: training is the pages'
// main workload, "MoM: Linear Sequence Modeling with Mixture-of-Memories",
// Key points; the rules: the authors' MoM blog post, experiments section and
// "Linear Recurrent Memory").  Token-serial, fp32, on CUDA cores.
//
// Forward, with a = e^(log alpha_t), b = beta_t, c = 1 (Gated DeltaNet) or 0
// (scalar-gated linear), row i of the state evolving on its own:
//   y_i = S_i . k,  u_i = b (v_i - c a y_i),  S_i <- a S_i + u_i k,  o_i = scale S_i . q
// Reverse, with G_i the adjoint of row i after token t (plus do_i scale q):
//   dq   += scale S_i(t) do_i            dv_i = b (G_i . k)
//   dbeta += (v_i - c a y_i)(G_i . k)     dalpha += G_i . S_i(t-1) - c b y_i (G_i . k)
//   dk   += u_i G_i - c a b (G_i . k) S_i(t-1)
//   G_i  <- a G_i - c a b (G_i . k) k
// (sums over the rows i; dlog_alpha = a dalpha).
//
// One CTA owns 32 state rows of one (segment, head): 8 warps of 4 rows, a
// lane holding d/32 columns of each, as in the token-serial forward; two
// CTAs share an SM, so two token-serial chains interleave there.  The
// reverse pass needs S(t-1) at every token: a forward sweep stores the rows
// every 16 tokens; the chunks are then walked backwards, each recomputed from
// its stored state with a copy kept every 2 tokens, and the state before a
// token is rebuilt from the nearest copy (at most 1 step).  The copies of
// the chunks in flight stay in L2 (8 per CTA: 256 KB; with 64-token chunks
// the ~300 resident CTAs' copies overflowed it and every rebuild waited on
// HBM).  The kernel is
// bound by instruction issue, the warp shuffles of the per-row dot products
// first: the 4 rows of a warp are summed together by a reduce-scatter and
// gather (9 shuffles, not 20).  The operands of
// each 16-token block (k, q, the CTA's v and d_o, the gates) are loaded once
// by the whole CTA into shared memory, so the replayed steps never wait on
// L2.  The sums over
// rows are reduced inside the CTA per token and written as one partial per
// 32-row tile, which a second kernel adds up (deterministic, no atomics).
#include "common.cuh"
#include "kernels.h"

namespace mom {
namespace {

constexpr int BR = 4;               // state rows per warp
static_assert(BR == 4, "warp_allreduce4 sums the 4 rows of a warp");
constexpr int BW = 8;               // warps per CTA (two CTAs fit an SM: two chains interleave)
constexpr int ROWS = BR * BW;       // state rows per CTA
constexpr int CK = 16;              // tokens between stored states (a chunk: one operand block)
constexpr int SUB = 2;              // tokens between the copies kept inside a chunk
constexpr int NSUB = CK / SUB;
constexpr int CACHE = 16;           // tokens whose operands one fill brings into shared memory
static_assert(CK % CACHE == 0 && CACHE % SUB == 0, "stored states and copies on operand-block bounds");

struct BwdTables {
    int32_t* chunk_cu;   // [n_seg + 1] first stored state of each segment
    float* ckpt;         // [max_chunks][H][tiles][ROWS][D]
    float* sub;          // [n_seg * tiles * H][NSUB][ROWS][D]
    float* part;         // [tiles][n_rows][H][2D + 2]: dq | dk | dlog_alpha | dbeta
};

// The sums over a warp of 4 values per lane, in every lane: a reduce-scatter
// (each lane pair halves its set of values, twice), the last value summed
// over the remaining 8 lanes, then the 4 totals gathered back -- 9 shuffles
// where four independent butterflies take 20.
__device__ __forceinline__ void warp_allreduce4(float* v) {
    const int lane = threadIdx.x & 31;
    const bool hi = lane & 16, hb = lane & 8;
    const float r0 = __shfl_xor_sync(0xffffffffu, hi ? v[0] : v[2], 16);
    const float r1 = __shfl_xor_sync(0xffffffffu, hi ? v[1] : v[3], 16);
    const float k0 = (hi ? v[2] : v[0]) + r0, k1 = (hi ? v[3] : v[1]) + r1;   // values base, base+1
    float x = (hb ? k1 : k0) + __shfl_xor_sync(0xffffffffu, hb ? k0 : k1, 8); // value base + hb
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    const float o = __shfl_xor_sync(0xffffffffu, x, 8);
    const float t0 = hb ? o : x, t1 = hb ? x : o;                            // totals base, base+1
    const float u0 = __shfl_xor_sync(0xffffffffu, t0, 16), u1 = __shfl_xor_sync(0xffffffffu, t1, 16);
    v[0] = hi ? u0 : t0;
    v[1] = hi ? u1 : t1;
    v[2] = hi ? t0 : u0;
    v[3] = hi ? t1 : u1;
}

__global__ void bwd_schedule_kernel(const int32_t* __restrict__ seg_cu, int n_seg, int64_t n_rows,
                                    int32_t* __restrict__ chunk_cu, void* err) {
    if (threadIdx.x != 0) return;
    int64_t acc = 0;
    for (int s = 0; s < n_seg; ++s) {
        chunk_cu[s] = (int32_t)acc;
        const int64_t a = seg_cu[s], b = seg_cu[s + 1];
        if (a < 0 || b < a || b > n_rows) { record_error(err, MOM_DEVERR_SEGMENT, s); continue; }
        acc += (b - a + CK - 1) / CK;
    }
    chunk_cu[n_seg] = (int32_t)acc;
}

template <int D>
struct BwdSmem {
    static constexpr int PW = 2 * D + 2;                      // partial width: dq | dk | dlog_alpha | dbeta
    static constexpr int RED = 0;                             // [2][BW][PW] per-warp sums over rows (two tokens)
    static constexpr int KC = RED + 2 * BW * PW;              // [CACHE][D] k of the cached tokens
    static constexpr int QC = KC + CACHE * D;                 // [CACHE][D] q
    static constexpr int VC = QC + CACHE * D;                 // [CACHE][ROWS] v of this CTA's rows
    static constexpr int DC = VC + CACHE * ROWS;              // [CACHE][ROWS] d_o
    static constexpr int BC = DC + CACHE * ROWS;              // [CACHE] beta
    static constexpr int AC = BC + CACHE;                     // [CACHE] alpha
    static constexpr int OKC = AC + CACHE;                    // [CACHE] 1: the token's row index is valid
    static constexpr int FLOATS = OKC + CACHE;
    static constexpr size_t BYTES = (size_t)FLOATS * 4;
};

template <typename T, int D>
__global__ void __launch_bounds__(BW * 32, 2)
gdn_bwd_kernel(GdnBwdArgs a, BwdTables tb) {
    using SM = BwdSmem<D>;
    constexpr int E = D / 32;
    constexpr int TILES = D / ROWS;
    constexpr int PW = SM::PW;
    constexpr int NT = BW * 32;
    extern __shared__ float smf[];
    float* red = smf + SM::RED;
    float* kc = smf + SM::KC;
    float* qc = smf + SM::QC;
    float* vc = smf + SM::VC;
    float* dc = smf + SM::DC;
    float* bc = smf + SM::BC;
    float* ac = smf + SM::AC;
    float* okc = smf + SM::OKC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = blockIdx.x / TILES, tile = blockIdx.x % TILES, h = blockIdx.y, H = a.H;
    const int rowt = warp * BR;                  // this warp's first row inside the tile
    const int row0 = tile * ROWS + rowt;         // ... and inside the head
    const T* q = reinterpret_cast<const T*>(a.q);
    const T* k = reinterpret_cast<const T*>(a.k);
    const T* v = reinterpret_cast<const T*>(a.v);
    const T* dout = reinterpret_cast<const T*>(a.d_o);
    const bool delta = a.rule == MOM_RULE_GATED_DELTA;

    int64_t r0 = a.seg_cu[seg], r1 = a.seg_cu[seg + 1];
    if (r0 < 0 || r1 < r0 || r1 > a.n_rows) r1 = r0;       // recorded by the schedule
    const int64_t nck = (r1 - r0 + CK - 1) / CK;
    const size_t ck_stride = (size_t)H * TILES * ROWS * D;
    float* ck = tb.ckpt + ((size_t)tb.chunk_cu[seg] * H * TILES + (size_t)h * TILES + tile) * ROWS * D +
                (size_t)rowt * D + lane * E;
    float* sub = tb.sub + ((size_t)blockIdx.y * gridDim.x + blockIdx.x) * NSUB * ROWS * D + (size_t)rowt * D + lane * E;

    // the operands of tokens ts .. ts+n-1 (n <= CACHE) into shared memory, by
    // the whole CTA (every replay and reverse step then reads them from there)
    auto fill = [&](int64_t ts, int n, bool want_do) {
        __syncthreads();                                      // the previous block's readers are done
        if (threadIdx.x < n) {
            const int64_t r = ts + threadIdx.x;
            const int64_t qr = a.qidx ? (int64_t)a.qidx[r] : r;
            const bool ok = qr >= 0 && qr < a.n_q_rows;
            if (!ok && tile == 0) record_error(a.ws, MOM_DEVERR_ROW_INDEX, r);
            const int64_t gr = a.gates_by_row ? r : qr;
            okc[threadIdx.x] = ok ? 1.f : 0.f;
            bc[threadIdx.x] = ok ? a.beta[gr * H + h] : 0.f;
            ac[threadIdx.x] = ok ? expf(a.log_alpha[gr * H + h]) : 1.f;
        }
        // k and q rows in pieces of 8 values (one 16-byte load of bf16):
        // a thread's k and q pieces loaded together, then stored (the state
        // and its adjoint stay in registers meanwhile, so one pair at a time)
        constexpr int PR = D / 8;                             // pieces per row
        constexpr int ITK = (CACHE * PR + NT - 1) / NT;
#pragma unroll
        for (int it = 0; it < ITK; ++it) {
            const int i = threadIdx.x + it * NT, j = i / PR, c = (i % PR) * 8;
            if (j < n) {
                const int64_t r = ts + j;
                const int64_t qr = a.qidx ? (int64_t)a.qidx[r] : r;
                float kv[8], qv[8];
                load_vec<8>(k + (r * H + h) * D + c, kv);
                if (qr >= 0 && qr < a.n_q_rows) load_vec<8>(q + (qr * H + h) * D + c, qv);
                else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) qv[e] = 0.f;
                }
                store_vec<8>(kc + j * D + c, kv);
                store_vec<8>(qc + j * D + c, qv);
            }
        }
        // this CTA's rows of v (and d_o): threads 0 .. VP-1 and VP .. 2 VP-1
        constexpr int VP = CACHE * ROWS / 8;
        static_assert(2 * VP <= NT, "one piece of v or d_o per thread");
        const int which = threadIdx.x / VP, i = threadIdx.x % VP, j = i / (ROWS / 8), c = (i % (ROWS / 8)) * 8;
        if (which < 2 && j < n && (which == 0 || want_do)) {
            const int64_t off = ((ts + j) * H + h) * D + tile * ROWS + c;
            float vv[8];
            load_vec<8>((which == 0 ? v : dout) + off, vv);
            store_vec<8>((which == 0 ? vc : dc) + j * ROWS + c, vv);
        }
        __syncthreads();
    };

    // S <- one forward step at cached token j (S holds the state before it)
    float S[BR][E];
    auto step = [&](int j) {
        if (okc[j] == 0.f) return;
        float kk[E];
        load_vec<E>(kc + j * D + lane * E, kk);
        const float b = bc[j], al = ac[j];
        float y[BR];
#pragma unroll
        for (int i = 0; i < BR; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) acc = fmaf(S[i][e], kk[e], acc);
            y[i] = acc;
        }
        warp_allreduce4(y);
        const float dl = delta ? al : 0.f;
#pragma unroll
        for (int i = 0; i < BR; ++i) {
            const float u = b * (vc[j * ROWS + rowt + i] - dl * y[i]);
#pragma unroll
            for (int e = 0; e < E; ++e) S[i][e] = fmaf(al, S[i][e], u * kk[e]);
        }
    };

    // ---- forward sweep: the rows every CK tokens
    const size_t hoff = (((size_t)seg * H + h) * D + row0) * D + lane * E;
#pragma unroll
    for (int i = 0; i < BR; ++i) {
        if (a.h0) load_vec<E>(a.h0 + hoff + (size_t)i * D, S[i]);
        else {
#pragma unroll
            for (int e = 0; e < E; ++e) S[i][e] = 0.f;
        }
    }
    for (int64_t ts = r0; ts < r1; ts += CACHE) {
        const int n = (int)(r1 - ts < CACHE ? r1 - ts : CACHE);
        fill(ts, n, false);
        if ((ts - r0) % CK == 0) {
#pragma unroll
            for (int i = 0; i < BR; ++i) store_vec<E>(ck + (size_t)((ts - r0) / CK) * ck_stride + (size_t)i * D, S[i]);
        }
        for (int j = 0; j < n; ++j) step(j);
    }

    // ---- reverse sweep
    float G[BR][E];
#pragma unroll
    for (int i = 0; i < BR; ++i) {
        if (a.dh_final) load_vec<E>(a.dh_final + hoff + (size_t)i * D, G[i]);
        else {
#pragma unroll
            for (int e = 0; e < E; ++e) G[i][e] = 0.f;
        }
    }
    // the per-warp sums of consecutive tokens alternate between two buffers:
    // a buffer is written again two tokens later, after every thread that
    // read it has passed the next token's barrier, so one barrier per token
    // suffices
    int par = 0;
    for (int64_t jc = nck - 1; jc >= 0; --jc) {
        const int64_t t0 = r0 + jc * CK, t1 = t0 + CK < r1 ? t0 + CK : r1;
#pragma unroll
        for (int i = 0; i < BR; ++i) load_vec<E>(ck + (size_t)jc * ck_stride + (size_t)i * D, S[i]);
        // a chunk of one operand block: the re-walk's fill (with d_o) serves the reverse too
        const int ncb = (int)((t1 - t0 + CACHE - 1) / CACHE);
        for (int64_t tc = t0; tc < t1; tc += CACHE) {
            const int n = (int)(t1 - tc < CACHE ? t1 - tc : CACHE);
            fill(tc, n, ncb == 1);
            for (int j = 0; j < n; ++j) {
                if (j % SUB == 0) {
#pragma unroll
                    for (int i = 0; i < BR; ++i)
                        store_vec<E>(sub + (size_t)((tc + j - t0) / SUB) * ROWS * D + (size_t)i * D, S[i]);
                }
                step(j);
            }
        }
        for (int cb = ncb - 1; cb >= 0; --cb) {
            const int64_t tc = t0 + (int64_t)cb * CACHE;
            const int n = (int)(t1 - tc < CACHE ? t1 - tc : CACHE);
            if (ncb > 1) fill(tc, n, true);
            for (int jt = n - 1; jt >= 0; --jt) {
                const int64_t t = tc + jt;
                // S(t-1): the nearest kept copy, then forward to t
                const int js = jt - jt % SUB;
#pragma unroll
                for (int i = 0; i < BR; ++i)
                    load_vec<E>(sub + (size_t)((tc + js - t0) / SUB) * ROWS * D + (size_t)i * D, S[i]);
                for (int j = js; j < jt; ++j) step(j);
                // the token's own reverse step
                float* w = red + (par * BW + warp) * PW;
                if (okc[jt] != 0.f) {
                    float kk[E], qq[E];
                    load_vec<E>(kc + jt * D + lane * E, kk);
                    load_vec<E>(qc + jt * D + lane * E, qq);
                    const float b = bc[jt], al = ac[jt];
                    const float dl = delta ? al : 0.f, cab = delta ? al * b : 0.f;
                    float y[BR], vv[BR];
#pragma unroll
                    for (int i = 0; i < BR; ++i) {
                        vv[i] = vc[jt * ROWS + rowt + i];
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < E; ++e) acc = fmaf(S[i][e], kk[e], acc);
                        y[i] = acc;
                    }
                    warp_allreduce4(y);
                    float u[BR], dq[E], dk[E];
#pragma unroll
                    for (int e = 0; e < E; ++e) { dq[e] = 0.f; dk[e] = 0.f; }
                    float gkv[BR], gsum = 0.f;            // G.k per row; G.S(t-1) summed over the rows
#pragma unroll
                    for (int i = 0; i < BR; ++i) {
                        u[i] = b * (vv[i] - dl * y[i]);
                        const float sq = dc[jt * ROWS + rowt + i] * a.scale;
                        float gk = 0.f, gs = 0.f;
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            G[i][e] = fmaf(sq, qq[e], G[i][e]);
                            const float st = fmaf(al, S[i][e], u[i] * kk[e]);     // S(t)
                            dq[e] = fmaf(sq, st, dq[e]);
                            gk = fmaf(G[i][e], kk[e], gk);
                            gs = fmaf(G[i][e], S[i][e], gs);
                        }
                        gkv[i] = gk;
                        gsum += gs;
                    }
                    warp_allreduce4(gkv);
                    warp_sum_n<1>(&gsum);
                    float dalpha = gsum, dbeta = 0.f;
#pragma unroll
                    for (int i = 0; i < BR; ++i) {
                        const float gk = gkv[i];
                        dbeta += (vv[i] - dl * y[i]) * gk;
                        dalpha -= delta ? b * y[i] * gk : 0.f;
                        if (lane == i) a.dv[(t * H + h) * D + row0 + i] = b * gk;
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            dk[e] = fmaf(u[i], G[i][e], dk[e]) - cab * gk * S[i][e];
                            G[i][e] = al * G[i][e] - cab * gk * kk[e];
                        }
                    }
#pragma unroll
                    for (int e = 0; e < E; ++e) { w[lane * E + e] = dq[e]; w[D + lane * E + e] = dk[e]; }
                    if (lane == 0) { w[2 * D] = al * dalpha; w[2 * D + 1] = dbeta; }
                } else {
                    for (int c = lane; c < PW; c += 32) w[c] = 0.f;
                }
                __syncthreads();
                float* pout = tb.part + (((size_t)tile * a.n_rows + t) * H + h) * PW;
                const float* rb = red + par * BW * PW;
                for (int c = threadIdx.x; c < PW; c += NT) {
                    float acc = 0.f;
#pragma unroll
                    for (int ww = 0; ww < BW; ++ww) acc += rb[ww * PW + c];
                    pout[c] = acc;
                }
                par ^= 1;
            }
        }
    }
    if (a.dh0) {
#pragma unroll
        for (int i = 0; i < BR; ++i) store_vec<E>(a.dh0 + hoff + (size_t)i * D, G[i]);
    }
}

// Adds the per-tile partials of every row inside the segments.
template <int D>
__global__ void __launch_bounds__(256)
bwd_reduce_kernel(GdnBwdArgs a, BwdTables tb) {
    constexpr int TILES = D / ROWS, PW = 2 * D + 2;
    const int64_t lo = a.seg_cu[0], hi = a.seg_cu[a.n_seg];
    if (lo < 0 || hi < lo || hi > a.n_rows) return;
    const int64_t total = (hi - lo) * a.H * PW;
    const size_t tile_stride = (size_t)a.n_rows * a.H * PW;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t rh = i / PW, c = i - rh * PW;
        const int64_t r = lo + rh / a.H, h = rh % a.H;
        const size_t off = ((size_t)r * a.H + h) * PW + c;
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < TILES; ++t) acc += tb.part[t * tile_stride + off];
        if (c < D) a.dq[((size_t)r * a.H + h) * D + c] = acc;
        else if (c < 2 * D) a.dk[((size_t)r * a.H + h) * D + (c - D)] = acc;
        else if (c == 2 * D) a.dlog_alpha[(size_t)r * a.H + h] = acc;
        else a.dbeta[(size_t)r * a.H + h] = acc;
    }
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdLayout {
    size_t chunk_cu, ckpt, sub, part, total;
};

BwdLayout bwd_layout(int64_t n_rows, int n_seg, int H, int d) {
    BwdLayout L;
    const int tiles = d / ROWS;
    const size_t max_chunks = (size_t)(n_rows / CK) + (size_t)n_seg;
    size_t off = MOM_WS_HEADER_BYTES;
    auto take = [&](size_t bytes) { size_t o = off; off += up256(bytes); return o; };
    L.chunk_cu = take(((size_t)n_seg + 1) * 4);
    L.ckpt = take(max_chunks * H * tiles * ROWS * (size_t)d * 4);
    L.sub = take((size_t)n_seg * tiles * H * NSUB * ROWS * (size_t)d * 4);
    L.part = take((size_t)tiles * n_rows * H * (2 * (size_t)d + 2) * 4);
    L.total = off;
    return L;
}

template <typename T, int D>
cudaError_t launch_bwd_t(const GdnBwdArgs& a, cudaStream_t st) {
    const BwdLayout L = bwd_layout(a.n_rows, a.n_seg, a.H, a.d);
    unsigned char* base = reinterpret_cast<unsigned char*>(a.ws);
    BwdTables tb{reinterpret_cast<int32_t*>(base + L.chunk_cu), reinterpret_cast<float*>(base + L.ckpt),
                 reinterpret_cast<float*>(base + L.sub), reinterpret_cast<float*>(base + L.part)};
    static unsigned long long optin_done = 0;
    cudaError_t e = smem_optin((const void*)gdn_bwd_kernel<T, D>, (int)BwdSmem<D>::BYTES, &optin_done);
    if (e != cudaSuccess) return e;
    bwd_schedule_kernel<<<1, 32, 0, st>>>(a.seg_cu, a.n_seg, a.n_rows, tb.chunk_cu, a.ws);
    dim3 grid((unsigned)a.n_seg * (D / ROWS), a.H);
    gdn_bwd_kernel<T, D><<<grid, BW * 32, BwdSmem<D>::BYTES, st>>>(a, tb);
    const int64_t work = a.n_rows * a.H * (2 * D + 2);
    const int64_t want = cdiv(work, 256);
    bwd_reduce_kernel<D><<<(unsigned)(want < 148 * 32 ? (want > 0 ? want : 1) : 148 * 32), 256, 0, st>>>(a, tb);
    count_launches(3);
    return cudaGetLastError();
}

}  // namespace

size_t gdn_bwd_ws_bytes(int64_t n_rows, int n_seg, int H, int d) { return bwd_layout(n_rows, n_seg, H, d).total; }

cudaError_t launch_gdn_bwd(const GdnBwdArgs& a, int dt, cudaStream_t st) {
    if (a.n_seg == 0) return cudaSuccess;
    if (dt == MOM_BF16) {
        switch (a.d) {
            case 64: return launch_bwd_t<bf16, 64>(a, st);
            case 128: return launch_bwd_t<bf16, 128>(a, st);
            case 256: return launch_bwd_t<bf16, 256>(a, st);
        }
    } else {
        switch (a.d) {
            case 64: return launch_bwd_t<float, 64>(a, st);
            case 128: return launch_bwd_t<float, 128>(a, st);
            case 256: return launch_bwd_t<float, 256>(a, st);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace mom
