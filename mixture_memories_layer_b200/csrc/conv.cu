// The short causal convolutions of the Gated DeltaNet block around the
// memories.  (The authors' MoM blog post, experiments section, names Gated
// DeltaNet as every memory's mixer; the pages print nothing of the block, so
// the plain Gated DeltaNet block is taken: q, k and v each pass through a
// depthwise causal convolution of a few taps and SiLU, q and k are then
// L2-normalised per head.)
//
//   out[r, c] = act( sum_{j=0}^{W-1} w[grp][W-1-j][c] * z[r-j, c] ),
//
// over the taps with r-j inside r's segment (rows before the segment's
// start count as zero), act = SiLU, then optionally the per-head L2 norm
// x / sqrt(|x|^2 + 1e-6).  Segments are the rows a recurrence sees: a
// sequence for the shared q, k, v; a (memory, sequence) segment of the
// reordered rows for memory m's k, v, whose filters are group m's
// (grp = segment / seg_per_group).
//
// HBM-bound: every row is read once from DRAM and written once.  One warp
// per task of RANGE consecutive rows x 256 channels (lane l: channels 8l ..
// 8l+7, one 16-byte vector per row), streamed through a register ring with
// each row's load issued P rows before its use; the W-1 rows before the task
// come from L2.  The filters are stored tap-major ([groups, W, C])
// so that a tap of the warp's 256 channels is one coalesced 1 KB read.  One
// launch takes several problems (the block's
// five: q, k_sh, v_sh over the sequences, k_p, v_p over the memory
// segments), their tasks numbered one after the other.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mom {
namespace {

using sm100::cp_async_16;
using sm100::cp_async_commit;
using sm100::cp_async_wait;

constexpr int RANGE = 32;         // rows per warp task
constexpr int MAXP = 8;           // problems per launch

struct ConvBatch {
    ConvProblem pr[MAXP];
    int64_t item_base[MAXP + 1];  // first item of each problem (upper bounds of its rows)
    int n;
    int C;                        // channels per row
    int d;                        // head width of the norm
    void* err;
};

__device__ __forceinline__ float bf_at(const uint4& u, int e) {
    const uint32_t w = e < 2 ? u.x : e < 4 ? u.y : e < 6 ? u.z : u.w;
    return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

template <int W>
__device__ __forceinline__ void load_filters(const float* w, int C, int grp, int c, float (&wv)[8][W]) {
    const float* base = w + (int64_t)grp * W * C + c;
#pragma unroll
    for (int t = 0; t < W; ++t) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(base + (int64_t)t * C));
        const float4 b = __ldg(reinterpret_cast<const float4*>(base + (int64_t)t * C) + 1);
        wv[0][t] = a.x; wv[1][t] = a.y; wv[2][t] = a.z; wv[3][t] = a.w;
        wv[4][t] = b.x; wv[5][t] = b.y; wv[6][t] = b.z; wv[7][t] = b.w;
    }
}

// Segment of row r0 (seg_cu[n_seg] > r0 >= seg_cu[0]): the last s with
// seg_cu[s] <= r0.  Up to 32 bounds are read by the warp in one load and
// counted by a ballot; longer tables by a binary search.
__device__ __forceinline__ int segment_of(const int32_t* seg_cu, int n_seg, int64_t r0, int lane) {
    if (n_seg <= 31) {
        const int32_t v = lane <= n_seg ? __ldg(seg_cu + lane) : 0x7fffffff;
        return __popc(__ballot_sync(0xffffffffu, v <= r0)) - 1;
    }
    int lo = 0, hi = n_seg;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(seg_cu + mid) <= r0) lo = mid; else hi = mid;
    }
    return lo;
}

// One warp streams a range of RANGE rows x 256 channels through a ring of P
// rows in shared memory filled by cp.async (every lane copies and later
// reads its own 16 bytes of a row, so no cross-lane synchronisation), each
// row requested P rows ahead of its use.  Rows are taken U at a time: each
// is converted to fp32 once, the W-1 rows before the group are carried over
// in registers, and rows before a segment's start are zeroed there, so the
// taps need no masks.
constexpr int P = 8;                                      // rows in flight per warp
constexpr int U = 4;                                      // rows per unrolled step
constexpr int CONV_THREADS = 256;

// SiLU(v) = v sigmoid(v) = v (1 + tanh(v/2)) / 2, with the hardware tanh
// approximation (relative error about 2^-11; the result is rounded to bf16)
__device__ __forceinline__ float silu_tanh(float v) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * v));
    const float h = 0.5f * v;
    return fmaf(h, t, h);
}

template <int W>
__global__ void __launch_bounds__(CONV_THREADS, 2) short_conv_kernel(const __grid_constant__ ConvBatch B) {
    constexpr int WP = W > 1 ? W - 1 : 1;
    __shared__ __align__(16) uint4 ring_all[CONV_THREADS / 32][P][32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(&ring_all[wid][0][lane]);
    constexpr uint32_t SLOT = 32 * 16;                    // bytes per ring slot
    const int nblk = (B.C + 255) / 256;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t C = B.C;
    int pi = 0;
    for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + wid; it < B.item_base[B.n]; it += nw) {
        while (it >= B.item_base[pi + 1]) ++pi;           // items only grow
        const ConvProblem& a = B.pr[pi];
        const int64_t r_beg = __ldg(a.seg_cu), r_end = __ldg(a.seg_cu + a.n_seg);
        if (r_beg < 0 || r_end < r_beg || r_end > a.n_rows) {
            if (lane == 0 && it == B.item_base[pi]) record_error(B.err, MOM_DEVERR_SEGMENT, pi);
            continue;
        }
        const int64_t local = it - B.item_base[pi];
        const int64_t ra = r_beg + (local / nblk) * RANGE;
        if (ra >= r_end) continue;                        // past the rows this problem really has
        const int nr = (int)(ra + RANGE < r_end ? RANGE : r_end - ra);     // rows of this task
        const int c = (int)(local % nblk) * 256 + 8 * lane;
        bool on = c < B.C;
        // ring entry i (slot i % P) holds row ra - (W-1) + i; rows outside
        // [r_beg, ra + nr) are zero-filled (their source: a valid row, unread)
        const bf16* zq = reinterpret_cast<const bf16*>(a.z) + (on ? c : 0);
        const int64_t q0 = ra - (W - 1);
        const int n_in = nr + W - 1;
        auto request = [&](int i) {
            const int64_t r = q0 + i;
            const bool in = on && i < n_in && r >= r_beg;
            cp_async_16(ring0 + (uint32_t)(i & (P - 1)) * SLOT, zq + (in ? r : r_beg) * C, in ? 16u : 0u);
            cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < P; ++i) request(i);
        int s = segment_of(a.seg_cu, a.n_seg, ra, lane);
        int64_t s_beg = __ldg(a.seg_cu + s), s_end = __ldg(a.seg_cu + s + 1);
        int grp = s / a.seg_per_group;
        if (grp >= a.n_groups) {
            if (lane == 0) record_error(B.err, MOM_DEVERR_SEGMENT, s);
            on = false;
            grp = 0;
        }
        float wv[8][W];
        load_filters<W>(a.w, B.C, grp, on ? c : 0, wv);
        // xs[0 .. W-2]: the rows before the group (oldest first); xs[W-1 + k]: row k of the group
        float xs[WP + U][8];
        int i = 0;
#pragma unroll
        for (int j = 0; j < W - 1; ++j, ++i) {            // the rows before the range
            cp_async_wait<P - 1>();
            const uint4 v = *reinterpret_cast<const uint4*>(&ring_all[wid][i & (P - 1)][lane]);
            request(i + P);
            const bool keep = q0 + j >= s_beg;
#pragma unroll
            for (int e = 0; e < 8; ++e) xs[j][e] = keep ? bf_at(v, e) : 0.f;
        }
        bf16* op = reinterpret_cast<bf16*>(a.out) + ra * C + c;
        for (int k0 = 0; k0 < nr; k0 += U) {
#pragma unroll
            for (int k = 0; k < U; ++k, ++i) {
                cp_async_wait<P - 1>();
                const uint4 v = *reinterpret_cast<const uint4*>(&ring_all[wid][i & (P - 1)][lane]);
                request(i + P);
#pragma unroll
                for (int e = 0; e < 8; ++e) xs[WP + k][e] = bf_at(v, e);
            }
#pragma unroll
            for (int k = 0; k < U; ++k) {
                if (k0 + k < nr) {                        // uniform over the warp
                    const int64_t r = ra + k0 + k;
                    if (r >= s_end) {                     // a segment starts here: no tap reaches back past it
                        while (s + 1 < a.n_seg && r >= __ldg(a.seg_cu + s + 1)) ++s;
                        s_beg = __ldg(a.seg_cu + s);
                        s_end = __ldg(a.seg_cu + s + 1);
                        const int g2 = s / a.seg_per_group;
                        if (g2 >= a.n_groups) {
                            if (lane == 0) record_error(B.err, MOM_DEVERR_SEGMENT, s);
                            on = false;
                        } else if (g2 != grp) {
                            grp = g2;
                            load_filters<W>(a.w, B.C, grp, on ? c : 0, wv);
                        }
#pragma unroll
                        for (int j = 0; j < WP + k; ++j)
#pragma unroll
                            for (int e = 0; e < 8; ++e) xs[j][e] = 0.f;
                    }
                    float acc[8], ss = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float t = wv[e][W - 1] * xs[WP + k][e];
#pragma unroll
                        for (int j = 1; j < W; ++j) t = fmaf(wv[e][W - 1 - j], xs[WP + k - j][e], t);
                        acc[e] = silu_tanh(t);
                        ss = fmaf(acc[e], acc[e], ss);
                    }
                    if (a.l2) {                           // uniform over the warp
                        if (!on) ss = 0.f;
                        for (int o = B.d >> 4; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                        const float sc = rsqrtf(ss + 1e-6f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] *= sc;
                    }
                    if (on) store_vec<8>(op, acc);
                    op += C;
                }
            }
            // the group's last W-1 rows lead the next group
#pragma unroll
            for (int j = 0; j < W - 1; ++j)
#pragma unroll
                for (int e = 0; e < 8; ++e) xs[j][e] = xs[U + j][e];
        }
        cp_async_wait<0>();                               // no copy of this task lands in the next one's slots
    }
}

template <int W>
cudaError_t launch_w(const ConvBatch& b, cudaStream_t st) {
    int64_t grid = cdiv(b.item_base[b.n], 8);
    if (grid > 148 * 16) grid = 148 * 16;
    if (grid < 1) grid = 1;
    short_conv_kernel<W><<<(unsigned)grid, CONV_THREADS, 0, st>>>(b);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_short_conv(const ConvProblem* problems, int n, int C, int W, int d, void* err, cudaStream_t st) {
    if (n < 1 || n > MAXP) return cudaErrorInvalidValue;
    ConvBatch b{};
    b.n = n;
    b.C = C;
    b.d = d;
    b.err = err;
    const int nblk = (C + 255) / 256;
    b.item_base[0] = 0;
    for (int i = 0; i < n; ++i) {
        b.pr[i] = problems[i];
        b.item_base[i + 1] = b.item_base[i] + cdiv(problems[i].n_rows, RANGE) * nblk;
    }
    if (b.item_base[n] == 0) return cudaSuccess;
    switch (W) {
        case 1: return launch_w<1>(b, st);
        case 2: return launch_w<2>(b, st);
        case 3: return launch_w<3>(b, st);
        case 4: return launch_w<4>(b, st);
    }
    return cudaErrorInvalidValue;
}


// ---------------------------------------------------------------- decode --
// One new row per sequence: each convolution reads its window of the W-1 raw
// rows before (bf16, oldest first, zero before the sequence's -- or for a
// memory, its routed tokens' -- start), writes act(conv) (+ the L2 norm)
// and shifts the new raw row into the window.  The shared q, k, v windows
// are per sequence; memory m's k, v windows per (sequence, memory), found
// through the routed row's token (perm) and its memory (the mem_offset range
// holding the row).  A sequence routes each memory at most once, so no two
// warps touch one window.
namespace {

template <int W>
__global__ void __launch_bounds__(256) conv_step_kernel(const __grid_constant__ ConvStepArgs a) {
    static_assert(W >= 2, "a window needs at least one row");
    const int lane = threadIdx.x & 31;
    const int nblk = (a.C + 255) / 256;
    const int64_t n_sh = 3LL * a.B * nblk, n_rt = 2LL * a.B * a.K * nblk;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < n_sh + n_rt; it += nw) {
        int pi, l2, m = 0;
        int64_t row, b;
        const float* filt;
        bf16* win;
        int blk;
        if (it < n_sh) {
            pi = (int)(it / ((int64_t)a.B * nblk));
            const int64_t rem = it % ((int64_t)a.B * nblk);
            row = rem / nblk;
            blk = (int)(rem % nblk);
            b = row;
            win = a.st_sh + ((b * 3 + pi) * (W - 1)) * (int64_t)a.C;
            filt = a.w[pi];
            l2 = pi < 2;
        } else {
            const int64_t it2 = it - n_sh;
            const int64_t per = (int64_t)a.B * a.K * nblk;
            pi = 3 + (int)(it2 / per);
            const int64_t rem = it2 % per;
            row = rem / nblk;
            blk = (int)(rem % nblk);
            b = __ldg(a.perm + row);
            const int32_t v = lane <= a.M ? __ldg(a.mem_offset + lane) : 0x7fffffff;
            m = __popc(__ballot_sync(0xffffffffu, v <= row)) - 1;
            if (b < 0 || b >= a.B || m < 0 || m >= a.M) {
                if (lane == 0) record_error(a.err, MOM_DEVERR_ROW_INDEX, row);
                continue;                                 // uniform over the warp
            }
            win = a.st_mem + (((b * a.M + m) * 2 + (pi - 3)) * (W - 1)) * (int64_t)a.C;
            filt = a.w[pi] + (int64_t)m * W * a.C;
            l2 = pi == 3;
        }
        const int c = blk * 256 + 8 * lane;
        const bool on = c < a.C;
        uint4 z = make_uint4(0u, 0u, 0u, 0u), wr[W - 1];
        float wv[8][W];
        if (on) {
            z = __ldg(reinterpret_cast<const uint4*>(a.z[pi] + row * a.C + c));
#pragma unroll
            for (int t = 0; t < W - 1; ++t) wr[t] = *reinterpret_cast<const uint4*>(win + (int64_t)t * a.C + c);
            load_filters<W>(filt, a.C, 0, c, wv);
        } else {
#pragma unroll
            for (int t = 0; t < W - 1; ++t) wr[t] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
                for (int t = 0; t < W; ++t) wv[e][t] = 0.f;
        }
        float acc[8], ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float s = wv[e][W - 1] * bf_at(z, e);
#pragma unroll
            for (int t = 0; t < W - 1; ++t) s = fmaf(wv[e][t], bf_at(wr[t], e), s);
            acc[e] = silu_tanh(s);
            ss = fmaf(acc[e], acc[e], ss);
        }
        if (l2) {                                         // uniform over the warp
            for (int o = a.d >> 4; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float sc = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] *= sc;
        }
        if (on) {
            store_vec<8>(a.out[pi] + row * a.C + c, acc);
#pragma unroll
            for (int t = 0; t < W - 2; ++t) *reinterpret_cast<uint4*>(win + (int64_t)t * a.C + c) = wr[t + 1];
            *reinterpret_cast<uint4*>(win + (int64_t)(W - 2) * a.C + c) = z;
        }
    }
}

// The windows a forward leaves: the raw rows of each sequence's (and each
// (memory, sequence) segment's) last W-1 rows, zero where the segment is
// shorter.
__global__ void __launch_bounds__(256) conv_state_kernel(const __grid_constant__ ConvStateArgs a) {
    const int lane = threadIdx.x & 31;
    const int nblk = (a.C + 255) / 256;
    const int Wm = a.W - 1;
    const int64_t n_sh = 3LL * a.S * Wm * nblk, n_rt = 2LL * a.M * a.S * Wm * nblk;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < n_sh + n_rt; it += nw) {
        const bool sh = it < n_sh;
        int64_t r = sh ? it : it - n_sh;
        const int blk = (int)(r % nblk);
        r /= nblk;
        const int j = (int)(r % Wm);
        r /= Wm;
        const int pi = (int)(r % (sh ? 3 : 2));
        r /= sh ? 3 : 2;
        int64_t lo, hi, lim;
        bf16* dst;
        const bf16* src;
        if (sh) {
            const int s = (int)r;
            lo = a.cu[s];
            hi = a.cu[s + 1];
            lim = a.n_tok;
            dst = a.st_sh + (((int64_t)s * 3 + pi) * Wm + j) * a.C;
            src = a.z[pi];
        } else {
            const int s = (int)(r % a.S), m = (int)(r / a.S);
            lo = a.seg_cu[m * a.S + s];
            hi = a.seg_cu[m * a.S + s + 1];
            lim = a.n_rows;
            dst = a.st_mem + ((((int64_t)s * a.M + m) * 2 + pi) * Wm + j) * a.C;
            src = a.z[3 + pi];
        }
        const bool bad = lo < 0 || hi < lo || hi > lim;
        if (bad && lane == 0 && blk == 0 && j == 0) record_error(a.err, MOM_DEVERR_SEGMENT, it);
        const int64_t row = hi - Wm + j;
        const int c = blk * 256 + 8 * lane;
        if (c < a.C) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (!bad && row >= lo) v = __ldg(reinterpret_cast<const uint4*>(src + row * a.C + c));
            *reinterpret_cast<uint4*>(dst + c) = v;
        }
    }
}

}  // namespace

cudaError_t launch_conv_step(const ConvStepArgs& a, int W, cudaStream_t st) {
    const int64_t items = (3LL * a.B + 2LL * a.B * a.K) * ((a.C + 255) / 256);
    if (items == 0) return cudaSuccess;
    int64_t grid = cdiv(items, 8);
    if (grid > 148 * 8) grid = 148 * 8;
    switch (W) {
        case 2: conv_step_kernel<2><<<(unsigned)grid, 256, 0, st>>>(a); break;
        case 3: conv_step_kernel<3><<<(unsigned)grid, 256, 0, st>>>(a); break;
        case 4: conv_step_kernel<4><<<(unsigned)grid, 256, 0, st>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_conv_state(const ConvStateArgs& a, cudaStream_t st) {
    const int64_t items = (3LL * a.S + 2LL * a.M * a.S) * (a.W - 1) * ((a.C + 255) / 256);
    if (items == 0) return cudaSuccess;
    int64_t grid = cdiv(items, 8);
    if (grid > 148 * 8) grid = 148 * 8;
    conv_state_kernel<<<(unsigned)grid, 256, 0, st>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
