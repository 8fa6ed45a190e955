// The layer's backward around its recurrences (training is the pages' main
// workload: "MoM: Linear Sequence Modeling with Mixture-of-Memories", Key
// points): the adjoints of the combine, of the renormalised router gates
// ("MoM: Mixture-of-Memories Fixes Linear Attention Recall", Router
// mechanics), of the per-head L2 norms and of the gates, the per-token sums
// of what the routed rows received, column sums, and one grouped float32
// GEMM for the input and weight gradients of every projection.  First path:
// CUDA cores, float32 accumulation.
#include "common.cuh"
#include "kernels.h"

namespace mom {
namespace {

// do_p[row_of(t,j)] = g_tj dout_t; dgate_tj = <dout_t, o_p[row_of(t,j)]>.  One warp per token.
template <typename T>
__global__ void __launch_bounds__(256)
combine_bwd_kernel(const T* __restrict__ dout, const T* __restrict__ o_p, const int32_t* __restrict__ row_of,
                   const float* __restrict__ gate, int64_t n_tok, int K, int HD, int64_t n_rows, T* __restrict__ do_p,
                   float* __restrict__ dgate, void* err) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < n_tok; t += warps) {
        for (int j = 0; j < K; ++j) {
            const int64_t r = row_of[t * K + j];
            if (r < 0 || r >= n_rows) {
                if (lane == 0) { record_error(err, MOM_DEVERR_ROW_INDEX, t * K + j); dgate[t * K + j] = 0.f; }
                continue;
            }
            const float g = gate[t * K + j];
            float acc = 0.f;
            for (int c = lane; c < HD; c += 32) {
                const float dy = to_f(dout[t * HD + c]);
                do_p[r * HD + c] = from_f<T>(g * dy);
                acc = fmaf(dy, to_f(o_p[r * HD + c]), acc);
            }
            acc = warp_sum(acc);
            if (lane == 0) dgate[t * K + j] = acc;
        }
    }
}

// dlogits = the adjoint of g_j = exp(l_j) / sum_i exp(l_i) over the chosen
// memories: dl_j = g_j (dg_j - sum_i g_i dg_i), zero for the others.
__global__ void __launch_bounds__(256)
router_bwd_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate, const float* __restrict__ dgate,
                  int64_t n_tok, int K, int M, float* __restrict__ dlogits, void* err) {
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_tok; t += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int j = 0; j < K; ++j) s = fmaf(gate[t * K + j], dgate[t * K + j], s);
        for (int m = 0; m < M; ++m) dlogits[t * M + m] = 0.f;
        for (int j = 0; j < K; ++j) {
            const int m = idx[t * K + j];
            if (m < 0 || m >= M) { record_error(err, MOM_DEVERR_MEM_INDEX, t); continue; }
            dlogits[t * M + m] = gate[t * K + j] * (dgate[t * K + j] - s);
        }
    }
}

// dst[t] = base[t] (or 0) + sum_j src[row_of(t, j)], rows of W floats.  One warp per token.
__global__ void __launch_bounds__(256)
rows_sum_kernel(const float* __restrict__ src, int64_t n_src, const int32_t* __restrict__ row_of, int K,
                const float* __restrict__ base, int64_t n_tok, int W, float* __restrict__ dst, void* err) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < n_tok; t += warps) {
        if (lane == 0)
            for (int j = 0; j < K; ++j) {
                const int64_t r = row_of[t * K + j];
                if (r < 0 || r >= n_src) record_error(err, MOM_DEVERR_ROW_INDEX, t * K + j);
            }
        for (int c = lane; c < W; c += 32) {
            float acc = base ? base[t * W + c] : 0.f;
            for (int j = 0; j < K; ++j) {
                const int64_t r = row_of[t * K + j];
                if (r >= 0 && r < n_src) acc += src[r * W + c];
            }
            dst[t * W + c] = acc;
        }
    }
}

// dz = (dy - y (y . dy)) / n per (row, head); y the normalised value, n its
// length sqrt(|z|^2 + eps).  One warp per (row, head).
template <typename T>
__global__ void __launch_bounds__(256)
l2norm_bwd_kernel(const T* __restrict__ y, const float* __restrict__ dy, const float* __restrict__ nrm, int64_t rows,
                  int H, int d, float* __restrict__ dz, int64_t ldz, int64_t col0) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t rh = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); rh < rows * H; rh += warps) {
        const int64_t r = rh / H;
        const int h = (int)(rh - r * H);
        const int64_t o = rh * d;
        float dot = 0.f;
        for (int c = lane; c < d; c += 32) dot = fmaf(to_f(y[o + c]), dy[o + c], dot);
        dot = warp_sum(dot);
        const float inv = 1.f / nrm[rh];
        for (int c = lane; c < d; c += 32)
            dz[r * ldz + col0 + (int64_t)h * d + c] = (dy[o + c] - to_f(y[o + c]) * dot) * inv;
    }
}

// beta = sigmoid(z_b): dz_b = dbeta beta (1 - beta).
// log alpha = -e^A softplus(z_a): dz_a = dla (-e^A) sigmoid(z_a), with
// sigmoid(z_a) = 1 - e^(-softplus(z_a)) and softplus(z_a) = -log alpha e^-A;
// dala = dla log alpha (summed over tokens: dA).  With a group table (goff,
// n_groups: the rows of group g are goff[g] .. goff[g+1]-1) row r takes the
// A of its group, A[g * H + h] (per-memory gates of the reordered rows).
__device__ __forceinline__ int group_of(const int32_t* goff, int n_groups, int64_t r) {
    int lo = 0, hi = n_groups;                       // the last g with goff[g] <= r
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(goff + mid) <= r) lo = mid; else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(256)
gates_bwd_kernel(const float* __restrict__ beta, const float* __restrict__ la, const float* __restrict__ dbeta,
                 const float* __restrict__ dla, const float* __restrict__ A, const int32_t* __restrict__ goff,
                 int n_groups, int64_t n, int H, float* __restrict__ dz, int64_t ldz, int64_t col_b, int64_t col_a,
                 float* __restrict__ dala) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n * H; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / H;
        const int h = (int)(i - r * H);
        const int g = goff ? group_of(goff, n_groups, r) : 0;
        const float b = beta[i], l = la[i], eA = expf(A[(int64_t)g * H + h]);
        dz[r * ldz + col_b + h] = dbeta[i] * b * (1.f - b);
        const float sp = -l / eA;
        const float sg = -expm1f(-sp);                  // 1 - e^-sp
        dz[r * ldz + col_a + h] = dla[i] * (-eA) * sg;
        dala[i] = dla[i] * l;
    }
}

// out[g * C + c] = sum over the rows r of group g of a[r * lda + c], c < C:
// one warp per (group, column), lanes over rows.  No group table: one group
// of rows 0 .. rows-1.
__global__ void __launch_bounds__(256)
col_sums_kernel(const float* __restrict__ a, int64_t rows, int64_t lda, int64_t C, const int32_t* __restrict__ goff,
                int n_groups, float* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < (int64_t)n_groups * C;
         w += warps) {
        const int64_t g = w / C, c = w - g * C;
        int64_t lo = 0, hi = rows;
        if (goff) {
            lo = __ldg(goff + g);
            hi = __ldg(goff + g + 1);
            if (lo < 0) lo = 0;
            if (hi > rows) hi = rows;
        }
        float acc = 0.f;
        for (int64_t r = lo + lane; r < hi; r += 32) acc += a[r * lda + c];
        acc = warp_sum(acc);
        if (lane == 0) out[w] = acc;
    }
}

// ------------------------------------------------------------ grouped GEMM
// 128 x 128 output tiles, 8-deep k steps double-buffered in shared memory,
// 256 threads with 8 x 8 outputs each (two 4 x 4 blocks 64 apart in each
// direction, so that a warp's shared-memory reads are broadcasts or
// consecutive 16-byte chunks).
constexpr int GBM = 128, GBN = 128, GBK = 8;

struct GemmArgs {
    int trans_a;
    const float* A;
    int64_t lda;
    const void* B;
    int64_t ldb;
    const int32_t* b_rows;     // TRANS: row of B for reduction row r (null: r)
    float* C;
    int64_t ldc;
    int64_t M, N, K;
    const int32_t* goff;
    const int32_t* gmem;
    int n_groups;
    int64_t b_group_stride, c_group_stride;
    int accumulate;
    int64_t n_b_rows;          // rows of B (bounds of b_rows)
    void* err;
    int splits;                // TRANS: the reduction of a group split over this many CTAs (atomic sums)
};

// trans_a = 0: the CTA's 128-row tile of a group (tiles listed over all groups)
// trans_a = 1: blockIdx.z is the group, the tile of C_g is (blockIdx.y, blockIdx.x)
template <typename TB>
__global__ void __launch_bounds__(256)
gemm_grouped_kernel(GemmArgs g) {
    __shared__ __align__(16) float As[2][GBK][GBM];
    __shared__ __align__(16) float Bs[2][GBK][GBN];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const TB* B = reinterpret_cast<const TB*>(g.B);
    const int64_t n0 = (int64_t)blockIdx.x * GBN;
    int64_t m0 = 0, m1 = 0, k0 = 0, k1 = 0;
    const TB* Bg = B;
    float* Cg = g.C;
    if (!g.trans_a) {
        int64_t t = blockIdx.y;
        int grp = -1;
        for (int q = 0; q < g.n_groups; ++q) {
            const int64_t lo = g.goff[q], hi = g.goff[q + 1];
            if (lo < 0 || hi < lo) { if (tid == 0 && blockIdx.x == 0) record_error(g.err, MOM_DEVERR_SEGMENT, q); return; }
            const int64_t nt = (hi - lo + GBM - 1) / GBM;
            if (t < nt) { grp = q; m0 = lo + t * GBM; m1 = m0 + GBM < hi ? m0 + GBM : hi; break; }
            t -= nt;
        }
        if (grp < 0) return;
        const int64_t w = g.gmem ? g.gmem[grp] : grp;
        Bg = B + w * g.b_group_stride;
        k0 = 0;
        k1 = g.K;
    } else {
        const int grp = blockIdx.z / g.splits, sp = blockIdx.z % g.splits;
        m0 = (int64_t)blockIdx.y * GBM;
        m1 = m0 + GBM < g.M ? m0 + GBM : g.M;
        if (m0 >= g.M) return;
        const int64_t lo = g.goff[grp], hi = g.goff[grp + 1];
        if (lo < 0 || hi < lo) { if (tid == 0 && blockIdx.x == 0) record_error(g.err, MOM_DEVERR_SEGMENT, grp); return; }
        // this CTA's share of the reduction, in whole k steps
        const int64_t steps = (hi - lo + GBK - 1) / GBK, per = (steps + g.splits - 1) / g.splits;
        k0 = lo + sp * per * GBK;
        k1 = k0 + per * GBK < hi ? k0 + per * GBK : hi;
        if (k0 >= k1) return;
        const int64_t w = g.gmem ? g.gmem[grp] : grp;
        Cg = g.C + w * g.c_group_stride;
    }
    // loader: 4 A values and 4 B values per thread per k step
    float ra[4], rb[4];
    auto load = [&](int64_t kb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int kk, mm;
            if (!g.trans_a) { mm = tid >> 1; kk = (tid & 1) * 4 + e; } else { kk = tid >> 5; mm = (tid & 31) * 4 + e; }
            const int64_t m = m0 + mm, k = kb + kk;
            ra[e] = (m < m1 && k < k1) ? (g.trans_a ? g.A[k * g.lda + m] : g.A[m * g.lda + k]) : 0.f;
        }
        const int kk = tid >> 5;
        const int64_t k = kb + kk;
        int64_t br = k;
        if (k < k1 && g.trans_a && g.b_rows) {
            br = g.b_rows[k];
            if (br < 0 || br >= g.n_b_rows) { record_error(g.err, MOM_DEVERR_ROW_INDEX, k); br = -1; }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t n = n0 + (tid & 31) * 4 + e;
            rb[e] = (k < k1 && br >= 0 && n < g.N) ? to_f(Bg[br * g.ldb + n]) : 0.f;
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (!g.trans_a) As[buf][(tid & 1) * 4 + e][tid >> 1] = ra[e];
            else As[buf][tid >> 5][(tid & 31) * 4 + e] = ra[e];
        }
        *reinterpret_cast<float4*>(&Bs[buf][tid >> 5][(tid & 31) * 4]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
    };
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    int buf = 0;
    if (k0 < k1) {
        load(k0);
        store(0);
    }
    __syncthreads();
    for (int64_t kb = k0; kb < k1; kb += GBK) {
        const bool more = kb + GBK < k1;
        if (more) load(kb + GBK);
#pragma unroll
        for (int kk = 0; kk < GBK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
        if (m >= m1) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
            if (n >= g.N) continue;
            float* c = Cg + m * g.ldc + n;
            if (g.trans_a) atomicAdd(c, acc[i][j]);          // split partial sums; C zeroed first unless accumulating
            else *c = g.accumulate ? *c + acc[i][j] : acc[i][j];
        }
    }
}

// The same products on the tensor cores when B is bf16: tf32 operands (B
// exactly, A rounded to a 10-bit mantissa), fp32 accumulation, m16n8k8
// MMAs.  Tiles of 128 x 128 over k steps of 16 held in padded shared memory
// (stride 136 floats: the fragment reads of a warp hit 32 banks), the next
// step's operands loaded into registers while the current one is multiplied;
// 8 warps, each a 64 x 32 piece (4 x 4 MMAs per k8 step).
constexpr int TBK = 16, TPAD = GBM + 8, TVAL = TBK * GBM / 256;   // values per thread per operand and step
constexpr int TPR = GBM / TVAL;                                      // threads per k row of an operand tile
static_assert(TBK / TVAL == 2, "two threads per row of a row-major A tile");
constexpr size_t TF32_SMEM = 2ull * 2 * TBK * TPAD * 4;

__device__ __forceinline__ uint32_t tf32_bits(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__global__ void __launch_bounds__(256, 2)
gemm_grouped_tf32_kernel(GemmArgs g) {
    extern __shared__ __align__(16) uint32_t tf32_smem[];
    auto As = reinterpret_cast<uint32_t (*)[TBK][TPAD]>(tf32_smem);
    auto Bs = reinterpret_cast<uint32_t (*)[TBK][TPAD]>(tf32_smem + 2 * TBK * TPAD);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bf16* B = reinterpret_cast<const bf16*>(g.B);
    const int64_t n0 = (int64_t)blockIdx.x * GBN;
    int64_t m0 = 0, m1 = 0, k0 = 0, k1 = 0;
    const bf16* Bg = B;
    float* Cg = g.C;
    if (!g.trans_a) {
        int64_t t = blockIdx.y;
        int grp = -1;
        for (int q = 0; q < g.n_groups; ++q) {
            const int64_t lo = g.goff[q], hi = g.goff[q + 1];
            if (lo < 0 || hi < lo) { if (tid == 0 && blockIdx.x == 0) record_error(g.err, MOM_DEVERR_SEGMENT, q); return; }
            const int64_t nt = (hi - lo + GBM - 1) / GBM;
            if (t < nt) { grp = q; m0 = lo + t * GBM; m1 = m0 + GBM < hi ? m0 + GBM : hi; break; }
            t -= nt;
        }
        if (grp < 0) return;
        const int64_t w = g.gmem ? g.gmem[grp] : grp;
        Bg = B + w * g.b_group_stride;
        k0 = 0;
        k1 = g.K;
    } else {
        const int grp = blockIdx.z / g.splits, sp = blockIdx.z % g.splits;
        m0 = (int64_t)blockIdx.y * GBM;
        m1 = m0 + GBM < g.M ? m0 + GBM : g.M;
        if (m0 >= g.M) return;
        const int64_t lo = g.goff[grp], hi = g.goff[grp + 1];
        if (lo < 0 || hi < lo) { if (tid == 0 && blockIdx.x == 0) record_error(g.err, MOM_DEVERR_SEGMENT, grp); return; }
        const int64_t steps = (hi - lo + TBK - 1) / TBK, per = (steps + g.splits - 1) / g.splits;
        k0 = lo + sp * per * TBK;
        k1 = k0 + per * TBK < hi ? k0 + per * TBK : hi;
        if (k0 >= k1) return;
        const int64_t w = g.gmem ? g.gmem[grp] : grp;
        Cg = g.C + w * g.c_group_stride;
    }
    // loader: TVAL A and B values per thread per k step.  A: row m = tid / 2,
    // k = (tid % 2) TVAL + e (trans_a = 0) or k = tid / TPR, m = (tid % TPR)
    // TVAL + e (trans_a = 1); B: k = tid / TPR, n = (tid % TPR) TVAL + e
    float ra[TVAL], rb[TVAL];
    // each thread's TVAL values of an operand are contiguous in memory (A's
    // k run or m run, B's n run): two 16-byte loads of A, one of B where the
    // run is whole and aligned, element loads at the ragged edges
    const bool a_vec = ((reinterpret_cast<uintptr_t>(g.A) & 15) == 0) && (g.lda % 4 == 0) &&
                       (g.trans_a || (k0 & 3) == 0);
    const bool b_vec = ((reinterpret_cast<uintptr_t>(Bg) & 15) == 0) && (g.ldb % 8 == 0);
    auto load = [&](int64_t kb) {
        int64_t am, ak;                                   // the first of the thread's A values
        if (!g.trans_a) { am = m0 + (tid >> 1); ak = kb + (tid & 1) * TVAL; } else { ak = kb + tid / TPR; am = m0 + (tid % TPR) * TVAL; }
        const bool a_whole = g.trans_a ? (ak < k1 && am + TVAL <= m1) : (am < m1 && ak + TVAL <= k1);
        if (a_vec && a_whole) {
            const float4* src = reinterpret_cast<const float4*>(g.A + (g.trans_a ? ak * g.lda + am : am * g.lda + ak));
#pragma unroll
            for (int v = 0; v < TVAL / 4; ++v) {
                const float4 q = __ldg(src + v);
                ra[4 * v] = q.x; ra[4 * v + 1] = q.y; ra[4 * v + 2] = q.z; ra[4 * v + 3] = q.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < TVAL; ++e) {
                const int64_t m = g.trans_a ? am + e : am, k = g.trans_a ? ak : ak + e;
                ra[e] = (m < m1 && k < k1) ? (g.trans_a ? g.A[k * g.lda + m] : g.A[m * g.lda + k]) : 0.f;
            }
        }
        const int kk = tid / TPR;
        const int64_t k = kb + kk;
        int64_t br = k;
        if (k < k1 && g.trans_a && g.b_rows) {
            br = g.b_rows[k];
            if (br < 0 || br >= g.n_b_rows) { record_error(g.err, MOM_DEVERR_ROW_INDEX, k); br = -1; }
        }
        const int64_t nb = n0 + (tid % TPR) * TVAL;
        if (b_vec && k < k1 && br >= 0 && nb + TVAL <= g.N) {
            static_assert(TVAL % 8 == 0, "whole 16-byte runs of B");
            const uint4* src = reinterpret_cast<const uint4*>(Bg + br * g.ldb + nb);
#pragma unroll
            for (int v = 0; v < TVAL / 8; ++v) {
                const uint4 q = __ldg(src + v);
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    rb[8 * v + 2 * e] = __uint_as_float(w4[e] << 16);
                    rb[8 * v + 2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < TVAL; ++e) {
                const int64_t n = nb + e;
                rb[e] = (k < k1 && br >= 0 && n < g.N) ? __bfloat162float(Bg[br * g.ldb + n]) : 0.f;
            }
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int e = 0; e < TVAL; ++e) {
            if (!g.trans_a) As[buf][(tid & 1) * TVAL + e][tid >> 1] = tf32_bits(ra[e]);
            else As[buf][tid / TPR][(tid % TPR) * TVAL + e] = tf32_bits(ra[e]);
            Bs[buf][tid / TPR][(tid % TPR) * TVAL + e] = tf32_bits(rb[e]);
        }
    };
    const int wm = warp >> 2, wn = warp & 3;          // 2 x 4 warps of 64 x 32
    const int gr = lane >> 2, gc = lane & 3;
    float acc[4][4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
    int buf = 0;
    if (k0 < k1) {
        load(k0);
        store(0);
    }
    __syncthreads();
    for (int64_t kb = k0; kb < k1; kb += TBK) {
        const bool more = kb + TBK < k1;
        if (more) load(kb + TBK);
#pragma unroll
        for (int ks = 0; ks < TBK; ks += 8) {
            uint32_t af[4][4], bfr[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int mb = wm * 64 + 16 * i + gr;
                af[i][0] = As[buf][ks + gc][mb];
                af[i][1] = As[buf][ks + gc][mb + 8];
                af[i][2] = As[buf][ks + gc + 4][mb];
                af[i][3] = As[buf][ks + gc + 4][mb + 8];
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int nb = wn * 32 + 8 * j + gr;
                bfr[j][0] = Bs[buf][ks + gc][nb];
                bfr[j][1] = Bs[buf][ks + gc + 4][nb];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) mma_16x8x8_tf32(acc[i][j], af[i], bfr[j]);
        }
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t m = m0 + wm * 64 + 16 * i + gr + 8 * h;
            if (m >= m1) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int64_t n = n0 + wn * 32 + 8 * j + 2 * gc + e;
                    if (n >= g.N) continue;
                    const float v = acc[i][j][2 * h + e];
                    float* c = Cg + m * g.ldc + n;
                    if (g.trans_a) atomicAdd(c, v);
                    else *c = g.accumulate ? *c + v : v;
                }
        }
}

// C_g = 0 for every group (the reduction form's partial sums are added into it)
__global__ void __launch_bounds__(256)
zero_groups_kernel(float* C, int64_t ldc, int64_t M, int64_t N, const int32_t* gmem, int64_t c_group_stride) {
    const int grp = blockIdx.y;
    const int64_t w = gmem ? gmem[grp] : grp;
    float* Cg = C + w * c_group_stride;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < M * N; i += (int64_t)gridDim.x * blockDim.x)
        Cg[(i / N) * ldc + i % N] = 0.f;
}

unsigned grid_rows(int64_t rows, int per_block) {
    const int64_t want = cdiv(rows > 0 ? rows : 1, per_block);
    return (unsigned)(want < 148 * 16 ? want : 148 * 16);
}

}  // namespace

cudaError_t launch_combine_bwd(const void* dout, const void* o_p, const int32_t* row_of, const float* gate,
                               int64_t n_tok, int K, int HD, int64_t n_rows, int dt, void* do_p, float* dgate,
                               void* err, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    if (dt == MOM_BF16)
        combine_bwd_kernel<bf16><<<grid_rows(n_tok, 8), 256, 0, st>>>((const bf16*)dout, (const bf16*)o_p, row_of, gate,
                                                                     n_tok, K, HD, n_rows, (bf16*)do_p, dgate, err);
    else
        combine_bwd_kernel<float><<<grid_rows(n_tok, 8), 256, 0, st>>>((const float*)dout, (const float*)o_p, row_of,
                                                                      gate, n_tok, K, HD, n_rows, (float*)do_p, dgate,
                                                                      err);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_router_bwd(const int32_t* idx, const float* gate, const float* dgate, int64_t n_tok, int K, int M,
                              float* dlogits, void* err, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    router_bwd_kernel<<<grid_rows(n_tok, 256), 256, 0, st>>>(idx, gate, dgate, n_tok, K, M, dlogits, err);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_rows_sum(const float* src, int64_t n_src, const int32_t* row_of, int K, const float* base,
                            int64_t n_tok, int W, float* dst, void* err, cudaStream_t st) {
    if (n_tok == 0) return cudaSuccess;
    rows_sum_kernel<<<grid_rows(n_tok, 8), 256, 0, st>>>(src, n_src, row_of, K, base, n_tok, W, dst, err);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_l2norm_bwd(const void* y, const float* dy, const float* nrm, int64_t rows, int H, int d, int dt,
                              float* dz, int64_t ldz, int64_t col0, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (dt == MOM_BF16)
        l2norm_bwd_kernel<bf16><<<grid_rows(rows * H, 8), 256, 0, st>>>((const bf16*)y, dy, nrm, rows, H, d, dz, ldz, col0);
    else
        l2norm_bwd_kernel<float><<<grid_rows(rows * H, 8), 256, 0, st>>>((const float*)y, dy, nrm, rows, H, d, dz, ldz,
                                                                        col0);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gates_bwd(const float* beta, const float* la, const float* dbeta, const float* dla, const float* A,
                             const int32_t* goff, int n_groups, int64_t n, int H, float* dz, int64_t ldz,
                             int64_t col_b, int64_t col_a, float* dala, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    gates_bwd_kernel<<<grid_rows(n * H, 256), 256, 0, st>>>(beta, la, dbeta, dla, A, goff, n_groups, n, H, dz, ldz,
                                                            col_b, col_a, dala);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_col_sums(const float* a, int64_t rows, int64_t lda, int64_t C, const int32_t* goff, int n_groups,
                            float* out, cudaStream_t st) {
    if (C == 0 || n_groups == 0) return cudaSuccess;
    col_sums_kernel<<<grid_rows((int64_t)n_groups * C, 8), 256, 0, st>>>(a, rows, lda, C, goff, n_groups, out);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gemm_grouped(int trans_a, const float* A, int64_t lda, const void* B, int64_t ldb, int dt,
                                const int32_t* b_rows, int64_t n_b_rows, float* C, int64_t ldc, int64_t M, int64_t N,
                                int64_t K, int64_t total_rows, const int32_t* goff, const int32_t* gmem, int n_groups,
                                int64_t b_group_stride, int64_t c_group_stride, int accumulate, void* err,
                                cudaStream_t st) {
    if (n_groups == 0 || N == 0) return cudaSuccess;
    GemmArgs g{trans_a, A, lda, B, ldb, b_rows, C, ldc, M, N, K, goff, gmem, n_groups, b_group_stride,
               c_group_stride, accumulate, n_b_rows, err, 1};
    dim3 grid;
    if (!trans_a) {
        grid = dim3((unsigned)cdiv(N, GBN), (unsigned)(cdiv(total_rows, GBM) + n_groups), 1);
    } else {
        // split each group's reduction until there are ~4 CTAs per SM
        const int64_t tiles = cdiv(N, GBN) * cdiv(M, GBM) * n_groups;
        int64_t sp = cdiv(148 * 4, tiles);
        g.splits = (int)(sp < 1 ? 1 : sp > 64 ? 64 : sp);
        grid = dim3((unsigned)cdiv(N, GBN), (unsigned)cdiv(M, GBM), (unsigned)(n_groups * g.splits));
        if (!accumulate) {
            zero_groups_kernel<<<dim3((unsigned)grid_rows(M * N, 256), (unsigned)n_groups), 256, 0, st>>>(
                C, ldc, M, N, gmem, c_group_stride);
            count_launches(1);
        }
    }
    if (dt == MOM_BF16) {
        static unsigned long long optin_done = 0;
        cudaError_t e = smem_optin((const void*)gemm_grouped_tf32_kernel, (int)TF32_SMEM, &optin_done);
        if (e != cudaSuccess) return e;
        gemm_grouped_tf32_kernel<<<grid, 256, TF32_SMEM, st>>>(g);
    } else {
        gemm_grouped_kernel<float><<<grid, 256, 0, st>>>(g);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace mom
