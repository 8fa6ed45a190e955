// Reordering of routed (token, slot) pairs into contiguous per-memory
// segments ("MoM: Mixture-of-Memories Fixes Linear Attention Recall",
// Solving scatter-gather without new kernels): a stable counting sort by
// memory, in four short launches that never leave the device:
//
//   count  : per tile of TILE tokens, how many pairs go to each memory
//   scan   : one CTA turns the (memory-major) tile counts into each tile's
//            first row per memory, and writes mem_offset
//   scatter: per tile, each pair's rank among the tile's pairs of the same
//            memory (warp ballots, token order) -> perm_token / row_of
//   bounds : per (memory, sequence), binary search of the memory's rows
//            (ascending tokens) for the sequence start -> seg_cu
//
// When the tile-count table is small (M x tiles <= FUSED_MAX_TABLE) the four
// steps run as ONE cooperative launch instead: counts, a grid barrier, then
// every CTA scans the whole table in shared memory (it is a few KB) and
// scatters its own tiles, and the (memory, sequence) bounds come from the
// scanned table plus a count over at most one tile -- no binary search.
//
// Counts stay on the device: later kernels read mem_offset / seg_cu
// themselves, so no host synchronisation is needed anywhere in the layer.
#include "common.cuh"
#include "kernels.h"

namespace mom {

static constexpr int TILE = 256;   // tokens per CTA (one thread per token)

// A token's k memories as a bit set; invalid or repeated indices are
// recorded and dropped.
__device__ __forceinline__ uint32_t token_mem_bits(const int32_t* idx, int64_t t, int K, int M, void* ws) {
    uint32_t bits = 0;
    for (int j = 0; j < K; ++j) {
        int m = idx[t * K + j];
        if (m < 0 || m >= M || ((bits >> m) & 1u)) {
            record_error(ws, MOM_DEVERR_MEM_INDEX, t);
            continue;
        }
        bits |= 1u << m;
    }
    return bits;
}

__global__ void __launch_bounds__(TILE)
permute_count_kernel(const int32_t* __restrict__ idx, int64_t n_tok, int K, int M, int n_tiles,
                     int32_t* __restrict__ tile_cnt, void* ws) {
    __shared__ int cnt[MOM_MAX_MEM];
    if (threadIdx.x < MOM_MAX_MEM) cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t t = (int64_t)blockIdx.x * TILE + threadIdx.x;
    if (t < n_tok) {
        uint32_t bits = token_mem_bits(idx, t, K, M, ws);
        while (bits) {
            int m = __ffs(bits) - 1;
            bits &= bits - 1;
            atomicAdd(&cnt[m], 1);
        }
    }
    __syncthreads();
    if (threadIdx.x < M) tile_cnt[(int64_t)threadIdx.x * n_tiles + blockIdx.x] = cnt[threadIdx.x];
}

// Exclusive scan over tile_cnt in memory-major order (one CTA of 1024).
__global__ void __launch_bounds__(1024)
permute_scan_kernel(const int32_t* __restrict__ tile_cnt, int64_t total, int n_tiles, int M,
                    int32_t* __restrict__ tile_base, int32_t* __restrict__ mem_offset) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t base = 0; base < total; base += 1024) {
        const int64_t i = base + threadIdx.x;
        int32_t v = i < total ? tile_cnt[i] : 0;
        int32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int32_t w = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int32_t n = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += n;
            }
            warp_tot[lane] = w;   // inclusive over warps
        }
        __syncthreads();
        const int32_t excl = carry + (warp ? warp_tot[warp - 1] : 0) + incl - v;
        if (i < total) {
            tile_base[i] = excl;
            if (i % n_tiles == 0) mem_offset[i / n_tiles] = excl;
        }
        __syncthreads();
        if (threadIdx.x == 0) carry += warp_tot[31];
        __syncthreads();
    }
    if (threadIdx.x == 0) mem_offset[M] = carry;
}

__global__ void __launch_bounds__(TILE)
permute_scatter_kernel(const int32_t* __restrict__ idx, int64_t n_tok, int K, int M, int n_tiles,
                       const int32_t* __restrict__ tile_base, int32_t* __restrict__ perm_token,
                       int32_t* __restrict__ row_of) {
    __shared__ int32_t warp_cnt[TILE / 32][MOM_MAX_MEM];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t = (int64_t)blockIdx.x * TILE + threadIdx.x;
    const bool live = t < n_tok;
    // errors were recorded by the count pass; here invalid entries are just skipped
    uint32_t bits = live ? token_mem_bits(idx, t, K, M, nullptr) : 0u;
    const uint32_t lt = (1u << lane) - 1u;
    int32_t my_rank[MOM_MAX_MEM];
#pragma unroll
    for (int m = 0; m < MOM_MAX_MEM; ++m) {
        if (m < M) {
            uint32_t b = __ballot_sync(0xffffffffu, (bits >> m) & 1u);
            my_rank[m] = __popc(b & lt);
            if (lane == 0) warp_cnt[warp][m] = __popc(b);
        }
    }
    __syncthreads();
    if (!live) return;
    for (int j = 0; j < K; ++j) {
        const int m = idx[t * K + j];
        if (m < 0 || m >= M || !((bits >> m) & 1u)) { row_of[t * K + j] = -1; continue; }
        bits &= ~(1u << m);   // a repeated index is only placed once
        int32_t r = tile_base[(int64_t)m * n_tiles + blockIdx.x];
        for (int w = 0; w < warp; ++w) r += warp_cnt[w][m];
        int32_t rk = 0;
#pragma unroll
        for (int mm = 0; mm < MOM_MAX_MEM; ++mm) if (mm == m) rk = my_rank[mm];
        r += rk;
        perm_token[r] = (int32_t)t;
        row_of[t * K + j] = r;
    }
}

// seg_cu[m*S + s] = mem_offset[m] + #{rows of memory m with token < cu[s]}.
__global__ void permute_bounds_kernel(const int32_t* __restrict__ perm_token, const int32_t* __restrict__ mem_offset,
                                      const int32_t* __restrict__ cu_seqlens, int64_t n_tok, int M, int S,
                                      int32_t* __restrict__ seg_cu) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i > (int64_t)M * S) return;
    if (i == (int64_t)M * S) { seg_cu[i] = mem_offset[M]; return; }
    const int m = (int)(i / S), s = (int)(i % S);
    const int64_t start = cu_seqlens ? cu_seqlens[s] : (s == 0 ? 0 : n_tok);
    int32_t lo = mem_offset[m], hi = mem_offset[m + 1];
    while (lo < hi) {                       // first row with token >= start
        int32_t mid = lo + ((hi - lo) >> 1);
        if (perm_token[mid] < start) lo = mid + 1; else hi = mid;
    }
    seg_cu[i] = lo;
}

// ----------------------------------------------------------- fused path --
static constexpr int FUSED_MAX_TABLE = 8192;       // M x tiles entries scanned in shared memory
static constexpr long long kBarrierCycles = 4000000000LL;

// Grid-wide barrier for a cooperative launch (all CTAs co-resident): one
// arrival per CTA on a zeroed counter, bounded spin.  False on timeout
// (recorded as MOM_DEVERR_TIMEOUT).
__device__ bool grid_barrier(unsigned* counter, unsigned target, void* ws, int* flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(counter, 1u);
        const long long t0 = clock64();
        int ok = 1;
        for (;;) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
            if (v >= target) break;
            if (clock64() - t0 > kBarrierCycles) { record_error(ws, MOM_DEVERR_TIMEOUT, -1); ok = 0; break; }
        }
        *flag = ok;
    }
    __syncthreads();
    return *flag != 0;
}

__global__ void __launch_bounds__(TILE)
permute_fused_kernel(const int32_t* __restrict__ idx, int64_t n_tok, int K, int M, int n_tiles,
                     const int32_t* __restrict__ cu_seqlens, int S, int32_t* __restrict__ tile_cnt,
                     unsigned* __restrict__ counter, int32_t* __restrict__ perm_token, int32_t* __restrict__ row_of,
                     int32_t* __restrict__ mem_offset, int32_t* __restrict__ seg_cu, void* ws) {
    extern __shared__ int32_t tab[];                   // M x n_tiles, memory-major
    __shared__ int cnt[MOM_MAX_MEM];
    __shared__ int32_t warp_cnt[TILE / 32][MOM_MAX_MEM];
    __shared__ int32_t part[TILE];
    __shared__ int flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // ---- 1. per-tile counts
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        if (tid < MOM_MAX_MEM) cnt[tid] = 0;
        __syncthreads();
        const int64_t t = (int64_t)tile * TILE + tid;
        if (t < n_tok) {
            uint32_t bits = token_mem_bits(idx, t, K, M, ws);
            while (bits) {
                const int m = __ffs(bits) - 1;
                bits &= bits - 1;
                atomicAdd(&cnt[m], 1);
            }
        }
        __syncthreads();
        if (tid < M) tile_cnt[(int64_t)tid * n_tiles + tile] = cnt[tid];
    }
    if (!grid_barrier(counter, gridDim.x, ws, &flag)) return;
    // ---- 2. exclusive scan of the whole table, memory-major (every CTA)
    const int L = M * n_tiles;
    const int per = (L + TILE - 1) / TILE;
    const int b0 = tid * per, b1 = b0 + per < L ? b0 + per : L;
    int32_t sum = 0;
    for (int i = b0; i < b1; ++i) {
        const int32_t v = __ldcg(tile_cnt + i);
        tab[i] = v;
        sum += v;
    }
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) part[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = lane < TILE / 32 ? part[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        if (lane < TILE / 32) part[TILE / 32 + lane] = w;        // inclusive over warps
    }
    __syncthreads();
    int32_t run = (warp ? part[TILE / 32 + warp - 1] : 0) + incl - sum;
    for (int i = b0; i < b1; ++i) {
        const int32_t v = tab[i];
        tab[i] = run;
        run += v;
    }
    const int32_t total = part[TILE / 32 + TILE / 32 - 1];
    __syncthreads();
    if (blockIdx.x == 0) {
        if (tid < M) mem_offset[tid] = tab[tid * n_tiles];
        if (tid == 0) mem_offset[M] = total;
    }
    // ---- 3. scatter this CTA's tiles (stable: token order inside a memory)
    const uint32_t lt = (1u << lane) - 1u;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int64_t t = (int64_t)tile * TILE + tid;
        const bool live = t < n_tok;
        uint32_t bits = live ? token_mem_bits(idx, t, K, M, nullptr) : 0u;
        int32_t my_rank[MOM_MAX_MEM];
#pragma unroll
        for (int m = 0; m < MOM_MAX_MEM; ++m) {
            if (m < M) {
                const uint32_t bl = __ballot_sync(0xffffffffu, (bits >> m) & 1u);
                my_rank[m] = __popc(bl & lt);
                if (lane == 0) warp_cnt[warp][m] = __popc(bl);
            }
        }
        __syncthreads();
        if (live) {
            for (int j = 0; j < K; ++j) {
                const int m = idx[t * K + j];
                if (m < 0 || m >= M || !((bits >> m) & 1u)) { row_of[t * K + j] = -1; continue; }
                bits &= ~(1u << m);
                int32_t r = tab[m * n_tiles + tile];
                for (int w = 0; w < warp; ++w) r += warp_cnt[w][m];
                int32_t rk = 0;
#pragma unroll
                for (int mm = 0; mm < MOM_MAX_MEM; ++mm) if (mm == m) rk = my_rank[mm];
                perm_token[r + rk] = (int32_t)t;
                row_of[t * K + j] = r + rk;
            }
        }
        __syncthreads();
    }
    // ---- 4. seg_cu[m S + s] = first row of memory m with token >= cu[s]:
    // the scanned base of cu[s]'s tile plus a count inside that tile
    for (int pr = blockIdx.x * (TILE / 32) + warp; pr <= M * S; pr += gridDim.x * (TILE / 32)) {
        if (pr == M * S) {
            if (lane == 0) seg_cu[pr] = total;
            continue;
        }
        const int m = pr / S, s = pr % S;
        const int64_t start = cu_seqlens ? cu_seqlens[s] : (s == 0 ? 0 : n_tok);
        const int tile = (int)(start / TILE);
        int32_t base;
        if (tile < n_tiles) base = tab[m * n_tiles + tile];
        else base = m + 1 < M ? tab[(m + 1) * n_tiles] : total;
        int c = 0;
        for (int q = lane; q < TILE; q += 32) {
            const int64_t t = (int64_t)tile * TILE + q;
            if (t < start && t < n_tok) c += (token_mem_bits(idx, t, K, M, nullptr) >> m) & 1u;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) seg_cu[pr] = base + c;
    }
}

static int fused_grid(int n_tiles, size_t smem) {
    static int dev_cached = -1, max_blocks = 0, coop = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev != dev_cached) {
        int sms = 0, per_sm = 0;
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_fused_kernel, TILE,
                                                          FUSED_MAX_TABLE * sizeof(int32_t)) != cudaSuccess)
            per_sm = 0;
        max_blocks = sms * per_sm;
        dev_cached = dev;
    }
    (void)smem;
    if (!coop || max_blocks <= 0) return 0;
    return n_tiles < max_blocks ? n_tiles : max_blocks;
}

size_t permute_scratch_bytes(int64_t n_tok, int M) {
    const int64_t n_tiles = cdiv(n_tok > 0 ? n_tok : 1, TILE);
    return 2 * (size_t)(M * n_tiles) * sizeof(int32_t) + 256;
}

cudaError_t launch_permute(const int32_t* idx, int64_t n_tok, int K, int M, const int32_t* cu_seqlens, int S,
                           int32_t* perm_token, int32_t* row_of, int32_t* mem_offset, int32_t* seg_cu,
                           void* ws, void* scratch, cudaStream_t st) {
    const int n_tiles = (int)cdiv(n_tok > 0 ? n_tok : 1, TILE);
    int32_t* tile_cnt = reinterpret_cast<int32_t*>(scratch);
    int32_t* tile_base = tile_cnt + (size_t)M * n_tiles;
    if ((int64_t)M * n_tiles <= FUSED_MAX_TABLE) {
        const size_t smem = (size_t)M * n_tiles * sizeof(int32_t);
        const int grid = fused_grid(n_tiles, smem);
        if (grid > 0) {
            // the barrier counter sits after both tables, in the scratch's slack
            unsigned* counter = reinterpret_cast<unsigned*>(tile_base + (size_t)M * n_tiles);
            cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(unsigned), st);
            if (e != cudaSuccess) return e;
            void* args[] = {(void*)&idx, (void*)&n_tok, (void*)&K, (void*)&M, (void*)&n_tiles, (void*)&cu_seqlens,
                            (void*)&S, (void*)&tile_cnt, (void*)&counter, (void*)&perm_token, (void*)&row_of,
                            (void*)&mem_offset, (void*)&seg_cu, (void*)&ws};
            e = cudaLaunchCooperativeKernel((const void*)permute_fused_kernel, dim3(grid), dim3(TILE), args, smem, st);
            count_launches(1);
            return e;
        }
    }
    if (n_tok > 0)
        permute_count_kernel<<<n_tiles, TILE, 0, st>>>(idx, n_tok, K, M, n_tiles, tile_cnt, ws);
    else
        cudaMemsetAsync(tile_cnt, 0, sizeof(int32_t) * (size_t)M * n_tiles, st);
    permute_scan_kernel<<<1, 1024, 0, st>>>(tile_cnt, (int64_t)M * n_tiles, n_tiles, M, tile_base, mem_offset);
    if (n_tok > 0)
        permute_scatter_kernel<<<n_tiles, TILE, 0, st>>>(idx, n_tok, K, M, n_tiles, tile_base, perm_token, row_of);
    const int64_t nb = (int64_t)M * S + 1;
    permute_bounds_kernel<<<(int)cdiv(nb, 256), 256, 0, st>>>(perm_token, mem_offset, cu_seqlens, n_tok, M, S, seg_cu);
    count_launches(n_tok > 0 ? 4 : 2);
    return cudaGetLastError();
}

}  // namespace mom
