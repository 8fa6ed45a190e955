// mom_permute_noalloc: the reordering of mom_permute for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a scratch buffer: a plug-in running
// inside a host engine that hands out all device memory from its own fixed
// pool (and forbids raw cudaMalloc), or a latency-critical serving loop
// where cudaMalloc / cudaFree are off limits because they can block the
// host and synchronise the device.  This entry point needs no workspace:
// the counting sort's per-tile counts live in the array below, which is part
// of the library image, so every GPU that loads the library holds it until
// the process exits.
//
// The array is shared by every call on a device and keeps whatever the last
// call left in it.  Each call clears the part that must start at zero (the
// error record) and overwrites the tile counts it reads.  Two calls whose
// kernels overlap on the GPU (different streams without ordering, or
// different host threads) race on it and may produce wrong results; order
// them on one stream.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

// Error record (MOM_WS_HEADER_BYTES) followed by the tile counts for the
// largest supported problem: MOM_PERMUTE_NOALLOC_MAX_TOKENS tokens, 32
// memories.
constexpr size_t kScratchBytes =
    MOM_WS_HEADER_BYTES + 2 * (size_t)MOM_MAX_MEM * (MOM_PERMUTE_NOALLOC_MAX_TOKENS / 256) * 4 + 256;

static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
// Per device: the CUDA context the address was looked up in, and the address.
// A device address belongs to one context; a host engine may run its own
// (non-primary) context on a device, and a context can be destroyed and
// replaced (cudaDeviceReset), so the cache is keyed on the context too.
CUcontext g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_addr[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, found through the runtime (no link-time
// libcuda dependency).
PFN_cuCtxGetCurrent_v4000 ctx_get_current_fn() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    });
    return fn;
}

// Device address of g_permute_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so the address must come
// from the runtime; it is looked up on the first call in each context of a
// device and cached for as long as that context stays current there.
mom_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOM_ERR_CUDA;
    auto get_ctx = ctx_get_current_fn();
    if (!get_ctx) return MOM_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return MOM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (ctx == nullptr || g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
        // the lookup also makes the runtime create the device's primary
        // context when none is current yet
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return MOM_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MOM_ERR_CUDA;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_addr[dev];
    return MOM_OK;
}

}  // namespace

extern "C" mom_status mom_permute_noalloc(const int32_t* topk_idx, int64_t n_tok, int top_k, int n_mem,
                                          const int32_t* cu_seqlens, int n_seq,
                                          int32_t* perm_token, int32_t* row_of, int32_t* mem_offset,
                                          int32_t* seg_cu, int32_t* status_out, void* stream) {
    if (n_tok < 0 || top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM || n_seq < 1) return MOM_ERR_ARG;
    if (!cu_seqlens && n_seq != 1) return MOM_ERR_ARG;
    if (!mem_offset || !seg_cu) return MOM_ERR_ARG;
    if (n_tok > 0 && (!topk_idx || !perm_token || !row_of)) return MOM_ERR_ARG;
    // larger problems than the static array holds are refused, not truncated
    if (n_tok > MOM_PERMUTE_NOALLOC_MAX_TOKENS) return MOM_ERR_UNSUPPORTED;
    if (MOM_WS_HEADER_BYTES + mom::permute_scratch_bytes(n_tok, n_mem) > kScratchBytes) return MOM_ERR_UNSUPPORTED;

    void* base = nullptr;
    mom_status s = scratch_address(&base);
    if (s != MOM_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the error record must start clear; the tile counts are rewritten below
    if (cudaMemsetAsync(base, 0, MOM_WS_HEADER_BYTES, st) != cudaSuccess) return MOM_ERR_CUDA;
    cudaError_t e = mom::launch_permute(topk_idx, n_tok, top_k, n_mem, cu_seqlens, n_seq, perm_token, row_of,
                                        mem_offset, seg_cu, base,
                                        static_cast<char*>(base) + MOM_WS_HEADER_BYTES, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    if (status_out &&
        cudaMemcpyAsync(status_out, base, 2 * sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return MOM_ERR_CUDA;
    return MOM_OK;
}
