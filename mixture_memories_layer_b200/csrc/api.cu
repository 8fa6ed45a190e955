// The C ABI of mom.h: argument validation, workspace carving and dispatch.
// Nothing here computes; every step of the layer runs in the kernels.
#include <string.h>

#include <atomic>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

using namespace mom;

static std::atomic<uint64_t> g_launches{0};
void mom::count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

cudaError_t mom::smem_optin(const void* func, int bytes, unsigned long long* done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
    if (bit && (__atomic_load_n(done, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) __atomic_fetch_or(done, bit, __ATOMIC_RELEASE);
    return e;
}

namespace {

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
inline size_t esize(int dt) { return dt == MOM_BF16 ? 2 : 4; }
inline bool dt_ok(int dt) { return dt == MOM_F32 || dt == MOM_BF16; }
inline bool head_dim_ok(int d) { return d == 64 || d == 128 || d == 256; }
inline mom_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOM_OK : MOM_ERR_CUDA; }

// A side stream of the library for work inside one call that does not
// depend on the rest of it (the decode step's gate projection beside its
// router and reordering): forked from the caller's stream by an event and
// joined back by another before anything reads its results, so the call as
// a whole stays ordered on the caller's stream.  One per (device, context):
// a stream belongs to the context it was made in.
struct Side {
    CUcontext ctx = nullptr;
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kSideDevices = 64;
std::mutex g_side_mutex;
Side g_side[kSideDevices];

PFN_cuCtxGetCurrent_v4000 current_ctx_fn() {
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

// The side stream of the current device and context (created on first use),
// or nullptr when none can be had: the caller then runs everything on its
// own stream.
const Side* side_stream() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSideDevices) return nullptr;
    auto get_ctx = current_ctx_fn();
    CUcontext ctx = nullptr;
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
    std::lock_guard<std::mutex> lock(g_side_mutex);
    Side& sd = g_side[dev];
    if (sd.s != nullptr && sd.ctx == ctx) return &sd;
    Side fresh;
    fresh.ctx = ctx;
    if (cudaStreamCreateWithFlags(&fresh.s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&fresh.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&fresh.join, cudaEventDisableTiming) != cudaSuccess) {
        cudaStreamDestroy(fresh.s);
        return nullptr;
    }
    sd = fresh;        // a stream of a context no longer current is left to that context
    return &sd;
}

// The side stream forked from `st` (work queued there starts after what is
// already queued on `st`), or `st` itself when there is none.  Every fork is
// closed by join_side(st, side) before anything on `st` reads the side's
// results.
cudaStream_t fork_side(cudaStream_t st) {
    const Side* sd = side_stream();
    if (sd == nullptr) return st;
    if (cudaEventRecord(sd->fork, st) != cudaSuccess || cudaStreamWaitEvent(sd->s, sd->fork, 0) != cudaSuccess)
        return st;
    return sd->s;
}

cudaError_t join_side(cudaStream_t st, cudaStream_t side) {
    if (side == st) return cudaSuccess;
    const Side* sd = side_stream();
    if (sd == nullptr || sd->s != side) return cudaErrorInvalidValue;
    cudaError_t e = cudaEventRecord(sd->join, side);
    return e == cudaSuccess ? cudaStreamWaitEvent(st, sd->join, 0) : e;
}

}  // namespace

extern "C" {

const char* mom_status_string(mom_status s) {
    switch (s) {
        case MOM_OK: return "ok";
        case MOM_ERR_ARG: return "invalid argument";
        case MOM_ERR_UNSUPPORTED: return "unsupported shape or type";
        case MOM_ERR_CUDA: return "CUDA runtime or launch error";
        case MOM_ERR_DEVICE: return "a kernel recorded a data violation";
    }
    return "unknown status";
}

mom_status mom_get_error(const void* ws, int32_t* code, int32_t* info, void* stream) {
    if (ws == nullptr) return MOM_ERR_ARG;
    int32_t rec[2] = {0, 0};
    if (cudaMemcpyAsync(rec, ws, sizeof(rec), cudaMemcpyDeviceToHost, as_stream(stream)) != cudaSuccess)
        return MOM_ERR_CUDA;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MOM_ERR_CUDA;
    if (code) *code = rec[0];
    if (info) *info = rec[1];
    return rec[0] == MOM_DEVERR_NONE ? MOM_OK : MOM_ERR_DEVICE;
}

uint64_t mom_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

mom_status mom_clear_error(void* ws, void* stream) {
    if (ws == nullptr) return MOM_ERR_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, 8, as_stream(stream)));
}

// ------------------------------------------------------------------ router
mom_status mom_router_topk(const void* x, const void* w_r, const float* b_r, mom_dtype dt,
                           int64_t n_tok, int d_model, int n_mem, int top_k,
                           int32_t* topk_idx, float* topk_gate, float* logits, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || d_model <= 0 || d_model % 8 != 0) return MOM_ERR_ARG;
    if (top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    if (!x || !w_r || !topk_idx || !topk_gate || !al16(x) || !al16(w_r)) return MOM_ERR_ARG;
    return cuda_status(launch_router(x, w_r, b_r, dt, n_tok, d_model, n_mem, top_k, topk_idx, topk_gate,
                                     logits, as_stream(stream)));
}

// ----------------------------------------------------------------- permute
size_t mom_permute_workspace_size(int64_t n_tok, int top_k, int n_mem, int n_seq) {
    (void)top_k; (void)n_seq;
    return MOM_WS_HEADER_BYTES + up256(permute_scratch_bytes(n_tok, n_mem > 0 ? n_mem : 1));
}

mom_status mom_permute(const int32_t* topk_idx, int64_t n_tok, int top_k, int n_mem,
                       const int32_t* cu_seqlens, int n_seq,
                       int32_t* perm_token, int32_t* row_of, int32_t* mem_offset, int32_t* seg_cu,
                       void* ws, size_t ws_bytes, void* stream) {
    if (n_tok < 0 || top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM || n_seq < 1) return MOM_ERR_ARG;
    if (n_tok * top_k >= ((int64_t)1 << 31)) return MOM_ERR_UNSUPPORTED;
    if (!cu_seqlens && n_seq != 1) return MOM_ERR_ARG;
    if (!mem_offset || !seg_cu || !ws || ws_bytes < mom_permute_workspace_size(n_tok, top_k, n_mem, n_seq))
        return MOM_ERR_ARG;
    if (n_tok > 0 && (!topk_idx || !perm_token || !row_of)) return MOM_ERR_ARG;
    return cuda_status(launch_permute(topk_idx, n_tok, top_k, n_mem, cu_seqlens, n_seq, perm_token, row_of,
                                      mem_offset, seg_cu, ws, (char*)ws + MOM_WS_HEADER_BYTES,
                                      as_stream(stream)));
}

// ------------------------------------------------------------- projections
size_t mom_kv_proj_workspace_size(int64_t n_tok, int d_model, int H, int d, int n_mem, int top_k) {
    (void)n_tok; (void)d_model; (void)H; (void)d; (void)n_mem; (void)top_k;
    return MOM_WS_HEADER_BYTES;
}


mom_status mom_kv_proj_grouped(const void* x, const int32_t* perm_token, const int32_t* mem_offset,
                               const void* w_shared, const void* w_gate, const float* A, const float* b_a,
                               const void* w_kv, mom_dtype dt,
                               int64_t n_tok, int d_model, int H, int d, int n_mem, int top_k,
                               void* q, void* k_sh, void* v_sh, float* beta, float* log_alpha,
                               void* k_p, void* v_p, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || d_model <= 0 || d_model % 64 != 0) return MOM_ERR_ARG;
    if (H < 1 || H > MOM_MAX_HEADS || top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM) return MOM_ERR_ARG;
    if (!head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (n_tok * top_k >= ((int64_t)1 << 31)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < mom_kv_proj_workspace_size(n_tok, d_model, H, d, n_mem, top_k)) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {x, perm_token, mem_offset, w_shared, w_kv, q, k_sh, v_sh, k_p, v_p};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    // the gates are optional here (both NULL: the caller runs mom_gate_proj)
    const bool gates = beta || log_alpha;
    if (gates) {
        const void* gp[] = {w_gate, A, b_a, beta, log_alpha};
        for (const void* p : gp)
            if (!p || !al16(p)) return MOM_ERR_ARG;
    }
    ProjArgs a{x, perm_token, mem_offset, w_shared, w_kv, n_tok, d_model, H, d, n_mem, top_k,
               q, k_sh, v_sh, k_p, v_p, ws};
    cudaStream_t st = as_stream(stream);
    if (gates) {
        cudaError_t e = launch_gate_proj(x, w_gate, A, b_a, dt, n_tok, d_model, H, beta, log_alpha, ws, st);
        if (e != cudaSuccess) return MOM_ERR_CUDA;
    }
    return cuda_status(proj_tc_supported(a, dt) ? launch_proj_tc(a, st) : launch_proj_simt(a, dt, st));
}

mom_status mom_proj_shared(const void* x, const void* w_shared, mom_dtype dt, int64_t n_tok, int d_model,
                           int H, int d, void* q, void* k_sh, void* v_sh, float* q_norm, float* k_sh_norm,
                           void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || d_model <= 0 || d_model % 64 != 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (!head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {x, w_shared, q, k_sh, v_sh};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    ProjArgs a{x, nullptr, nullptr, w_shared, nullptr, n_tok, d_model, H, d, 1, 1,
               q, k_sh, v_sh, nullptr, nullptr, ws};
    a.parts = PROJ_SHARED;
    a.q_norm = q_norm;
    a.k_sh_norm = k_sh_norm;
    cudaStream_t st = as_stream(stream);
    return cuda_status(proj_tc_supported(a, dt) ? launch_proj_tc(a, st) : launch_proj_simt(a, dt, st));
}

mom_status mom_kv_proj_groups(const void* x, int64_t n_x, const int32_t* perm_token, int64_t n_rows,
                              const int32_t* group_offset, const int32_t* group_mem, int n_groups,
                              const void* w_kv, mom_dtype dt, int d_model, int H, int d, int n_mem,
                              void* k_p, void* v_p, float* k_norm, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_x < 0 || n_rows < 0 || d_model <= 0 || d_model % 64 != 0) return MOM_ERR_ARG;
    if (H < 1 || H > MOM_MAX_HEADS || n_mem < 1 || n_mem > MOM_MAX_MEM || n_groups < 0) return MOM_ERR_ARG;
    if (!head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (n_rows >= ((int64_t)1 << 31) || n_x >= ((int64_t)1 << 31)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_rows == 0 || n_groups == 0) return MOM_OK;
    if (n_x == 0) return MOM_ERR_ARG;
    const void* ptrs[] = {x, w_kv, k_p, v_p};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    if (!group_offset || !group_mem) return MOM_ERR_ARG;
    ProjArgs a{x, perm_token, group_offset, nullptr, w_kv, n_x, d_model, H, d, n_mem, 1,
               nullptr, nullptr, nullptr, k_p, v_p, ws};
    a.parts = PROJ_ROUTED;
    a.group_mem = group_mem;
    a.n_groups = n_groups;
    a.n_routed = n_rows;
    a.k_p_norm = k_norm;
    cudaStream_t st = as_stream(stream);
    return cuda_status(proj_tc_supported(a, dt) ? launch_proj_tc(a, st) : launch_proj_simt(a, dt, st));
}

mom_status mom_copy_rows(const void* src, int64_t n_src, int64_t src_stride, int64_t src_off,
                         const int32_t* idx, int64_t n_rows, int64_t row_bytes,
                         void* dst, int64_t dst_stride, int64_t dst_off, void* ws, size_t ws_bytes, void* stream) {
    if (n_src < 0 || n_rows < 0 || row_bytes < 0 || src_stride < 0 || dst_stride < 0 || src_off < 0 || dst_off < 0)
        return MOM_ERR_ARG;
    const int64_t al[] = {src_stride, src_off, row_bytes, dst_stride, dst_off};
    for (int64_t v : al)
        if (v % 16 != 0) return MOM_ERR_ARG;
    if (src_off + row_bytes > src_stride || dst_off + row_bytes > dst_stride) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_rows == 0 || row_bytes == 0) return MOM_OK;
    if (!src || !dst || !al16(src) || !al16(dst) || n_src == 0) return MOM_ERR_ARG;
    return cuda_status(launch_copy_rows(src, n_src, src_stride, src_off, idx, n_rows, row_bytes, dst, dst_stride,
                                        dst_off, ws, as_stream(stream)));
}

size_t mom_gate_proj_workspace_size(int64_t n_tok, int d_model, int H) {
    (void)n_tok; (void)d_model; (void)H;
    return MOM_WS_HEADER_BYTES;
}

mom_status mom_gate_proj(const void* x, const void* w_gate, const float* A, const float* b_a, mom_dtype dt,
                         int64_t n_tok, int d_model, int H, float* beta, float* log_alpha,
                         void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || d_model <= 0 || d_model % 8 != 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (!ws || ws_bytes < mom_gate_proj_workspace_size(n_tok, d_model, H)) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {x, w_gate, A, b_a, beta, log_alpha};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    return cuda_status(launch_gate_proj(x, w_gate, A, b_a, dt, n_tok, d_model, H, beta, log_alpha, ws,
                                        as_stream(stream)));
}

mom_status mom_mem_gate_proj(const void* x, const int32_t* perm_token, const int32_t* mem_offset,
                             const void* w_gate_mem, const float* A_mem, const float* b_a_mem, mom_dtype dt,
                             int64_t n_tok, int d_model, int H, int n_mem, int top_k,
                             float* beta_p, float* log_alpha_p, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || d_model <= 0 || d_model % 8 != 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {x, perm_token, mem_offset, w_gate_mem, A_mem, b_a_mem, beta_p, log_alpha_p};
    for (const void* p : ptrs)
        if (!p) return MOM_ERR_ARG;
    if (!al16(x) || !al16(w_gate_mem)) return MOM_ERR_ARG;
    return cuda_status(launch_mem_gate_proj(x, perm_token, mem_offset, w_gate_mem, A_mem, b_a_mem, dt, n_tok,
                                            n_tok * top_k, d_model, H, n_mem, beta_p, log_alpha_p, ws,
                                            as_stream(stream)));
}

mom_status mom_mem_gate_proj_groups(const void* x, int64_t n_x, const int32_t* perm_token, int64_t n_rows,
                                    const int32_t* group_offset, const int32_t* group_mem, int n_groups,
                                    const void* w_gate_mem, const float* A_mem, const float* b_a_mem, int n_mem,
                                    mom_dtype dt, int d_model, int H, float* beta_p, float* log_alpha_p, void* ws,
                                    size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_x < 0 || n_rows < 0 || d_model <= 0 || d_model % 8 != 0 || H < 1 || H > MOM_MAX_HEADS)
        return MOM_ERR_ARG;
    if (n_groups < 1 || n_groups > MOM_MAX_MEM || n_mem < 1) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_rows == 0) return MOM_OK;
    const void* ptrs[] = {x, group_offset, group_mem, w_gate_mem, A_mem, b_a_mem, beta_p, log_alpha_p};
    for (const void* p : ptrs)
        if (!p) return MOM_ERR_ARG;
    if (!perm_token && n_x < n_rows) return MOM_ERR_ARG;
    if (!al16(x) || !al16(w_gate_mem)) return MOM_ERR_ARG;
    return cuda_status(launch_mem_gate_proj(x, perm_token, group_offset, w_gate_mem, A_mem, b_a_mem, dt, n_x, n_rows,
                                            d_model, H, n_groups, beta_p, log_alpha_p, ws, as_stream(stream),
                                            group_mem, n_mem));
}

// --------------------------------------------------------- chunked GDN
size_t mom_gdn_workspace_size(int64_t n_rows, int n_seg, int H, int d, mom_dtype dt) {
    size_t extra = (dt == MOM_BF16 && head_dim_ok(d)) ? gdn_tc_ws_bytes(n_rows, n_seg, H, d) : 0;
    return MOM_WS_HEADER_BYTES + up256(extra);
}

static mom_status gdn_call(const void* q, const int32_t* qidx, const void* k, const void* v, const float* beta,
                           const float* log_alpha, const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                           int H, int d, float scale, mom_dtype dt, const float* h0, float* h_final, void* o,
                           void* ws, size_t ws_bytes, void* stream, int phase, int rule = MOM_RULE_GATED_DELTA,
                           int gates = MOM_GATES_BY_TOKEN) {
    if (!dt_ok(dt) || n_seg < 0 || n_rows < 0 || n_q_rows < 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (rule != MOM_RULE_GATED_DELTA && rule != MOM_RULE_GATED_LINEAR) return MOM_ERR_ARG;
    if (gates != MOM_GATES_BY_TOKEN && gates != MOM_GATES_BY_ROW) return MOM_ERR_ARG;
    if (!head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < mom_gdn_workspace_size(n_rows, n_seg, H, d, dt)) return MOM_ERR_ARG;
    if (n_seg == 0) return MOM_OK;
    if (!seg_cu) return MOM_ERR_ARG;
    if ((h0 && !al16(h0)) || (h_final && !al16(h_final))) return MOM_ERR_ARG;
    if (n_rows > 0) {
        const void* ptrs[] = {q, k, v, beta, log_alpha, o};
        for (const void* p : ptrs)
            if (!p || !al16(p)) return MOM_ERR_ARG;
    }
    GdnArgs a{q, qidx, k, v, beta, log_alpha, seg_cu, n_seg, n_rows, n_q_rows, H, d, scale,
              h0, h_final, o, ws, ws_bytes};
    a.phase = phase;
    a.rule = rule;
    a.gates_by_row = gates == MOM_GATES_BY_ROW;
    cudaStream_t st = as_stream(stream);
    if (gdn_tc_supported(a, dt)) return cuda_status(launch_gdn_tc(a, st));
    return cuda_status(launch_gdn_recurrent(a, dt, st));
}

mom_status mom_gdn_chunk_fwd(const void* q, const int32_t* qidx, const void* k, const void* v,
                             const float* beta, const float* log_alpha,
                             const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                             int H, int d, float scale, mom_dtype dt,
                             const float* h0, float* h_final, void* o,
                             void* ws, size_t ws_bytes, void* stream) {
    return gdn_call(q, qidx, k, v, beta, log_alpha, seg_cu, n_seg, n_rows, n_q_rows, H, d, scale, dt, h0, h_final, o,
                    ws, ws_bytes, stream, GDN_PREP | GDN_STATE);
}

mom_status mom_gdn_chunk_prep(const void* q, const int32_t* qidx, const void* k, const void* v,
                              const float* beta, const float* log_alpha,
                              const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                              int H, int d, float scale, mom_dtype dt,
                              const float* h0, float* h_final, void* o,
                              void* ws, size_t ws_bytes, void* stream) {
    return gdn_call(q, qidx, k, v, beta, log_alpha, seg_cu, n_seg, n_rows, n_q_rows, H, d, scale, dt, h0, h_final, o,
                    ws, ws_bytes, stream, GDN_PREP);
}

mom_status mom_gdn_chunk_state(const void* q, const int32_t* qidx, const void* k, const void* v,
                               const float* beta, const float* log_alpha,
                               const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                               int H, int d, float scale, mom_dtype dt,
                               const float* h0, float* h_final, void* o,
                               void* ws, size_t ws_bytes, void* stream) {
    return gdn_call(q, qidx, k, v, beta, log_alpha, seg_cu, n_seg, n_rows, n_q_rows, H, d, scale, dt, h0, h_final, o,
                    ws, ws_bytes, stream, GDN_STATE);
}

#define MOM_MEMORY_CALL(NAME, PHASE)                                                                       \
    mom_status NAME(const void* q, const int32_t* qidx, const void* k, const void* v, const float* beta,     \
                    const float* log_alpha, const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows, \
                    int H, int d, float scale, mom_dtype dt, mom_rule rule, mom_gates gates, const float* h0, \
                    float* h_final, void* o, void* ws, size_t ws_bytes, void* stream) {                      \
        return gdn_call(q, qidx, k, v, beta, log_alpha, seg_cu, n_seg, n_rows, n_q_rows, H, d, scale, dt, h0,  \
                        h_final, o, ws, ws_bytes, stream, PHASE, rule, gates);                               \
    }
MOM_MEMORY_CALL(mom_memory_chunk_fwd, GDN_PREP | GDN_STATE)
MOM_MEMORY_CALL(mom_memory_chunk_prep, GDN_PREP)
MOM_MEMORY_CALL(mom_memory_chunk_state, GDN_STATE)
#undef MOM_MEMORY_CALL

// ------------------------------------------------------- reverse pass
size_t mom_memory_chunk_bwd_workspace_size(int64_t n_rows, int n_seg, int H, int d) {
    if (n_rows < 0 || n_seg < 0 || H < 1 || !head_dim_ok(d)) return 0;
    return gdn_bwd_ws_bytes(n_rows, n_seg, H, d);
}

mom_status mom_memory_chunk_bwd(const void* q, const int32_t* qidx, const void* k, const void* v,
                                const float* beta, const float* log_alpha,
                                const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                                int H, int d, float scale, mom_dtype dt, mom_rule rule, mom_gates gates,
                                const float* h0, const void* d_o, const float* dh_final,
                                float* dq, float* dk, float* dv, float* dbeta, float* dlog_alpha, float* dh0,
                                void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_seg < 0 || n_rows < 0 || n_q_rows < 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (rule != MOM_RULE_GATED_DELTA && rule != MOM_RULE_GATED_LINEAR) return MOM_ERR_ARG;
    if (gates != MOM_GATES_BY_TOKEN && gates != MOM_GATES_BY_ROW) return MOM_ERR_ARG;
    if (!head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (n_rows >= ((int64_t)1 << 31)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < mom_memory_chunk_bwd_workspace_size(n_rows, n_seg, H, d)) return MOM_ERR_ARG;
    if (n_seg == 0) return MOM_OK;
    if (!seg_cu) return MOM_ERR_ARG;
    const void* opt[] = {h0, dh_final, dh0};
    for (const void* p : opt)
        if (p && !al16(p)) return MOM_ERR_ARG;
    if (n_rows > 0) {
        const void* ptrs[] = {q, k, v, beta, log_alpha, d_o, dq, dk, dv, dbeta, dlog_alpha};
        for (const void* p : ptrs)
            if (!p || !al16(p)) return MOM_ERR_ARG;
    }
    GdnBwdArgs a{q, qidx, k, v, beta, log_alpha, seg_cu, n_seg, n_rows, n_q_rows, H, d, scale, rule,
                 gates == MOM_GATES_BY_ROW ? 1 : 0, h0, d_o, dh_final, dq, dk, dv, dbeta, dlog_alpha, dh0, ws};
    return cuda_status(launch_gdn_bwd(a, dt, as_stream(stream)));
}

// --------------------------------------------------- backward pieces
mom_status mom_combine_bwd(const void* dout, const void* o_p, const int32_t* row_of, const float* gate,
                           int64_t n_tok, int top_k, int64_t n_rows, int H, int d, mom_dtype dt,
                           void* do_p, float* dgate, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || n_rows < 0 || top_k < 1 || H < 1 || d < 1) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {dout, o_p, row_of, gate, do_p, dgate};
    for (const void* p : ptrs)
        if (!p) return MOM_ERR_ARG;
    return cuda_status(launch_combine_bwd(dout, o_p, row_of, gate, n_tok, top_k, H * d, n_rows, dt, do_p, dgate, ws,
                                          as_stream(stream)));
}

mom_status mom_router_bwd(const int32_t* topk_idx, const float* gate, const float* dgate, int64_t n_tok,
                          int top_k, int n_mem, float* dlogits, void* ws, size_t ws_bytes, void* stream) {
    if (n_tok < 0 || top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    if (!topk_idx || !gate || !dgate || !dlogits) return MOM_ERR_ARG;
    return cuda_status(launch_router_bwd(topk_idx, gate, dgate, n_tok, top_k, n_mem, dlogits, ws, as_stream(stream)));
}

mom_status mom_rows_sum(const float* src, int64_t n_src, const int32_t* row_of, int top_k, const float* base,
                        int64_t n_tok, int W, float* dst, void* ws, size_t ws_bytes, void* stream) {
    if (n_src < 0 || n_tok < 0 || top_k < 1 || W < 0) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0 || W == 0) return MOM_OK;
    if (!src || !row_of || !dst) return MOM_ERR_ARG;
    return cuda_status(launch_rows_sum(src, n_src, row_of, top_k, base, n_tok, W, dst, ws, as_stream(stream)));
}

mom_status mom_l2norm_bwd(const void* y, const float* dy, const float* norm, int64_t rows, int H, int d,
                          mom_dtype dt, float* dz, int64_t ldz, int64_t col0, void* stream) {
    if (!dt_ok(dt) || rows < 0 || H < 1 || d < 1 || col0 < 0 || ldz < col0 + (int64_t)H * d) return MOM_ERR_ARG;
    if (rows == 0) return MOM_OK;
    if (!y || !dy || !norm || !dz) return MOM_ERR_ARG;
    return cuda_status(launch_l2norm_bwd(y, dy, norm, rows, H, d, dt, dz, ldz, col0, as_stream(stream)));
}

mom_status mom_gates_bwd(const float* beta, const float* log_alpha, const float* dbeta, const float* dlog_alpha,
                         const float* A, int64_t n, int H, float* dz, int64_t ldz, int64_t col_b, int64_t col_a,
                         float* dala, void* stream) {
    if (n < 0 || H < 1 || col_b < 0 || col_a < 0 || ldz < col_b + H || ldz < col_a + H) return MOM_ERR_ARG;
    if (n == 0) return MOM_OK;
    const void* ptrs[] = {beta, log_alpha, dbeta, dlog_alpha, A, dz, dala};
    for (const void* p : ptrs)
        if (!p) return MOM_ERR_ARG;
    return cuda_status(launch_gates_bwd(beta, log_alpha, dbeta, dlog_alpha, A, nullptr, 1, n, H, dz, ldz, col_b,
                                        col_a, dala, as_stream(stream)));
}

mom_status mom_gates_bwd_by_group(const float* beta, const float* log_alpha, const float* dbeta, const float* dlog_alpha,
                                  const float* A, const int32_t* group_offset, int n_groups, int64_t n, int H, float* dz,
                                  int64_t ldz, int64_t col_b, int64_t col_a, float* dala, void* stream) {
    if (n < 0 || H < 1 || n_groups < 1 || col_b < 0 || col_a < 0 || ldz < col_b + H || ldz < col_a + H)
        return MOM_ERR_ARG;
    if (n == 0) return MOM_OK;
    const void* ptrs[] = {beta, log_alpha, dbeta, dlog_alpha, A, group_offset, dz, dala};
    for (const void* p : ptrs)
        if (!p) return MOM_ERR_ARG;
    return cuda_status(launch_gates_bwd(beta, log_alpha, dbeta, dlog_alpha, A, group_offset, n_groups, n, H, dz, ldz,
                                        col_b, col_a, dala, as_stream(stream)));
}

mom_status mom_col_sums(const float* a, int64_t rows, int64_t lda, int64_t cols, float* out, void* stream) {
    if (rows < 0 || cols < 0 || lda < cols) return MOM_ERR_ARG;
    if (cols == 0) return MOM_OK;
    if (!out || (rows > 0 && !a)) return MOM_ERR_ARG;
    return cuda_status(launch_col_sums(a, rows, lda, cols, nullptr, 1, out, as_stream(stream)));
}

mom_status mom_col_sums_grouped(const float* a, int64_t rows, int64_t lda, int64_t cols, const int32_t* group_offset,
                                int n_groups, float* out, void* stream) {
    if (rows < 0 || cols < 0 || lda < cols || n_groups < 1) return MOM_ERR_ARG;
    if (cols == 0) return MOM_OK;
    if (!out || !group_offset || (rows > 0 && !a)) return MOM_ERR_ARG;
    return cuda_status(launch_col_sums(a, rows, lda, cols, group_offset, n_groups, out, as_stream(stream)));
}

mom_status mom_gemm_grouped(int trans_a, const float* A, int64_t lda, const void* B, int64_t ldb, mom_dtype dt,
                            const int32_t* b_rows, int64_t n_b_rows, float* C, int64_t ldc, int64_t M, int64_t N,
                            int64_t K, int64_t total_rows, const int32_t* group_offset, const int32_t* group_index,
                            int n_groups, int64_t b_group_stride, int64_t c_group_stride, int accumulate,
                            void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || (trans_a != 0 && trans_a != 1) || n_groups < 0 || N < 0 || M < 0 || K < 0 || total_rows < 0)
        return MOM_ERR_ARG;
    if (ldb < N || ldc < N || (trans_a ? lda < M : lda < K)) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_groups == 0 || N == 0 || (trans_a && M == 0)) return MOM_OK;
    if (!A || !B || !C || !group_offset) return MOM_ERR_ARG;
    return cuda_status(launch_gemm_grouped(trans_a, A, lda, B, ldb, dt, b_rows, n_b_rows, C, ldc, M, N, K, total_rows,
                                           group_offset, group_index, n_groups, b_group_stride, c_group_stride,
                                           accumulate, ws, as_stream(stream)));
}

// ------------------------------------------------------------------- block
mom_status mom_block_proj(const void* x, const int32_t* perm_token, const int32_t* mem_offset,
                          const void* w_shared4, const void* w_kv, mom_dtype dt,
                          int64_t n_tok, int d_model, int H, int d, int n_mem, int top_k,
                          void* q, void* k_sh, void* v_sh, void* g, void* k_p, void* v_p,
                          void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || d_model <= 0 || d_model % 64 != 0) return MOM_ERR_ARG;
    if (H < 1 || H > MOM_MAX_HEADS || top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM) return MOM_ERR_ARG;
    if (!head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (n_tok * top_k >= ((int64_t)1 << 31)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {x, perm_token, mem_offset, w_shared4, w_kv, q, k_sh, v_sh, g, k_p, v_p};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    ProjArgs a{x, perm_token, mem_offset, w_shared4, w_kv, n_tok, d_model, H, d, n_mem, top_k,
               q, k_sh, v_sh, k_p, v_p, ws};
    a.raw = 1;
    a.g = g;
    if (!proj_tc_supported(a, dt)) return MOM_ERR_UNSUPPORTED;
    return cuda_status(launch_proj_tc(a, as_stream(stream)));
}

namespace {
mom_status conv_check(const mom_conv_problem& q, int channels, int head_dim) {
    if (q.n_rows < 0 || q.n_seg < 1 || q.seg_per_group < 1 || q.n_groups < 1) return MOM_ERR_ARG;
    if (q.l2norm != 0 && q.l2norm != 1) return MOM_ERR_ARG;
    if (q.l2norm && (head_dim < 8 || head_dim > 256 || (head_dim & (head_dim - 1)) != 0 || channels % head_dim != 0))
        return MOM_ERR_ARG;
    if (q.n_rows > 0 && (!q.z || !q.out || !q.seg_cu || !q.w || !al16(q.z) || !al16(q.out) || !al16(q.w) ||
                         q.z == q.out))
        return MOM_ERR_ARG;
    return MOM_OK;
}
}  // namespace

mom_status mom_short_conv_batch(const mom_conv_problem* problems, int n_problems, int channels, int width,
                                int head_dim, mom_dtype dt, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || !problems || n_problems < 1 || channels < 8 || channels % 8 != 0 || width < 1)
        return MOM_ERR_ARG;
    if (dt != MOM_BF16 || width > 4 || n_problems > 8) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    ConvProblem pr[8];
    int n = 0;
    for (int i = 0; i < n_problems; ++i) {
        const mom_conv_problem& q = problems[i];
        const mom_status e = conv_check(q, channels, head_dim);
        if (e != MOM_OK) return e;
        if (q.n_rows > 0)
            pr[n++] = ConvProblem{q.z, q.out, q.n_rows, q.seg_cu, q.n_seg, q.seg_per_group, q.n_groups, q.w, q.l2norm};
    }
    if (n == 0) return MOM_OK;
    return cuda_status(launch_short_conv(pr, n, channels, width, head_dim, ws, as_stream(stream)));
}

mom_status mom_short_conv(const void* z, int64_t n_rows, int channels, const int32_t* seg_cu, int n_seg,
                          int seg_per_group, int n_groups, const float* w, int width, int head_dim,
                          int l2norm, mom_dtype dt, void* out, void* ws, size_t ws_bytes, void* stream) {
    const mom_conv_problem q{z, out, n_rows, seg_cu, n_seg, seg_per_group, n_groups, w, l2norm};
    return mom_short_conv_batch(&q, 1, channels, width, head_dim, dt, ws, ws_bytes, stream);
}

mom_status mom_combine_norm_gate(const void* o_sh, const void* o_p, const int32_t* row_of,
                                 const float* topk_gate, const void* g, const float* w_norm, float eps,
                                 int64_t n_tok, int top_k, int H, int d, mom_dtype dt, void* out,
                                 void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || top_k < 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (d < 8 || d > 256 || (d & (d - 1)) != 0 || !(eps >= 0.f)) return MOM_ERR_ARG;
    if (dt != MOM_BF16) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {o_sh, g, w_norm, out};
    for (const void* p : ptrs)
        if (!p) return MOM_ERR_ARG;
    if (top_k > 0 && (!o_p || !row_of || !topk_gate || !al16(o_p))) return MOM_ERR_ARG;
    if (!al16(o_sh) || !al16(g) || !al16(out) || !al16(w_norm)) return MOM_ERR_ARG;
    return cuda_status(launch_combine_norm_gate(o_sh, o_p, row_of, topk_gate, g, w_norm, eps, n_tok, top_k, H, d,
                                                out, ws, as_stream(stream)));
}

mom_status mom_linear(const void* x, const void* w, mom_dtype dt, int64_t n_rows, int k_in, int n_out, void* y,
                      void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_rows < 0 || k_in <= 0 || n_out <= 0) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_rows == 0) return MOM_OK;
    if (!x || !w || !y || !al16(x) || !al16(w) || !al16(y)) return MOM_ERR_ARG;
    ProjArgs a{x, nullptr, nullptr, w, nullptr, n_rows, k_in, 1, n_out, 1, 1,
               y, nullptr, nullptr, nullptr, nullptr, ws};
    a.parts = PROJ_SHARED;
    a.plain_n = n_out;
    if (!proj_tc_supported(a, dt)) return MOM_ERR_UNSUPPORTED;
    return cuda_status(launch_proj_tc(a, as_stream(stream)));
}

// ----------------------------------------------------------------- combine
mom_status mom_combine_unpermute(const void* o_sh, const void* o_p, const int32_t* row_of,
                                 const float* topk_gate, int64_t n_tok, int top_k, int H, int d,
                                 mom_dtype dt, void* out, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || top_k < 1 || H < 1 || d < 8 || (H * d) % 8 != 0) return MOM_ERR_ARG;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    if (n_tok == 0) return MOM_OK;
    const void* ptrs[] = {o_sh, o_p, row_of, topk_gate, out};
    for (const void* p : ptrs)
        if (!p) return MOM_ERR_ARG;
    if (!al16(o_sh) || !al16(o_p) || !al16(out)) return MOM_ERR_ARG;
    return cuda_status(launch_combine(o_sh, o_p, row_of, topk_gate, n_tok, top_k, H, d, dt, out, ws,
                                      as_stream(stream)));
}

// ------------------------------------------------------------------ decode
namespace {
struct DecodeLayout {
    size_t idx, gate, perm, row_of, mem_off, seg_cu, q, k_sh, v_sh, beta, la, beta_p, la_p, k_p, v_p, perm_scratch,
        total;
};
DecodeLayout decode_layout(int B, int H, int d, int M, int K, int dt) {
    DecodeLayout L;
    size_t off = MOM_WS_HEADER_BYTES;
    auto take = [&](size_t bytes) { size_t o = off; off += up256(bytes); return o; };
    const size_t BK = (size_t)B * K, HD = (size_t)H * d;
    L.idx = take(BK * 4);
    L.gate = take(BK * 4);
    L.perm = take(BK * 4);
    L.row_of = take(BK * 4);
    L.mem_off = take((M + 1) * 4);
    L.seg_cu = take((M + 1) * 4);
    L.q = take((size_t)B * HD * esize(dt));
    L.k_sh = take((size_t)B * HD * esize(dt));
    L.v_sh = take((size_t)B * HD * esize(dt));
    L.beta = take((size_t)B * H * 4);
    L.la = take((size_t)B * H * 4);
    L.beta_p = take(BK * H * 4);
    L.la_p = take(BK * H * 4);
    L.k_p = take(BK * HD * esize(dt));
    L.v_p = take(BK * HD * esize(dt));
    L.perm_scratch = take(permute_scratch_bytes(B, M));
    L.total = off;
    return L;
}
}  // namespace

size_t mom_decode_workspace_size(int B, int d_model, int H, int d, int n_mem, int top_k) {
    (void)d_model;
    if (B < 0 || H < 1 || d < 1 || n_mem < 1 || top_k < 1) return 0;
    // sized for the larger element type so one workspace serves both modes
    return decode_layout(B, H, d, n_mem, top_k, MOM_F32).total;
}

mom_status mom_decode_step(const void* x, const mom_weights* w, int B, int d_model, int H, int d,
                           int n_mem, int top_k, float scale, mom_dtype dt,
                           float* state, void* out, int32_t* topk_idx,
                           void* ws, size_t ws_bytes, void* stream) {
    return mom_decode_step_rule(x, w, nullptr, B, d_model, H, d, n_mem, top_k, scale, dt, MOM_RULE_GATED_DELTA,
                                state, out, topk_idx, ws, ws_bytes, stream);
}

mom_status mom_decode_step_rule(const void* x, const mom_weights* w, const mom_memory_gates* mg,
                                int B, int d_model, int H, int d,
                                int n_mem, int top_k, float scale, mom_dtype dt, mom_rule rule,
                                float* state, void* out, int32_t* topk_idx,
                                void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || B < 0 || d_model <= 0 || d_model % 64 != 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (rule != MOM_RULE_GATED_DELTA && rule != MOM_RULE_GATED_LINEAR) return MOM_ERR_ARG;
    if (top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM || !w) return MOM_ERR_ARG;
    if (!head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < mom_decode_workspace_size(B, d_model, H, d, n_mem, top_k)) return MOM_ERR_ARG;
    if (B == 0) return MOM_OK;
    const void* ptrs[] = {x, w->w_r, w->w_shared, w->w_gate, w->A, w->b_a, w->w_kv, state, out};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    if (mg && (!mg->w_gate_mem || !al16(mg->w_gate_mem) || !mg->A_mem || !mg->b_a_mem)) return MOM_ERR_ARG;
    cudaStream_t st = as_stream(stream);
    const DecodeLayout L = decode_layout(B, H, d, n_mem, top_k, dt);
    char* base = reinterpret_cast<char*>(ws);
    int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(base + L.idx);
    float* gate = reinterpret_cast<float*>(base + L.gate);
    int32_t* perm = reinterpret_cast<int32_t*>(base + L.perm);
    int32_t* row_of = reinterpret_cast<int32_t*>(base + L.row_of);
    int32_t* mem_off = reinterpret_cast<int32_t*>(base + L.mem_off);
    int32_t* seg_cu = reinterpret_cast<int32_t*>(base + L.seg_cu);
    float* beta = reinterpret_cast<float*>(base + L.beta);
    float* la = reinterpret_cast<float*>(base + L.la);

    // the gates need no routing: on the side stream beside the router and the reordering
    const cudaStream_t ss = fork_side(st);
    cudaError_t e = launch_gate_proj(x, w->w_gate, w->A, w->b_a, dt, B, d_model, H, beta, la, ws, ss);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    e = launch_router(x, w->w_r, w->b_r, dt, B, d_model, n_mem, top_k, idx, gate, nullptr, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    e = launch_permute(idx, B, top_k, n_mem, nullptr, 1, perm, row_of, mem_off, seg_cu, ws,
                       base + L.perm_scratch, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    if (join_side(st, ss) != cudaSuccess) return MOM_ERR_CUDA;
    ProjArgs pa{x, perm, mem_off, w->w_shared, w->w_kv, B, d_model, H, d, n_mem, top_k,
                base + L.q, base + L.k_sh, base + L.v_sh, base + L.k_p, base + L.v_p, ws};
    e = proj_tc_supported(pa, dt) ? launch_proj_tc(pa, st) : launch_proj_simt(pa, dt, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    DecodeArgs da{base + L.q, base + L.k_sh, base + L.v_sh, base + L.k_p, base + L.v_p, beta, la, gate,
                  idx, row_of, B, H, d, n_mem, top_k, scale, state, out, ws};
    da.rule = rule;
    if (mg) {
        float* beta_p = reinterpret_cast<float*>(base + L.beta_p);
        float* la_p = reinterpret_cast<float*>(base + L.la_p);
        e = launch_mem_gate_proj(x, perm, mem_off, mg->w_gate_mem, mg->A_mem, mg->b_a_mem, dt, B, (int64_t)B * top_k,
                                 d_model, H, n_mem, beta_p, la_p, ws, st);
        if (e != cudaSuccess) return MOM_ERR_CUDA;
        da.beta_p = beta_p;
        da.log_alpha_p = la_p;
    }
    return cuda_status(launch_decode_state(da, dt, st));
}

// ------------------------------------------------------------ block decode
namespace {
struct BlockDecodeLayout {
    DecodeLayout base;
    size_t q_raw, k_sh_raw, v_sh_raw, g, k_p_raw, v_p_raw, comb, o_tilde, total;
};
BlockDecodeLayout block_decode_layout(int B, int H, int d, int M, int K) {
    BlockDecodeLayout L;
    L.base = decode_layout(B, H, d, M, K, MOM_F32);
    size_t off = L.base.total;
    auto take = [&](size_t bytes) { size_t o = off; off += up256(bytes); return o; };
    const size_t row = (size_t)H * d * 2, BK = (size_t)B * K;
    L.q_raw = take(B * row);
    L.k_sh_raw = take(B * row);
    L.v_sh_raw = take(B * row);
    L.g = take(B * row);
    L.k_p_raw = take(BK * row);
    L.v_p_raw = take(BK * row);
    L.comb = take(B * row);
    L.o_tilde = take(B * row);
    L.total = off;
    return L;
}
}  // namespace

size_t mom_block_decode_workspace_size(int B, int d_model, int H, int d, int n_mem, int top_k) {
    (void)d_model;
    if (B < 0 || H < 1 || d < 1 || n_mem < 1 || top_k < 1) return 0;
    return block_decode_layout(B, H, d, n_mem, top_k).total;
}

mom_status mom_block_decode_step(const void* x, const mom_weights* w, const mom_block_weights* bw,
                                 const mom_memory_gates* mg, int width, float eps, int B, int d_model, int H, int d,
                                 int n_mem, int top_k, float scale, mom_dtype dt, mom_rule rule, float* state,
                                 void* conv_sh, void* conv_mem, void* y, int32_t* topk_idx, void* ws,
                                 size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || B < 0 || d_model <= 0 || d_model % 64 != 0 || H < 1 || H > MOM_MAX_HEADS) return MOM_ERR_ARG;
    if (rule != MOM_RULE_GATED_DELTA && rule != MOM_RULE_GATED_LINEAR) return MOM_ERR_ARG;
    if (top_k < 1 || n_mem < top_k || n_mem > MOM_MAX_MEM || !w || !bw || !(eps >= 0.f)) return MOM_ERR_ARG;
    if (width < 2 || width > 4 || dt != MOM_BF16 || !head_dim_ok(d)) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < mom_block_decode_workspace_size(B, d_model, H, d, n_mem, top_k)) return MOM_ERR_ARG;
    if (B == 0) return MOM_OK;
    const void* ptrs[] = {x, w->w_r, w->w_gate, w->A, w->b_a, w->w_kv, bw->w_shared4, bw->w_o, bw->conv_q,
                          bw->conv_k_sh, bw->conv_v_sh, bw->conv_k, bw->conv_v, bw->w_norm, state, conv_sh,
                          conv_mem, y};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    if (mg && (!mg->w_gate_mem || !al16(mg->w_gate_mem) || !mg->A_mem || !mg->b_a_mem)) return MOM_ERR_ARG;
    const int Hd = H * d;
    cudaStream_t st = as_stream(stream);
    const BlockDecodeLayout BL = block_decode_layout(B, H, d, n_mem, top_k);
    const DecodeLayout& L = BL.base;
    char* base = reinterpret_cast<char*>(ws);
    int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(base + L.idx);
    float* gate = reinterpret_cast<float*>(base + L.gate);
    int32_t* perm = reinterpret_cast<int32_t*>(base + L.perm);
    int32_t* row_of = reinterpret_cast<int32_t*>(base + L.row_of);
    int32_t* mem_off = reinterpret_cast<int32_t*>(base + L.mem_off);
    int32_t* seg_cu = reinterpret_cast<int32_t*>(base + L.seg_cu);
    float* beta = reinterpret_cast<float*>(base + L.beta);
    float* la = reinterpret_cast<float*>(base + L.la);

    const cudaStream_t ss = fork_side(st);
    cudaError_t e = launch_gate_proj(x, w->w_gate, w->A, w->b_a, dt, B, d_model, H, beta, la, ws, ss);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    e = launch_router(x, w->w_r, w->b_r, dt, B, d_model, n_mem, top_k, idx, gate, nullptr, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    e = launch_permute(idx, B, top_k, n_mem, nullptr, 1, perm, row_of, mem_off, seg_cu, ws, base + L.perm_scratch, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    if (join_side(st, ss) != cudaSuccess) return MOM_ERR_CUDA;
    // the raw projections and the output gate
    ProjArgs pa{x, perm, mem_off, bw->w_shared4, w->w_kv, B, d_model, H, d, n_mem, top_k,
                base + BL.q_raw, base + BL.k_sh_raw, base + BL.v_sh_raw, base + BL.k_p_raw, base + BL.v_p_raw, ws};
    pa.raw = 1;
    pa.g = base + BL.g;
    if (!proj_tc_supported(pa, dt)) return MOM_ERR_UNSUPPORTED;
    e = launch_proj_tc(pa, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    // one row of every convolution, the windows shifted
    ConvStepArgs ca;
    const char* raws[5] = {base + BL.q_raw, base + BL.k_sh_raw, base + BL.v_sh_raw, base + BL.k_p_raw,
                           base + BL.v_p_raw};
    char* outs[5] = {base + L.q, base + L.k_sh, base + L.v_sh, base + L.k_p, base + L.v_p};
    const float* filts[5] = {bw->conv_q, bw->conv_k_sh, bw->conv_v_sh, bw->conv_k, bw->conv_v};
    for (int i = 0; i < 5; ++i) {
        ca.z[i] = reinterpret_cast<const bf16*>(raws[i]);
        ca.out[i] = reinterpret_cast<bf16*>(outs[i]);
        ca.w[i] = filts[i];
    }
    ca.st_sh = reinterpret_cast<bf16*>(conv_sh);
    ca.st_mem = reinterpret_cast<bf16*>(conv_mem);
    ca.perm = perm;
    ca.mem_offset = mem_off;
    ca.B = B; ca.K = top_k; ca.M = n_mem; ca.C = Hd; ca.d = d;
    ca.err = ws;
    e = launch_conv_step(ca, width, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    // the recurrences' step and the combine
    DecodeArgs da{base + L.q, base + L.k_sh, base + L.v_sh, base + L.k_p, base + L.v_p, beta, la, gate,
                  idx, row_of, B, H, d, n_mem, top_k, scale, state, base + BL.comb, ws};
    da.rule = rule;
    if (mg) {
        float* beta_p = reinterpret_cast<float*>(base + L.beta_p);
        float* la_p = reinterpret_cast<float*>(base + L.la_p);
        e = launch_mem_gate_proj(x, perm, mem_off, mg->w_gate_mem, mg->A_mem, mg->b_a_mem, dt, B, (int64_t)B * top_k,
                                 d_model, H, n_mem, beta_p, la_p, ws, st);
        if (e != cudaSuccess) return MOM_ERR_CUDA;
        da.beta_p = beta_p;
        da.log_alpha_p = la_p;
    }
    e = launch_decode_state(da, dt, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    // the gated norm, then W_o
    e = launch_combine_norm_gate(base + BL.comb, nullptr, nullptr, nullptr, base + BL.g, bw->w_norm, eps, B, 0, H, d,
                                 base + BL.o_tilde, ws, st);
    if (e != cudaSuccess) return MOM_ERR_CUDA;
    ProjArgs lo{base + BL.o_tilde, nullptr, nullptr, bw->w_o, nullptr, B, Hd, 1, d_model, 1, 1,
                y, nullptr, nullptr, nullptr, nullptr, ws};
    lo.parts = PROJ_SHARED;
    lo.plain_n = d_model;
    if (!proj_tc_supported(lo, dt)) return MOM_ERR_UNSUPPORTED;
    return cuda_status(launch_proj_tc(lo, st));
}

mom_status mom_block_conv_state(const void* q_raw, const void* k_sh_raw, const void* v_sh_raw, const void* k_p_raw,
                                const void* v_p_raw, int64_t n_tok, int top_k, const int32_t* cu_seqlens,
                                const int32_t* seg_cu, int n_seq, int n_mem, int channels, int width, mom_dtype dt,
                                void* conv_sh, void* conv_mem, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || top_k < 1 || n_seq < 1 || n_mem < 1 || n_mem > MOM_MAX_MEM) return MOM_ERR_ARG;
    if (channels < 8 || channels % 8 != 0) return MOM_ERR_ARG;
    if (width < 2 || width > 4 || dt != MOM_BF16) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    const void* ptrs[] = {q_raw, k_sh_raw, v_sh_raw, k_p_raw, v_p_raw, conv_sh, conv_mem};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    if (!cu_seqlens || !seg_cu) return MOM_ERR_ARG;
    ConvStateArgs a;
    const void* raws[5] = {q_raw, k_sh_raw, v_sh_raw, k_p_raw, v_p_raw};
    for (int i = 0; i < 5; ++i) a.z[i] = reinterpret_cast<const bf16*>(raws[i]);
    a.st_sh = reinterpret_cast<bf16*>(conv_sh);
    a.st_mem = reinterpret_cast<bf16*>(conv_mem);
    a.cu = cu_seqlens;
    a.seg_cu = seg_cu;
    a.S = n_seq; a.M = n_mem; a.C = channels; a.W = width;
    a.n_tok = n_tok;
    a.n_rows = n_tok * top_k;
    a.err = ws;
    return cuda_status(launch_conv_state(a, as_stream(stream)));
}

// ----------------------------------------------------------- block bwd
mom_status mom_norm_gate_bwd(const void* o_sh, const void* o_p, const int32_t* row_of, const float* topk_gate,
                             const void* g, const float* w_norm, float eps, const void* d_y, int64_t n_tok,
                             int top_k, int H, int d, mom_dtype dt, void* d_o, float* dg, int64_t ldg,
                             float* dw_norm, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || n_tok < 0 || top_k < 0 || H < 1 || H > MOM_MAX_HEADS || !(eps >= 0.f)) return MOM_ERR_ARG;
    if (d < 8 || d > 256 || (d & (d - 1)) != 0 || ldg < (int64_t)H * d) return MOM_ERR_ARG;
    if (dt != MOM_BF16) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES || !dw_norm || !w_norm || !al16(w_norm)) return MOM_ERR_ARG;
    const void* ptrs[] = {o_sh, g, d_y, d_o, dg};
    for (const void* p : ptrs)
        if (!p || !al16(p)) return MOM_ERR_ARG;
    if (ldg % 4 != 0) return MOM_ERR_ARG;
    if (top_k > 0 && (!o_p || !row_of || !topk_gate || !al16(o_p))) return MOM_ERR_ARG;
    return cuda_status(launch_norm_gate_bwd(o_sh, o_p, row_of, topk_gate, g, w_norm, eps, d_y, n_tok, top_k, H, d,
                                            d_o, dg, ldg, dw_norm, ws, as_stream(stream)));
}

mom_status mom_short_conv_bwd(const mom_conv_bwd_problem* problems, int n_problems, int channels, int width,
                              int head_dim, mom_dtype dt, void* ws, size_t ws_bytes, void* stream) {
    if (!dt_ok(dt) || !problems || n_problems < 1 || channels < 8 || channels % 8 != 0 || width < 1) return MOM_ERR_ARG;
    if (dt != MOM_BF16 || width > 4 || n_problems > 8) return MOM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < MOM_WS_HEADER_BYTES) return MOM_ERR_ARG;
    ConvBwdArgs pr[8];
    for (int i = 0; i < n_problems; ++i) {
        const mom_conv_bwd_problem& q = problems[i];
        if (q.n_rows < 0 || q.n_seg < 1 || q.seg_per_group < 1 || q.n_groups < 1) return MOM_ERR_ARG;
        if (q.l2norm != 0 && q.l2norm != 1) return MOM_ERR_ARG;
        if (q.l2norm && (head_dim < 8 || head_dim > 256 || (head_dim & (head_dim - 1)) != 0 || channels % head_dim))
            return MOM_ERR_ARG;
        if (q.ldz < q.col0 + channels || q.col0 < 0 || q.ldz % 4 || q.col0 % 4) return MOM_ERR_ARG;
        const void* ptrs[] = {q.z, q.dout, q.dz, q.seg_cu, q.w, q.dw};
        for (const void* p : ptrs)
            if (!p || !al16(p)) return MOM_ERR_ARG;
        pr[i] = ConvBwdArgs{q.z, q.dout, q.da, q.dz, q.ldz, q.col0, q.n_rows, q.seg_cu, q.n_seg, q.seg_per_group,
                            q.n_groups, q.w, q.dw, q.l2norm};
    }
    return cuda_status(launch_conv_bwd(pr, n_problems, channels, width, head_dim, ws, as_stream(stream)));
}

mom_status mom_convert(const void* src, mom_dtype src_dt, void* dst, mom_dtype dst_dt, int64_t n, void* stream) {
    if (!dt_ok(src_dt) || !dt_ok(dst_dt) || n < 0) return MOM_ERR_ARG;
    if (n == 0) return MOM_OK;
    if (!src || !dst) return MOM_ERR_ARG;
    return cuda_status(launch_convert(src, src_dt, dst, dst_dt, n, as_stream(stream)));
}

}  // extern "C"
