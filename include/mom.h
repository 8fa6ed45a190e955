/*
 * mom.h -- C ABI of the B200 (sm_100a) Mixture-of-Memories layer library.
 *
 * One MoM layer forward: a linear router picks each token's top-k memories;
 * tokens are reordered into contiguous per-memory segments; every memory
 * (and an always-on shared memory) projects its own keys/values and runs a
 * Gated DeltaNet recurrence over only the tokens routed to it; the outputs
 * are summed with the router weights.  A constant-cost recurrent decode
 * step runs the same layer one token per sequence.
 *
 * Sources (page title, section):
 *   "MoM: Linear Sequence Modeling with Mixture-of-Memories" (paper card),
 *       Summary -- the layer as a whole;
 *   "MoM: Mixture-of-Memories Fixes Linear Attention Recall" (explainer),
 *       "Router mechanics, step by step" and "Solving scatter-gather without
 *       new kernels";
 *   the authors' MoM blog post, sections "Mixture-of-Memories" and
 *       "硬件高效實現" (hardware-efficient implementation), and its
 *       experiments section, which fixes Gated DeltaNet as the memory rule.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless documented otherwise; every array
 *     is dense row-major and 16-byte aligned.
 *   - The caller owns every buffer.  The library never allocates or frees;
 *     scratch space is the caller's `ws` of at least the size that the
 *     matching mom_*_workspace_size() returns.  The first MOM_WS_HEADER_BYTES
 *     of any workspace hold a device-side error record (see mom_get_error);
 *     zero the workspace once before its first use.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise the host, except mom_get_error.
 *   - Projection weights use the [out_features, in_features] layout
 *     (y = x W^T).  Activations are [rows, H, d]; recurrent states are
 *     [.., H, d_v, d_k] float32 so that o = S q.
 *   - `dt` selects the element type of activations and weights (MOM_F32 or
 *     MOM_BF16).  Router gates, logits, beta, log alpha and states are
 *     always float32.
 *   - Arguments are validated before any launch; a failed validation
 *     launches nothing, writes nothing and returns MOM_ERR_ARG or
 *     MOM_ERR_UNSUPPORTED.  A failed launch returns MOM_ERR_CUDA.
 *   - Data-dependent violations seen on the device (a memory index >= M, a
 *     row index out of range, inconsistent segment bounds) are skipped
 *     without any out-of-bounds access and recorded in the workspace's error
 *     record; no kernel traps or aborts.
 */
#ifndef MOM_H
#define MOM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int mom_status;
#define MOM_OK               0
#define MOM_ERR_ARG          1  /* bad pointer, size or alignment */
#define MOM_ERR_UNSUPPORTED  2  /* valid but not implemented (e.g. d not in {64,128,256}) */
#define MOM_ERR_CUDA         3  /* a launch or CUDA runtime call failed */
#define MOM_ERR_DEVICE       4  /* mom_get_error: a kernel recorded a data violation */

typedef int mom_dtype;
#define MOM_F32   0
#define MOM_BF16  1

/* Memory update rules.  The authors' MoM blog post ("Linear Recurrent
 * Memory") lists the family of rules a memory can use -- linear attention,
 * RetNet, GLA, DeltaNet, Gated DeltaNet, Mamba2, HGRN2 -- in one
 * linear-attention form (the page's formulas were lost in extraction); its
 * experiments use Gated DeltaNet.  Both rules here have a scalar gate
 * alpha_t = exp(log_alpha_t) and a write strength beta_t per token and head:
 *   MOM_RULE_GATED_DELTA   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *                          (Gated DeltaNet; DeltaNet with alpha = 1)
 *   MOM_RULE_GATED_LINEAR  S_t = alpha_t S_{t-1} + beta_t v_t k_t^T
 *                          (linear attention with alpha = beta = 1, RetNet with a
 *                          fixed alpha per head, Mamba2-style memories)
 * and the readout o_t = S_t (scale q_t).  Rules with a per-dimension gate
 * (GLA, HGRN2) are not provided. */
typedef int mom_rule;
#define MOM_RULE_GATED_DELTA   0
#define MOM_RULE_GATED_LINEAR  1

/* Device error record codes (mom_get_error's *code). */
#define MOM_DEVERR_NONE       0
#define MOM_DEVERR_MEM_INDEX  1  /* topk_idx entry outside [0, n_mem) or repeated in a row */
#define MOM_DEVERR_ROW_INDEX  2  /* a row / token index outside its array */
#define MOM_DEVERR_SEGMENT    3  /* segment bounds decreasing or beyond n_rows */
#define MOM_DEVERR_TIMEOUT    4  /* a pipeline wait inside a kernel gave up (internal error) */

#define MOM_WS_HEADER_BYTES 256

/* Largest supported sizes. */
#define MOM_MAX_MEM   32   /* routed memories M */
#define MOM_MAX_HEADS 64

/* Human-readable name of a status code (static string). */
const char* mom_status_string(mom_status s);

/* Reads the device error record of `ws` (synchronises `stream`).  Writes the
 * first recorded code (MOM_DEVERR_*) and its offending index to *code and
 * *info (either may be NULL).  Returns MOM_OK when no violation was
 * recorded, MOM_ERR_DEVICE when one was, MOM_ERR_CUDA on a runtime error. */
mom_status mom_get_error(const void* ws, int32_t* code, int32_t* info, void* stream);

/* Clears the device error record of `ws` (asynchronous on `stream`). */
mom_status mom_clear_error(void* ws, void* stream);

/* Diagnostic: the number of kernels this library has launched in this
 * process (all devices, all streams).  Host-side counter, thread-safe. */
uint64_t mom_launch_count(void);

/* Diagnostic self-test of the failure path every pipelined kernel shares:
 * launches one thread that waits, with the library's bounded barrier wait,
 * on a barrier that nothing signals.  After `limit_cycles` SM cycles
 * (1 .. 4e9; about 2e6 is a millisecond) the wait gives up, records
 * MOM_DEVERR_TIMEOUT with info MOM_SELFTEST_WAIT_SITE in the error record of
 * `ws` (at least MOM_WS_HEADER_BYTES), and the kernel returns: the context
 * stays usable and mom_get_error reports the record.  Asynchronous on
 * `stream`.  MOM_ERR_ARG for a NULL or short workspace or a limit out of
 * range. */
#define MOM_SELFTEST_WAIT_SITE 990
mom_status mom_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t limit_cycles, void* stream);

/* ------------------------------------------------------------------------
 * mom_router_topk -- the router: one matmul, one softmax, one top-k, one
 * renormalisation (explainer, "Router mechanics, step by step"; blog post,
 * "Mixture-of-Memories").
 *
 *   logits[t, m] = x[t, :] . w_r[m, :] + b_r[m]        (float32 accumulate)
 *   topk_idx[t, :] = the top_k memories by logit, in descending order; equal
 *                    logits go to the lower memory index
 *   topk_gate[t, j] = softmax(logits[t])[idx_j] / sum_j' softmax(logits[t])[idx_j']
 *
 * x [n_tok, d_model] (dt); w_r [n_mem, d_model] (dt); b_r [n_mem] float32 or
 * NULL (zero bias).  Outputs: topk_idx [n_tok, top_k] int32, topk_gate
 * [n_tok, top_k] float32, logits [n_tok, n_mem] float32 or NULL.
 * Requires 1 <= top_k <= n_mem <= MOM_MAX_MEM, d_model % 8 == 0,
 * n_tok >= 0 (n_tok == 0 launches nothing).
 * ---------------------------------------------------------------------- */
mom_status mom_router_topk(const void* x, const void* w_r, const float* b_r, mom_dtype dt,
                           int64_t n_tok, int d_model, int n_mem, int top_k,
                           int32_t* topk_idx, float* topk_gate, float* logits, void* stream);

/* ------------------------------------------------------------------------
 * mom_permute -- reorder the routed (token, slot) pairs into contiguous
 * per-memory segments (explainer, "Solving scatter-gather without new
 * kernels"): a stable counting sort by memory.
 *
 * Pair r = t*top_k + j routes token t to memory topk_idx[t, j].  Outputs:
 *   perm_token [n_tok*top_k]  token of each reordered row;
 *   row_of     [n_tok*top_k]  reordered row of pair t*top_k + j;
 *   mem_offset [n_mem+1]      first row of each memory (mem_offset[n_mem] =
 *                             number of valid pairs);
 *   seg_cu     [n_mem*n_seq+1] segment bounds, one segment per (memory,
 *                             sequence), memory-major; rows inside a segment
 *                             keep token order.  Empty segments are allowed.
 * cu_seqlens [n_seq+1] int32 (device) gives the sequences of the packed
 * batch (cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seq] = n_tok).
 * A pair whose memory index is out of range is recorded
 * (MOM_DEVERR_MEM_INDEX) and dropped.  ws: mom_permute_workspace_size().
 * ---------------------------------------------------------------------- */
size_t mom_permute_workspace_size(int64_t n_tok, int top_k, int n_mem, int n_seq);
mom_status mom_permute(const int32_t* topk_idx, int64_t n_tok, int top_k, int n_mem,
                       const int32_t* cu_seqlens, int n_seq,
                       int32_t* perm_token, int32_t* row_of, int32_t* mem_offset, int32_t* seg_cu,
                       void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * mom_permute_noalloc -- mom_permute without a workspace.  The MoM pages
 * have no counterpart to this: it exists for callers that cannot allocate
 * device memory, such as a plug-in inside a host engine that owns every
 * byte of the device through its own fixed pool and forbids raw
 * cudaMalloc, or a latency-critical serving loop where cudaMalloc and
 * cudaFree are not allowed because they can block the host and synchronise
 * the device.
 *
 * Same arguments, outputs and results as mom_permute, minus ws/ws_bytes.
 * Its scratch space is a fixed array inside the library (about 1 MiB per
 * GPU that loads the library, held until the process exits), so:
 *   - n_tok may not exceed MOM_PERMUTE_NOALLOC_MAX_TOKENS: a larger n_tok
 *     returns MOM_ERR_UNSUPPORTED and launches nothing; n_mem above
 *     MOM_MAX_MEM returns MOM_ERR_ARG, as for mom_permute;
 *   - the first call in a CUDA context on a device looks up the array's
 *     device address in that context (a runtime query, then cached while
 *     that context stays current on the device); make that first call
 *     before any stream capture on that device, and again after a
 *     cudaDeviceReset or a switch to another context;
 *   - every call on a device shares the array: calls whose kernels overlap
 *     on the GPU (unordered streams, several host threads) race and may
 *     give wrong results -- order them on one stream;
 *   - each call clears the array's error record first; status_out (device
 *     int32[2], or NULL) receives this call's record {code, info}
 *     (MOM_DEVERR_*), asynchronously on `stream`.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * ---------------------------------------------------------------------- */
#define MOM_PERMUTE_NOALLOC_MAX_TOKENS (1 << 20)
mom_status mom_permute_noalloc(const int32_t* topk_idx, int64_t n_tok, int top_k, int n_mem,
                               const int32_t* cu_seqlens, int n_seq,
                               int32_t* perm_token, int32_t* row_of, int32_t* mem_offset, int32_t* seg_cu,
                               int32_t* status_out, void* stream);

/* ------------------------------------------------------------------------
 * mom_kv_proj_grouped -- every projection of the layer (paper card,
 * Summary: a shared query, and key/value projections of each memory's own):
 *
 *   q     = l2norm_h(x W_q^T)              k_sh = l2norm_h(x W_k_sh^T)
 *   v_sh  = x W_v_sh^T                     beta = sigmoid(x W_beta^T)
 *   log_alpha = -exp(A) * softplus(x W_a^T + b_a)
 *   for each memory m and reordered row r in [mem_offset[m], mem_offset[m+1]):
 *     k_p[r] = l2norm_h(x[perm_token[r]] W_k^m^T),  v_p[r] = x[perm_token[r]] W_v^m^T
 *
 * l2norm_h(y) = y / sqrt(|y|^2 + 1e-6) per head of d elements.
 * x [n_tok, d_model]; w_shared [3*H*d, d_model] = rows W_q | W_k_sh | W_v_sh;
 * w_gate [2*H, d_model] = rows W_beta | W_a; A, b_a [H] float32;
 * w_kv [n_mem, 2*H*d, d_model] = per memory rows W_k^m | W_v^m.
 * Outputs q, k_sh, v_sh [n_tok, H, d] (dt); beta, log_alpha [n_tok, H]
 * float32; k_p, v_p [n_tok*top_k, H, d] (dt).  Rows of k_p / v_p past
 * mem_offset[n_mem] are not written.  Requires d in {64, 128, 256},
 * d_model % 64 == 0.  ws: mom_kv_proj_workspace_size().
 * beta and log_alpha may both be NULL (w_gate, A, b_a then unused): the
 * gates are left to mom_gate_proj, which needs no routing and can run on
 * another stream while the router and the reordering run.
 * ---------------------------------------------------------------------- */
size_t mom_kv_proj_workspace_size(int64_t n_tok, int d_model, int H, int d, int n_mem, int top_k);
mom_status mom_kv_proj_grouped(const void* x, const int32_t* perm_token, const int32_t* mem_offset,
                               const void* w_shared, const void* w_gate, const float* A, const float* b_a,
                               const void* w_kv, mom_dtype dt,
                               int64_t n_tok, int d_model, int H, int d, int n_mem, int top_k,
                               void* q, void* k_sh, void* v_sh, float* beta, float* log_alpha,
                               void* k_p, void* v_p, void* ws, size_t ws_bytes, void* stream);

/* mom_proj_shared -- the shared projections of mom_kv_proj_grouped alone
 * (q, k_sh, v_sh), which need no routing: a memory-parallel layer runs them
 * on the tokens' own rank.  Arguments as in mom_kv_proj_grouped; q_norm and
 * k_sh_norm [n_tok, H] float32 or NULL receive sqrt(|z|^2 + 1e-6) of every
 * (token, head) before its L2 norm (what the norm's backward needs).
 * ws: mom_kv_proj_workspace_size(n_tok, d_model, H, d, 1, 1). */
mom_status mom_proj_shared(const void* x, const void* w_shared, mom_dtype dt, int64_t n_tok, int d_model,
                           int H, int d, void* q, void* k_sh, void* v_sh, float* q_norm, float* k_sh_norm,
                           void* ws, size_t ws_bytes, void* stream);

/* mom_kv_proj_groups -- the routed key/value projections over an explicit
 * group table: the rows a memory-parallel layer receives, grouped by
 * (source rank, memory) (explainer, "Memory count scaling": memories spread
 * over GPUs).  Group g covers rows group_offset[g] .. group_offset[g+1]-1
 * (non-decreasing, group_offset[n_groups] <= n_rows) and uses memory
 * group_mem[g]'s weights (0 <= group_mem[g] < n_mem):
 *   k_p[r] = l2norm_h(x[perm_token[r]] W_k^m^T),  v_p[r] = x[perm_token[r]] W_v^m^T
 * with perm_token NULL meaning row r reads x row r.  x [n_x, d_model];
 * w_kv [n_mem, 2*H*d, d_model]; k_p, v_p [n_rows, H, d] (dt); k_norm
 * [n_rows, H] float32 or NULL receives sqrt(|z|^2 + 1e-6) of every (row,
 * head) of k before its norm.  Rows past group_offset[n_groups] are not
 * written.  A corrupt table or index is recorded in ws (MOM_DEVERR_*) and
 * the affected tiles are skipped.  ws: at least MOM_WS_HEADER_BYTES. */
mom_status mom_kv_proj_groups(const void* x, int64_t n_x, const int32_t* perm_token, int64_t n_rows,
                              const int32_t* group_offset, const int32_t* group_mem, int n_groups,
                              const void* w_kv, mom_dtype dt, int d_model, int H, int d, int n_mem,
                              void* k_p, void* v_p, float* k_norm, void* ws, size_t ws_bytes, void* stream);

/* mom_copy_rows -- row copies in 16-byte granules, for packing the routed
 * rows a memory-parallel layer sends to the owners of their memories and
 * unpacking what it receives:
 *   dst[i*dst_stride + dst_off .. + row_bytes) = src[s*src_stride + src_off .. + row_bytes)
 * for i < n_rows, s = idx[i] (idx NULL: s = i).  Byte strides and offsets
 * and row_bytes are multiples of 16; src and dst 16-byte aligned.  An index
 * outside [0, n_src) is recorded (MOM_DEVERR_ROW_INDEX) and its row
 * zero-filled.  ws: at least MOM_WS_HEADER_BYTES. */
mom_status mom_copy_rows(const void* src, int64_t n_src, int64_t src_stride, int64_t src_off,
                         const int32_t* idx, int64_t n_rows, int64_t row_bytes,
                         void* dst, int64_t dst_stride, int64_t dst_off, void* ws, size_t ws_bytes, void* stream);

/* mom_gate_proj -- the per-token gates of the memories alone (the Gated
 * DeltaNet gating every memory uses: blog post, experiments section):
 *   beta = sigmoid(x W_beta^T),  log_alpha = -exp(A) * softplus(x W_a^T + b_a)
 * x [n_tok, d_model] (dt), w_gate [2*H, d_model] = rows W_beta | W_a, A and
 * b_a [H] float32; beta, log_alpha [n_tok, H] float32.  The same values
 * mom_kv_proj_grouped writes when given beta / log_alpha.
 * ws: mom_gate_proj_workspace_size(). */
size_t mom_gate_proj_workspace_size(int64_t n_tok, int d_model, int H);
mom_status mom_gate_proj(const void* x, const void* w_gate, const float* A, const float* b_a, mom_dtype dt,
                         int64_t n_tok, int d_model, int H, float* beta, float* log_alpha,
                         void* ws, size_t ws_bytes, void* stream);

/* mom_mem_gate_proj -- per-memory gates of the routed rows: memory m keeps
 * its own W_beta^m, W_a^m, A^m, b_a^m (paper card, Summary: every memory has
 * its own recurrent update; the blog post's memories are Gated DeltaNet
 * layers, gates included).  For routed row r of memory m (mem_offset[m] <=
 * r < mem_offset[m+1]) and token t = perm_token[r]:
 *   beta_p[r]      = sigmoid(x[t] W_beta^m^T)
 *   log_alpha_p[r] = -exp(A^m) * softplus(x[t] W_a^m^T + b_a^m)
 * x [n_tok, d_model] (dt); perm_token, mem_offset as mom_permute writes
 * them (n_tok*top_k rows in memory order); w_gate_mem [n_mem, 2*H, d_model]
 * (dt) = rows W_beta^m | W_a^m per memory; A_mem, b_a_mem [n_mem, H]
 * float32.  Outputs beta_p, log_alpha_p [n_tok*top_k, H] float32, for the
 * memory calls with MOM_GATES_BY_ROW.  float32 accumulation (bf16 inputs on
 * the tensor cores).  A row that no memory holds or whose token is out of
 * range is recorded (MOM_DEVERR_ROW_INDEX) and gets beta = log_alpha = 0.
 * Requires 1 <= top_k <= n_mem <= MOM_MAX_MEM, d_model % 8 == 0.
 * ws: at least MOM_WS_HEADER_BYTES. */
mom_status mom_mem_gate_proj(const void* x, const int32_t* perm_token, const int32_t* mem_offset,
                             const void* w_gate_mem, const float* A_mem, const float* b_a_mem, mom_dtype dt,
                             int64_t n_tok, int d_model, int H, int n_mem, int top_k,
                             float* beta_p, float* log_alpha_p, void* ws, size_t ws_bytes, void* stream);

/* mom_mem_gate_proj_groups -- mom_mem_gate_proj over groups of rows that
 * name their memory: rows group_offset[g] .. group_offset[g+1]-1 (device,
 * n_groups + 1 entries, n_groups <= MOM_MAX_MEM) take memory group_mem[g]'s
 * gates (W^m, A^m, b_a^m of the n_mem in w_gate_mem, A_mem, b_a_mem), and
 * row r reads x row perm_token[r] (NULL: row r).  For the rows a
 * memory-parallel owner receives (groups: (source rank, memory)).  A group
 * whose memory is out of range is recorded (MOM_DEVERR_ROW_INDEX) and its
 * rows get beta = log_alpha = 0. */
mom_status mom_mem_gate_proj_groups(const void* x, int64_t n_x, const int32_t* perm_token, int64_t n_rows,
                                    const int32_t* group_offset, const int32_t* group_mem, int n_groups,
                                    const void* w_gate_mem, const float* A_mem, const float* b_a_mem, int n_mem,
                                    mom_dtype dt, int d_model, int H, float* beta_p, float* log_alpha_p, void* ws,
                                    size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * mom_gdn_chunk_fwd -- the Gated DeltaNet recurrence of one memory over
 * each segment (blog post, experiments section: every memory uses Gated
 * DeltaNet's gate and update rule; "Mixture-of-Memories": each memory runs
 * over only the tokens routed to it):
 *
 *   S_0 = h0[seg] (or 0);  for each row r of the segment, in order:
 *     S_r = alpha_r S_{r-1} (I - beta_r k_r k_r^T) + beta_r v_r k_r^T,
 *     o_r = S_r (scale * q_r),         alpha_r = exp(log_alpha_r)
 *   h_final[seg] = S_last.
 *
 * k, v, o [n_rows, H, d]; q [n_q_rows, H, d]; beta, log_alpha [n_q_rows, H]
 * float32.  When qidx (int32 [n_rows]) is non-NULL, row r reads q, beta and
 * log_alpha at row qidx[r] (the routed memories read the shared query of
 * the token behind each reordered row); otherwise at row r.  seg_cu
 * [n_seg+1] int32 row bounds (seg_cu[0] = 0, non-decreasing, <= n_rows).
 * h0, h_final [n_seg, H, d, d] float32 or NULL.  An empty segment writes
 * h_final = h0 (or zeros).  In MOM_BF16 mode q, k, v, o are bf16 while the
 * state and every accumulation stay float32; in MOM_F32 mode everything is
 * float32.  Requires d in {64, 128, 256}.  ws: mom_gdn_workspace_size().
 * ---------------------------------------------------------------------- */
size_t mom_gdn_workspace_size(int64_t n_rows, int n_seg, int H, int d, mom_dtype dt);
mom_status mom_gdn_chunk_fwd(const void* q, const int32_t* qidx, const void* k, const void* v,
                             const float* beta, const float* log_alpha,
                             const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                             int H, int d, float scale, mom_dtype dt,
                             const float* h0, float* h_final, void* o,
                             void* ws, size_t ws_bytes, void* stream);

/* The same call in two stream-ordered halves, for callers that schedule
 * several GDN problems (the layer's shared memory and its routed memories)
 * against each other:
 *   mom_gdn_chunk_prep  -- the state-independent work of every chunk (the
 *                          within-chunk triangular solve and decay masks),
 *                          left in ws;
 *   mom_gdn_chunk_state -- the serial walk over each segment's chunks, which
 *                          reads what the prep left in ws and writes o and
 *                          h_final.
 * Both take exactly the arguments of mom_gdn_chunk_fwd; the state call must
 * follow a prep call with the same arguments and ws (on the same stream, or
 * ordered after it by an event), and ws must not be reused in between.
 * prep followed by state is mom_gdn_chunk_fwd.  When the float32 token-serial
 * path runs (MOM_F32, or a shape the tensor-core path does not take) prep does
 * nothing and state does everything. */
mom_status mom_gdn_chunk_prep(const void* q, const int32_t* qidx, const void* k, const void* v,
                              const float* beta, const float* log_alpha,
                              const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                              int H, int d, float scale, mom_dtype dt,
                              const float* h0, float* h_final, void* o,
                              void* ws, size_t ws_bytes, void* stream);
mom_status mom_gdn_chunk_state(const void* q, const int32_t* qidx, const void* k, const void* v,
                               const float* beta, const float* log_alpha,
                               const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                               int H, int d, float scale, mom_dtype dt,
                               const float* h0, float* h_final, void* o,
                               void* ws, size_t ws_bytes, void* stream);

/* The same three calls for either memory rule (MOM_RULE_*) and either gate
 * layout (MOM_GATES_*); the mom_gdn_* calls are these with
 * MOM_RULE_GATED_DELTA and MOM_GATES_BY_TOKEN.  Same arguments otherwise,
 * same workspace (mom_gdn_workspace_size); MOM_ERR_ARG for an unknown rule
 * or layout.  With MOM_GATES_BY_ROW, beta and log_alpha are [n_rows, H]:
 * row r's own gates (the per-memory gates mom_mem_gate_proj writes), read at
 * row r whether or not qidx is given. */
typedef int mom_gates;
#define MOM_GATES_BY_TOKEN  0   /* beta, log_alpha [n_q_rows, H], read like q */
#define MOM_GATES_BY_ROW    1   /* beta, log_alpha [n_rows, H], one per row of k, v */
mom_status mom_memory_chunk_fwd(const void* q, const int32_t* qidx, const void* k, const void* v,
                                const float* beta, const float* log_alpha,
                                const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                                int H, int d, float scale, mom_dtype dt, mom_rule rule, mom_gates gates,
                                const float* h0, float* h_final, void* o,
                                void* ws, size_t ws_bytes, void* stream);
mom_status mom_memory_chunk_prep(const void* q, const int32_t* qidx, const void* k, const void* v,
                                 const float* beta, const float* log_alpha,
                                 const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                                 int H, int d, float scale, mom_dtype dt, mom_rule rule, mom_gates gates,
                                 const float* h0, float* h_final, void* o,
                                 void* ws, size_t ws_bytes, void* stream);
mom_status mom_memory_chunk_state(const void* q, const int32_t* qidx, const void* k, const void* v,
                                  const float* beta, const float* log_alpha,
                                  const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                                  int H, int d, float scale, mom_dtype dt, mom_rule rule, mom_gates gates,
                                  const float* h0, float* h_final, void* o,
                                  void* ws, size_t ws_bytes, void* stream);

/* mom_memory_chunk_bwd -- the reverse pass of mom_memory_chunk_fwd (either
 * rule, either gate layout) for the loss <d_o, o> + sum_s <dh_final[s],
 * h_final[s]> (training is the pages' main workload: paper card, Key points):
 *   dq, dk, dv [n_rows, H, d] float32, dbeta, dlog_alpha [n_rows, H] float32
 *   -- one per ROW of the segments (with qidx, row r's dq / dbeta /
 *   dlog_alpha belong to q row qidx[r]: the caller adds them up per token) --
 *   and dh0 [n_seg, H, d, d] float32 (NULL: not written).
 * Inputs as mom_memory_chunk_fwd (q, k, v, the gates, seg_cu, h0 NULL = zero
 * states), plus d_o [n_rows, H, d] (dt) and dh_final [n_seg, H, d, d]
 * float32 or NULL (zero).  Rows outside [seg_cu[0], seg_cu[n_seg]) are not
 * written; a row whose q index is out of range is recorded
 * (MOM_DEVERR_ROW_INDEX) and contributes nothing.  Token-serial on CUDA
 * cores in float32 whatever dt is.  Requires d in {64, 128, 256}.
 * ws: mom_memory_chunk_bwd_workspace_size() (states kept for the reverse
 * sweep and one partial sum per 64 state rows: about
 * n_rows * H * d * 8 * d / 64 bytes). */
size_t mom_memory_chunk_bwd_workspace_size(int64_t n_rows, int n_seg, int H, int d);
mom_status mom_memory_chunk_bwd(const void* q, const int32_t* qidx, const void* k, const void* v,
                                const float* beta, const float* log_alpha,
                                const int32_t* seg_cu, int n_seg, int64_t n_rows, int64_t n_q_rows,
                                int H, int d, float scale, mom_dtype dt, mom_rule rule, mom_gates gates,
                                const float* h0, const void* d_o, const float* dh_final,
                                float* dq, float* dk, float* dv, float* dbeta, float* dlog_alpha, float* dh0,
                                void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The layer's backward around the recurrences (training: paper card, Key
 * points).  MoMLayer.backward strings these with mom_memory_chunk_bwd; the
 * routing is held fixed (the top-k choice is piecewise constant), gradients
 * flow through the renormalised gates.  float32 gradients; every call is
 * asynchronous on `stream`; ws (at least MOM_WS_HEADER_BYTES) takes the
 * device error record where a call reads indices.
 *
 * mom_combine_bwd -- for out_t = o_sh,t + sum_j gate[t,j] o_p[row_of(t,j)]:
 *   do_p[row_of(t,j)] = gate[t,j] dout[t]          (dt)
 *   dgate[t,j]        = <dout[t], o_p[row_of(t,j)]>  (float32)
 * dout [n_tok, H*d], o_p and do_p [n_rows, H*d] (dt); row_of [n_tok*top_k];
 * gate, dgate [n_tok, top_k].
 * ---------------------------------------------------------------------- */
mom_status mom_combine_bwd(const void* dout, const void* o_p, const int32_t* row_of, const float* gate,
                           int64_t n_tok, int top_k, int64_t n_rows, int H, int d, mom_dtype dt,
                           void* do_p, float* dgate, void* ws, size_t ws_bytes, void* stream);

/* mom_router_bwd -- the adjoint of the renormalised gates g_j = exp(l_j) /
 * sum_i exp(l_i) over the chosen memories (explainer, Router mechanics):
 * dlogits[t, idx[t,j]] = g_j (dgate_j - sum_i g_i dgate_i), zero elsewhere.
 * topk_idx, gate, dgate [n_tok, top_k]; dlogits [n_tok, n_mem] float32. */
mom_status mom_router_bwd(const int32_t* topk_idx, const float* gate, const float* dgate, int64_t n_tok,
                          int top_k, int n_mem, float* dlogits, void* ws, size_t ws_bytes, void* stream);

/* mom_rows_sum -- dst[t] = base[t] (NULL: 0) + sum_j src[row_of[t*top_k+j]]
 * over float32 rows of width W (a token's gradient from its routed rows).
 * dst may be base. */
mom_status mom_rows_sum(const float* src, int64_t n_src, const int32_t* row_of, int top_k, const float* base,
                        int64_t n_tok, int W, float* dst, void* ws, size_t ws_bytes, void* stream);

/* mom_l2norm_bwd -- for y = z / sqrt(|z|^2 + 1e-6) per (row, head):
 * dz[r*ldz + col0 + h*d + c] = (dy - y (y . dy)) / norm[r, h]; y [rows, H, d]
 * (dt), dy [rows, H, d] float32, norm [rows, H] float32 (the projections'
 * norm outputs). */
mom_status mom_l2norm_bwd(const void* y, const float* dy, const float* norm, int64_t rows, int H, int d,
                          mom_dtype dt, float* dz, int64_t ldz, int64_t col0, void* stream);

/* mom_gates_bwd -- beta = sigmoid(z_b), log_alpha = -exp(A) softplus(z_a):
 * dz[r*ldz + col_b + h] = dbeta beta (1 - beta);
 * dz[r*ldz + col_a + h] = dlog_alpha (-exp(A_h)) sigmoid(z_a) (sigmoid(z_a)
 * from log_alpha); dala = dlog_alpha log_alpha.  All [n, H] float32. */
mom_status mom_gates_bwd(const float* beta, const float* log_alpha, const float* dbeta, const float* dlog_alpha,
                         const float* A, int64_t n, int H, float* dz, int64_t ldz, int64_t col_b, int64_t col_a,
                         float* dala, void* stream);

/* mom_col_sums -- out[c] = sum_r a[r*lda + c], c < cols (float32). */
mom_status mom_col_sums(const float* a, int64_t rows, int64_t lda, int64_t cols, float* out, void* stream);

/* mom_gates_bwd_by_group -- mom_gates_bwd for rows in groups with their own
 * A: group g covers rows group_offset[g] .. group_offset[g+1]-1 (device
 * array, n_groups + 1 entries, non-decreasing, covering 0 .. n) and its rows
 * take A[g*H + h] (the per-memory gates' A_mem [M, H] over the reordered
 * rows, group g = memory g). */
mom_status mom_gates_bwd_by_group(const float* beta, const float* log_alpha, const float* dbeta, const float* dlog_alpha,
                                  const float* A, const int32_t* group_offset, int n_groups, int64_t n, int H, float* dz,
                                  int64_t ldz, int64_t col_b, int64_t col_a, float* dala, void* stream);

/* mom_col_sums_grouped -- out[g*cols + c] = sum over the rows r of group g
 * (group_offset as above, clipped to 0 .. rows) of a[r*lda + c] (float32):
 * the per-memory gates' dA and db_a. */
mom_status mom_col_sums_grouped(const float* a, int64_t rows, int64_t lda, int64_t cols, const int32_t* group_offset,
                                int n_groups, float* out, void* stream);

/* mom_gemm_grouped -- float32 C (+)= op(A) B over groups of rows, for the
 * projections' input and weight gradients.  A float32, B (dt), C float32,
 * row-major with leading dimensions lda, ldb, ldc (elements):
 *   trans_a = 0: group g covers rows group_offset[g]..[g+1]-1 of A [*, K] and
 *     of C [*, N]; C[r] (+)= A[r] B_g with B_g = B + group_index[g] *
 *     b_group_stride, [K, N] (the input gradient dZ W);
 *   trans_a = 1: group g covers reduction rows group_offset[g]..[g+1]-1;
 *     C_g (+)= sum_r A[r, :M]^T B[b_rows[r] (or r), :N] with C_g = C +
 *     group_index[g] * c_group_stride, [M, N] (the weight gradient dZ^T X).
 * group_index NULL: g.  total_rows: group_offset[n_groups] (trans_a = 0).
 * accumulate: 0 overwrite, 1 add.  A bad row index is recorded in ws and
 * reads as zero.  With B in bf16 the products run on the tensor cores in
 * tf32 (B exact, A rounded to a 10-bit mantissa, fp32 accumulation); with B
 * in float32, on CUDA cores in fp32. */
mom_status mom_gemm_grouped(int trans_a, const float* A, int64_t lda, const void* B, int64_t ldb, mom_dtype dt,
                            const int32_t* b_rows, int64_t n_b_rows, float* C, int64_t ldc, int64_t M, int64_t N,
                            int64_t K, int64_t total_rows, const int32_t* group_offset, const int32_t* group_index,
                            int n_groups, int64_t b_group_stride, int64_t c_group_stride, int accumulate,
                            void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * mom_combine_unpermute -- the combine (paper card, Summary: outputs are
 * combined using the router weights; blog post, "硬件高效實現": summing the
 * weighted per-memory outputs equals reading out the mixed memory):
 *
 *   out[t] = o_sh[t] + sum_j topk_gate[t, j] * o_p[row_of[t*top_k + j]]
 *
 * o_sh, out [n_tok, H, d] (dt); o_p [n_tok*top_k, H, d] (dt); row_of
 * [n_tok*top_k] int32; topk_gate [n_tok, top_k] float32.  float32
 * arithmetic.  An out-of-range row_of entry is recorded
 * (MOM_DEVERR_ROW_INDEX) and contributes nothing.
 * ws: at least MOM_WS_HEADER_BYTES.
 * ---------------------------------------------------------------------- */
mom_status mom_combine_unpermute(const void* o_sh, const void* o_p, const int32_t* row_of,
                                 const float* topk_gate, int64_t n_tok, int top_k, int H, int d,
                                 mom_dtype dt, void* out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * mom_decode_step -- one recurrent decode step, one new token per
 * sequence, constant cost per token (blog post, introduction and
 * "推理效率" (inference efficiency); paper card, Summary: constant-memory
 * inference).  For every sequence b: route x[b]; project q, beta, alpha,
 * the shared memory's k/v and the k/v of the top_k chosen memories; update
 * those top_k + 1 states in place with the rule of mom_gdn_chunk_fwd; and
 * write out[b] = o_sh + sum_j gate_j o_j.  The other memories' states are
 * untouched.
 *
 * x [B, d_model] (dt); weights as in mom_router_topk / mom_kv_proj_grouped;
 * state [B, n_mem+1, H, d, d] float32, slot n_mem being the shared memory,
 * updated in place; out [B, H, d] (dt); topk_idx [B, top_k] int32 or NULL
 * (receives the routing).  `w` is a HOST pointer to a struct of device
 * pointers; it is read during the call only.  ws: mom_decode_workspace_size().
 * ---------------------------------------------------------------------- */
typedef struct mom_weights {
    const void*  w_r;       /* [n_mem, d_model] */
    const float* b_r;       /* [n_mem] or NULL */
    const void*  w_shared;  /* [3*H*d, d_model] */
    const void*  w_gate;    /* [2*H, d_model] */
    const float* A;         /* [H] */
    const float* b_a;       /* [H] */
    const void*  w_kv;      /* [n_mem, 2*H*d, d_model] */
} mom_weights;

size_t mom_decode_workspace_size(int B, int d_model, int H, int d, int n_mem, int top_k);
mom_status mom_decode_step(const void* x, const mom_weights* w, int B, int d_model, int H, int d,
                           int n_mem, int top_k, float scale, mom_dtype dt,
                           float* state, void* out, int32_t* topk_idx,
                           void* ws, size_t ws_bytes, void* stream);
/* Per-memory gates for mom_decode_step_rule (device pointers, as in
 * mom_mem_gate_proj). */
typedef struct mom_memory_gates {
    const void*  w_gate_mem;  /* [n_mem, 2*H, d_model]: rows W_beta^m | W_a^m */
    const float* A_mem;       /* [n_mem, H] */
    const float* b_a_mem;     /* [n_mem, H] */
} mom_memory_gates;

/* mom_decode_step for either memory rule (MOM_RULE_*), and with per-memory
 * gates when `mg` (a HOST pointer, read during the call only) is non-NULL:
 * each routed slot then takes its memory's own beta and alpha, the shared
 * slot the layer's.  mom_decode_step is this with MOM_RULE_GATED_DELTA and
 * mg = NULL.  Same workspace. */
mom_status mom_decode_step_rule(const void* x, const mom_weights* w, const mom_memory_gates* mg,
                                int B, int d_model, int H, int d,
                                int n_mem, int top_k, float scale, mom_dtype dt, mom_rule rule,
                                float* state, void* out, int32_t* topk_idx,
                                void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The Gated DeltaNet block around the memories.  The pages name Gated
 * DeltaNet as each memory's token mixer (the authors' MoM blog post,
 * experiments section) and print nothing of the block that holds it; the
 * calls below are the plain Gated DeltaNet block's steps, in bf16:
 *
 *   q^, k^_sh, v^_sh, g = x [W_q | W_k_sh | W_v_sh | W_g]^T     (unnormalised)
 *   k^_p, v^_p          = x_perm [W_k^m | W_v^m]^T              (mom_block_proj)
 *   q = l2norm(SiLU(conv(q^))), k likewise, v = SiLU(conv(v^))  (mom_short_conv)
 *   the recurrences and the combine as in the layer, then per head
 *   o~ = o / sqrt(mean(o^2) + eps) * w_norm * SiLU(g)           (mom_combine_norm_gate)
 *   y  = o~ W_o^T                                               (mom_linear)
 *
 * conv is a causal depthwise convolution along the rows a recurrence sees
 * (a sequence for the shared q, k, v; a (memory, sequence) segment of the
 * reordered rows for memory m's k, v, with memory m's own filters).
 * ---------------------------------------------------------------------- */

/* mom_block_proj -- the layer's projection GEMM in the block's form: every
 * output unnormalised (the norm follows the convolution) and the output gate
 * as a fourth shared part.  w_shared4 [4*H*d, d_model] (rows W_q | W_k_sh |
 * W_v_sh | W_g); w_kv, perm_token, mem_offset and the routed outputs as in
 * mom_kv_proj_grouped; q, k_sh, v_sh, g [n_tok, H*d]; k_p, v_p [n_tok*top_k,
 * H*d].  bf16 only (MOM_ERR_UNSUPPORTED otherwise), H*d a multiple of 256,
 * d_model of 64; every pointer 16-byte aligned.  ws: MOM_WS_HEADER_BYTES. */
mom_status mom_block_proj(const void* x, const int32_t* perm_token, const int32_t* mem_offset,
                          const void* w_shared4, const void* w_kv, mom_dtype dt,
                          int64_t n_tok, int d_model, int H, int d, int n_mem, int top_k,
                          void* q, void* k_sh, void* v_sh, void* g, void* k_p, void* v_p,
                          void* ws, size_t ws_bytes, void* stream);

/* mom_short_conv -- out[r, c] = SiLU(sum_{j<width} w[grp, width-1-j, c] *
 * z[r-j, c]) over the taps with r-j >= the start of r's segment, then, when
 * l2norm is 1, each head of head_dim channels divided by sqrt(|.|^2 +
 * 1e-6).  Segment s covers rows seg_cu[s] .. seg_cu[s+1]-1 (device int32
 * [n_seg+1], non-decreasing, seg_cu[n_seg] <= n_rows); its filters are group
 * grp = s / seg_per_group (< n_groups).  Rows outside every segment are not
 * written.  z, out [n_rows, channels] bf16, distinct buffers, 16-byte
 * aligned; w [n_groups, width, channels] float32, tap-major (w[grp, j, c];
 * tap width-1 multiplies the current row), 16-byte aligned.  channels a multiple of 8; width 1..4; with l2norm, head_dim
 * a power of two in 8..256 dividing channels.  Corrupt segment bounds are
 * recorded in ws (MOM_DEVERR_SEGMENT).  ws: MOM_WS_HEADER_BYTES. */
mom_status mom_short_conv(const void* z, int64_t n_rows, int channels, const int32_t* seg_cu, int n_seg,
                          int seg_per_group, int n_groups, const float* w, int width, int head_dim,
                          int l2norm, mom_dtype dt, void* out, void* ws, size_t ws_bytes, void* stream);

/* One convolution of a batch (fields as the arguments of mom_short_conv). */
typedef struct mom_conv_problem {
    const void*    z;
    void*          out;
    int64_t        n_rows;
    const int32_t* seg_cu;
    int            n_seg;
    int            seg_per_group;
    int            n_groups;
    const float*   w;
    int            l2norm;
} mom_conv_problem;

/* mom_short_conv_batch -- 1..8 convolutions of the same channel count, width
 * and head_dim in one launch (the block's five: q, k_sh, v_sh over the
 * sequences, k_p, v_p over the memory segments).  `problems` is a HOST
 * array read during the call only; each problem is validated as in
 * mom_short_conv. */
mom_status mom_short_conv_batch(const mom_conv_problem* problems, int n_problems, int channels, int width,
                                int head_dim, mom_dtype dt, void* ws, size_t ws_bytes, void* stream);

/* mom_combine_norm_gate -- the combine of mom_combine_unpermute followed,
 * per head of d channels, by the block's gated RMS norm:
 *   o = o_sh[t] + sum_j topk_gate[t,j] o_p[row_of[t*top_k+j]],
 *   out[t] = o / sqrt(mean(o^2) + eps) * w_norm * SiLU(g[t]).
 * o_sh, g, out [n_tok, H*d], o_p [n_tok*top_k, H*d] bf16; w_norm [d]
 * float32; d a power of two in 8..256; every array 16-byte aligned.  Row
 * errors as in the combine.  top_k = 0: o = o_sh (o_p, row_of and
 * topk_gate unused): the norm and gate of an output combined elsewhere. */
mom_status mom_combine_norm_gate(const void* o_sh, const void* o_p, const int32_t* row_of,
                                 const float* topk_gate, const void* g, const float* w_norm, float eps,
                                 int64_t n_tok, int top_k, int H, int d, mom_dtype dt, void* out,
                                 void* ws, size_t ws_bytes, void* stream);

/* mom_linear -- y = x w^T on the tensor cores (the block's output
 * projection): x [n_rows, k_in], w [n_out, k_in], y [n_rows, n_out], bf16,
 * fp32 accumulation; k_in a multiple of 64, n_out of 256; 16-byte aligned.
 * ws: MOM_WS_HEADER_BYTES. */
mom_status mom_linear(const void* x, const void* w, mom_dtype dt, int64_t n_rows, int k_in, int n_out, void* y,
                      void* ws, size_t ws_bytes, void* stream);

/* The block's weights for its decode step (device pointers). */
typedef struct mom_block_weights {
    const void*  w_shared4;   /* [4*H*d, d_model]: W_q | W_k_sh | W_v_sh | W_g */
    const void*  w_o;         /* [d_model, H*d] */
    const float* conv_q;      /* [width, H*d] tap-major (tap width-1: the current row) */
    const float* conv_k_sh;   /* [width, H*d] */
    const float* conv_v_sh;   /* [width, H*d] */
    const float* conv_k;      /* [n_mem, width, H*d] */
    const float* conv_v;      /* [n_mem, width, H*d] */
    const float* w_norm;      /* [d] */
} mom_block_weights;

/* mom_block_decode_step -- one new token per sequence through the block
 * (constant-cost inference: the blog post's introduction, "推理效率"; the
 * paper card, Summary): router, reordering and gates as mom_decode_step; the
 * block's raw projections and output gate; one row of each short
 * convolution from the sequence's window (the shared q, k, v) or from the
 * (sequence, memory) window of each routed memory (its k, v); the k+1
 * recurrence steps and the combine; the gated per-head RMS norm (eps); W_o.
 *   state     [B, n_mem+1, H, d, d] float32, as mom_decode_step, in place;
 *   conv_sh   [B, 3, width-1, H*d] (dt): the raw q, k_sh, v_sh of each
 *             sequence's last width-1 tokens, oldest first, zero before its
 *             start; updated in place;
 *   conv_mem  [B, n_mem, 2, width-1, H*d] (dt): the raw k, v of the last
 *             width-1 tokens of each sequence routed to each memory; the
 *             windows of the memories a token is not routed to are kept;
 *   y         [B, d_model] (dt); topk_idx [B, top_k] or NULL; mg as in
 *             mom_decode_step_rule (a HOST pointer) or NULL.
 * bf16 only, width 2..4 (MOM_ERR_UNSUPPORTED otherwise); H*d a multiple of
 * 256, d_model of 256; ws: mom_block_decode_workspace_size(). */
size_t mom_block_decode_workspace_size(int B, int d_model, int H, int d, int n_mem, int top_k);
mom_status mom_block_decode_step(const void* x, const mom_weights* w, const mom_block_weights* bw,
                                 const mom_memory_gates* mg, int width, float eps, int B, int d_model, int H, int d,
                                 int n_mem, int top_k, float scale, mom_dtype dt, mom_rule rule, float* state,
                                 void* conv_sh, void* conv_mem, void* y, int32_t* topk_idx, void* ws,
                                 size_t ws_bytes, void* stream);

/* mom_block_conv_state -- the convolution windows a block forward over
 * whole sequences leaves, for mom_block_decode_step: conv_sh[s, i, j] = raw
 * row cu_seqlens[s+1] - (width-1) + j of q, k_sh, v_sh (i = 0, 1, 2), zero
 * when it falls before the sequence's start; conv_mem[s, m, i, j] the same
 * over memory m's segment seg_cu[m*n_seq + s] .. of k_p, v_p (i = 0, 1).
 * q_raw, k_sh_raw, v_sh_raw [n_tok, channels], k_p_raw, v_p_raw
 * [n_tok*top_k, channels] (dt): the forward's unnormalised projections
 * (mom_block_proj); cu_seqlens [n_seq+1], seg_cu [n_mem*n_seq+1] device
 * int32 (corrupt bounds are recorded in ws and give zero windows).  bf16
 * only, width 2..4. */
mom_status mom_block_conv_state(const void* q_raw, const void* k_sh_raw, const void* v_sh_raw, const void* k_p_raw,
                                const void* v_p_raw, int64_t n_tok, int top_k, const int32_t* cu_seqlens,
                                const int32_t* seg_cu, int n_seq, int n_mem, int channels, int width, mom_dtype dt,
                                void* conv_sh, void* conv_mem, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The block's reverse pass (training is the pages' main workload: the paper
 * card, Key points).  With the forward of the calls above:
 * ---------------------------------------------------------------------- */

/* mom_norm_gate_bwd -- the adjoint of mom_combine_norm_gate: per head of the
 * combined output o (recomputed from o_sh and the routed rows), r =
 * 1/sqrt(mean(o^2) + eps), n = o r, s = SiLU(g), dn = d_y w_norm s:
 *   d_o = r (dn - n mean(dn n))                 [n_tok, H*d] (dt)
 *   dg[t*ldg + c] = d_y n w_norm SiLU'(g)        float32
 *   dw_norm = sum over tokens and heads of d_y n s   [d] float32 (overwritten)
 * The other arguments as mom_combine_norm_gate (d_y is the adjoint of its
 * output).  bf16 only. */
mom_status mom_norm_gate_bwd(const void* o_sh, const void* o_p, const int32_t* row_of, const float* topk_gate,
                             const void* g, const float* w_norm, float eps, const void* d_y, int64_t n_tok,
                             int top_k, int H, int d, mom_dtype dt, void* d_o, float* dg, int64_t ldg,
                             float* dw_norm, void* ws, size_t ws_bytes, void* stream);

/* One convolution's adjoint (the forward: one problem of mom_short_conv_batch):
 * out = [l2norm] SiLU(a), a = conv(z). */
typedef struct mom_conv_bwd_problem {
    const void*    z;         /* the forward's raw rows [n_rows, channels] (dt) */
    const float*   dout;      /* adjoint of out [n_rows, channels] */
    float*         da;        /* reserved: not read or written (may be NULL) */
    float*         dz;        /* adjoint of z: dz[r*ldz + col0 + c], overwritten for rows in a segment */
    int64_t        ldz;
    int64_t        col0;
    int64_t        n_rows;
    const int32_t* seg_cu;    /* as the forward */
    int            n_seg;
    int            seg_per_group;
    int            n_groups;
    const float*   w;         /* the forward's filters [n_groups, width, channels] */
    float*         dw;        /* their adjoint, same layout (overwritten) */
    int            l2norm;
} mom_conv_bwd_problem;

/* mom_short_conv_bwd -- for 1..8 problems of the same channel count, width
 * and head_dim: da = the adjoint of a (a recomputed from z, the L2 norm's
 * adjoint per head when l2norm, then SiLU's, kept on chip); dz[t] = sum_j
 * w[W-1-j] da[t+j] over the rows t+j in t's segment; dw[grp][W-1-j] =
 * sum_t da[t] z[t-j].  `problems` is a HOST array read during the call.
 * bf16 z only.  dout may alias nothing that the call writes. */
mom_status mom_short_conv_bwd(const mom_conv_bwd_problem* problems, int n_problems, int channels, int width,
                              int head_dim, mom_dtype dt, void* ws, size_t ws_bytes, void* stream);

/* mom_convert -- dst[i] = src[i] converted between float32 and bf16 (round
 * to nearest even), i < n. */
mom_status mom_convert(const void* src, mom_dtype src_dt, void* dst, mom_dtype dst_dt, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOM_H */
