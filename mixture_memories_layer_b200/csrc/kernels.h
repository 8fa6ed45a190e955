// Internal launchers of the MoM kernels (host side).  The public C ABI in
// mom.h validates arguments and calls these; they only launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mom.h"

namespace mom {

// Counts every kernel launch (mom_launch_count).
void count_launches(int n);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device.  The limit is a per-device setting, so it is set once per
// (kernel, device): `done` holds one bit per device already set (devices
// 0..63; others are set on every call).
cudaError_t smem_optin(const void* func, int bytes, unsigned long long* done);

// tma_host.cu: tensor maps for bf16 row-major matrices (128-byte swizzle,
// boxes of box_rows x box_cols with box_cols * 2 == 128 bytes) and the
// device-generation check of the tcgen05 paths.
bool tma_available();
bool make_tma_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t row_pitch_elems,
                      uint32_t box_cols, uint32_t box_rows);
// Same without swizzle (row-major shared tile, e.g. an output staging tile).
bool make_tma_2d_bf16_plain(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t row_pitch_elems,
                            uint32_t box_cols, uint32_t box_rows);
bool device_is_sm100();

// router.cu
cudaError_t launch_router(const void* x, const void* w_r, const float* b_r, int dt, int64_t n_tok, int D,
                          int M, int K, int32_t* idx, float* gate, float* logits, cudaStream_t st);
// mem_gates.cu: per-memory gates of the routed rows (beta_p, log_alpha_p [n_rows, H])
cudaError_t launch_mem_gate_proj(const void* x, const int32_t* perm, const int32_t* mem_offset, const void* w_gate_mem,
                                 const float* A_mem, const float* b_a_mem, int dt, int64_t n_tok, int64_t n_rows, int D,
                                 int H, int M, float* beta, float* log_alpha, void* err, cudaStream_t st,
                                 const int32_t* group_mem = nullptr, int n_w = 0);
cudaError_t launch_gate_proj(const void* x, const void* w_gate, const float* A, const float* b_a, int dt,
                             int64_t n_tok, int D, int H, float* beta, float* log_alpha, void* err, cudaStream_t st);

// skinny.cu: the same two products for bf16 inputs, four threads per token
// and the weights staged in shared memory (used when skinny_ok holds)
bool skinny_ok(int dt, int D, int ncol);
cudaError_t launch_router_skinny(const void* x, const void* w_r, const float* b_r, int64_t n_tok, int D, int M,
                                 int K, int32_t* idx, float* gate, float* logits, cudaStream_t st);
cudaError_t launch_gate_skinny(const void* x, const void* w_gate, const float* A, const float* b_a, int64_t n_tok,
                               int D, int H, float* beta, float* log_alpha, void* err, cudaStream_t st);

// permute.cu
// `err` is the workspace whose header receives device error records;
// `scratch` (permute_scratch_bytes) holds the tile counts.
size_t permute_scratch_bytes(int64_t n_tok, int M);
cudaError_t launch_permute(const int32_t* idx, int64_t n_tok, int K, int M, const int32_t* cu_seqlens, int S,
                           int32_t* perm_token, int32_t* row_of, int32_t* mem_offset, int32_t* seg_cu,
                           void* err, void* scratch, cudaStream_t st);

// proj_simt.cu: grouped projections on CUDA cores (float32 mode, and any
// shape the tensor-core path does not take)
enum ProjPart { PROJ_SHARED = 1, PROJ_ROUTED = 2 };
struct ProjArgs {
    const void* x;                // [n_tok, D]
    const int32_t* perm_token;    // routed row -> x row (null: row r reads x row r)
    const int32_t* mem_offset;    // group g: routed rows mem_offset[g] .. mem_offset[g+1]
    const void* w_shared;
    const void* w_kv;
    int64_t n_tok;
    int D, H, d, M, K;
    void *q, *k_sh, *v_sh, *k_p, *v_p;
    void* ws;
    // which problems run (PROJ_SHARED | PROJ_ROUTED)
    int parts = PROJ_SHARED | PROJ_ROUTED;
    // routed groups: n_groups (0: M, one per memory) with group g using
    // memory group_mem[g]'s weights (null: memory g); n_routed routed rows
    // (< 0: n_tok * K)
    const int32_t* group_mem = nullptr;
    int n_groups = 0;
    int64_t n_routed = -1;
    // optional: sqrt(|z|^2 + 1e-6) of every normalised (row, head) -- the
    // lengths the backward of the norm needs: [n_tok, H] for q and k_sh,
    // [routed rows, H] for k_p
    float* q_norm = nullptr;
    float* k_sh_norm = nullptr;
    float* k_p_norm = nullptr;
    // the Gated DeltaNet block's form: raw = 1 leaves q, k_sh and k_p
    // unnormalised (the norm follows the short convolution); g non-null adds
    // the output gate x W_g^T as a fourth shared part (w_shared holds
    // [W_q | W_k_sh | W_v_sh | W_g]); plain_n > 0 makes the shared problem
    // one plain product y = x w_shared^T of plain_n columns, written to q
    int raw = 0;
    void* g = nullptr;
    int plain_n = 0;
    __host__ __device__ int groups() const { return n_groups > 0 ? n_groups : M; }
    __host__ __device__ int64_t routed_rows() const { return n_routed >= 0 ? n_routed : n_tok * K; }
};
cudaError_t launch_proj_simt(const ProjArgs& a, int dt, cudaStream_t st);

// proj_tc.cu: grouped projections on the tcgen05 tensor cores (bf16)
bool proj_tc_supported(const ProjArgs& a, int dt);
cudaError_t launch_proj_tc(const ProjArgs& a, cudaStream_t st);

// gdn_recurrent.cu: token-serial Gated DeltaNet on CUDA cores
enum GdnPhase { GDN_PREP = 1, GDN_STATE = 2 };
struct GdnArgs {
    const void* q;
    const int32_t* qidx;
    const void* k;
    const void* v;
    const float* beta;
    const float* log_alpha;
    const int32_t* seg_cu;
    int n_seg;
    int64_t n_rows, n_q_rows;
    int H, d;
    float scale;
    const float* h0;
    float* h_final;
    void* o;
    void* ws;
    size_t ws_bytes;
    // GDN_PREP: the state-independent per-chunk work; GDN_STATE: the serial
    // walk over the chunks (reads what GDN_PREP left in ws); both by default
    int phase = GDN_PREP | GDN_STATE;
    // MOM_RULE_GATED_DELTA or MOM_RULE_GATED_LINEAR
    int rule = MOM_RULE_GATED_DELTA;
    // 0: beta / log_alpha [n_q_rows, H], read through qidx like q; 1: one
    // gate per row of k / v ([n_rows, H], the per-memory gates)
    int gates_by_row = 0;
};
cudaError_t launch_gdn_recurrent(const GdnArgs& a, int dt, cudaStream_t st);

// gdn_bwd.cu: reverse pass of the recurrence (both rules), token-serial fp32
struct GdnBwdArgs {
    const void* q;
    const int32_t* qidx;
    const void* k;
    const void* v;
    const float* beta;
    const float* log_alpha;
    const int32_t* seg_cu;
    int n_seg;
    int64_t n_rows, n_q_rows;
    int H, d;
    float scale;
    int rule;
    int gates_by_row;
    const float* h0;          // [n_seg, H, d, d] or null
    const void* d_o;          // [n_rows, H, d] (dt)
    const float* dh_final;    // [n_seg, H, d, d] or null
    float* dq;                // [n_rows, H, d], per row
    float* dk;
    float* dv;
    float* dbeta;             // [n_rows, H], per row
    float* dlog_alpha;
    float* dh0;               // [n_seg, H, d, d] or null
    void* ws;
};
size_t gdn_bwd_ws_bytes(int64_t n_rows, int n_seg, int H, int d);
cudaError_t launch_gdn_bwd(const GdnBwdArgs& a, int dt, cudaStream_t st);

// layer_bwd.cu: the layer's backward around the recurrences
cudaError_t launch_combine_bwd(const void* dout, const void* o_p, const int32_t* row_of, const float* gate,
                               int64_t n_tok, int K, int HD, int64_t n_rows, int dt, void* do_p, float* dgate,
                               void* err, cudaStream_t st);
cudaError_t launch_router_bwd(const int32_t* idx, const float* gate, const float* dgate, int64_t n_tok, int K, int M,
                              float* dlogits, void* err, cudaStream_t st);
cudaError_t launch_rows_sum(const float* src, int64_t n_src, const int32_t* row_of, int K, const float* base,
                            int64_t n_tok, int W, float* dst, void* err, cudaStream_t st);
cudaError_t launch_l2norm_bwd(const void* y, const float* dy, const float* nrm, int64_t rows, int H, int d, int dt,
                              float* dz, int64_t ldz, int64_t col0, cudaStream_t st);
cudaError_t launch_gates_bwd(const float* beta, const float* la, const float* dbeta, const float* dla, const float* A,
                             const int32_t* goff, int n_groups, int64_t n, int H, float* dz, int64_t ldz,
                             int64_t col_b, int64_t col_a, float* dala, cudaStream_t st);
cudaError_t launch_col_sums(const float* a, int64_t rows, int64_t lda, int64_t C, const int32_t* goff, int n_groups,
                            float* out, cudaStream_t st);
cudaError_t launch_gemm_grouped(int trans_a, const float* A, int64_t lda, const void* B, int64_t ldb, int dt,
                                const int32_t* b_rows, int64_t n_b_rows, float* C, int64_t ldc, int64_t M, int64_t N,
                                int64_t K, int64_t total_rows, const int32_t* goff, const int32_t* gmem, int n_groups,
                                int64_t b_group_stride, int64_t c_group_stride, int accumulate, void* err,
                                cudaStream_t st);

// gdn_chunk_tc.cu: chunked Gated DeltaNet on the tcgen05 tensor cores (bf16)
bool gdn_tc_supported(const GdnArgs& a, int dt);
size_t gdn_tc_ws_bytes(int64_t n_rows, int n_seg, int H, int d);
cudaError_t launch_gdn_tc(const GdnArgs& a, cudaStream_t st);

// copy_rows.cu: dst row i = bytes of src row idx[i] (or i), 16-byte granules
cudaError_t launch_copy_rows(const void* src, int64_t n_src, int64_t src_stride, int64_t src_off, const int32_t* idx,
                             int64_t n_rows, int64_t row_bytes, void* dst, int64_t dst_stride, int64_t dst_off,
                             void* err, cudaStream_t st);

// combine.cu
cudaError_t launch_combine(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                           int64_t n_tok, int K, int H, int d, int dt, void* out, void* ws, cudaStream_t st);

// decode.cu: the state pass of one decode step with the combine fused
struct DecodeArgs {
    const void *q, *k_sh, *v_sh, *k_p, *v_p;
    const float *beta, *log_alpha, *gate;
    const int32_t *idx, *row_of;
    int B, H, d, M, K;
    float scale;
    float* state;
    void* out;
    void* ws;
    int rule = MOM_RULE_GATED_DELTA;
    // per-memory gates of the routed slots, [B*K, H] by reordered row (row_of),
    // or null: every slot takes the token's beta / log_alpha
    const float *beta_p = nullptr, *log_alpha_p = nullptr;
};
cudaError_t launch_decode_state(const DecodeArgs& a, int dt, cudaStream_t st);

// conv.cu: the block's short causal convolutions (SiLU, optional per-head L2
// norm), up to 8 problems of the same channel count per launch
struct ConvProblem {
    const void* z;
    void* out;
    int64_t n_rows;
    const int32_t* seg_cu;
    int n_seg, seg_per_group, n_groups;
    const float* w;               // [n_groups, W, C] (tap-major)
    int l2;
};
cudaError_t launch_short_conv(const ConvProblem* problems, int n, int C, int W, int d, void* err, cudaStream_t st);
// one decode row per sequence through the five convolutions, windows updated in place
struct ConvStepArgs {
    const bf16* z[5];             // raw rows: q, k_sh, v_sh [B, C]; k_p, v_p [B*K, C]
    bf16* out[5];
    const float* w[5];            // tap-major filters: [W, C] (shared), [M, W, C] (memories)
    bf16* st_sh;                  // [B][3][W-1][C]
    bf16* st_mem;                 // [B][M][2][W-1][C]
    const int32_t* perm;          // routed row -> sequence
    const int32_t* mem_offset;    // [M + 1]
    int B, K, M, C, d;
    void* err;
};
cudaError_t launch_conv_step(const ConvStepArgs& a, int W, cudaStream_t st);
// the windows a forward leaves
struct ConvStateArgs {
    const bf16* z[5];             // raw forward rows: q, k_sh, v_sh [n_tok, C]; k_p, v_p [n_rows, C]
    bf16* st_sh;
    bf16* st_mem;
    const int32_t* cu;            // [S + 1]
    const int32_t* seg_cu;        // [M * S + 1]
    int S, M, C, W;
    int64_t n_tok, n_rows;
    void* err;
};
cudaError_t launch_conv_state(const ConvStateArgs& a, cudaStream_t st);
// combine.cu: the combine with the block's gated per-head RMS norm
cudaError_t launch_combine_norm_gate(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                                     const void* g, const float* w_norm, float eps, int64_t n_tok, int K, int H,
                                     int d, void* out, void* ws, cudaStream_t st);

// block_bwd.cu: the block's reverse pass
cudaError_t launch_norm_gate_bwd(const void* o_sh, const void* o_p, const int32_t* row_of, const float* gate,
                                 const void* g, const float* w_norm, float eps, const void* dy, int64_t n_tok, int K,
                                 int H, int d, void* d_o, float* dg, int64_t ldg, float* dw_norm, void* ws,
                                 cudaStream_t st);
struct ConvBwdArgs {
    const void* z;                // raw rows [n_rows, C] (bf16)
    const float* dout;            // adjoint of the convolution's (normalised) output [n_rows, C]
    float* da;                    // scratch [n_rows, C]
    float* dz;                    // adjoint of the raw rows: dz[r * ldz + col0 + c]
    int64_t ldz, col0, n_rows;
    const int32_t* seg_cu;
    int n_seg, seg_per_group, n_groups;
    const float* w;               // [n_groups, W, C] tap-major
    float* dw;                    // [n_groups, W, C] (zeroed, then summed into)
    int l2;
};
cudaError_t launch_conv_bwd(const ConvBwdArgs* problems, int n, int C, int W, int d, void* err, cudaStream_t st);
cudaError_t launch_convert(const void* src, int src_dt, void* dst, int dst_dt, int64_t n, cudaStream_t st);

}  // namespace mom
