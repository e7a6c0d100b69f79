// kernels.cuh -- argument blocks and launchers of the libmoe kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Launch `kernel` on `st`; pdl: with programmatic stream serialization, so the
// launch overlaps the previous kernel of the stream (the kernel itself waits
// for that kernel's completion before touching memory).  The first kernel of
// an entry point launches without it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 bool pdl, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

struct RouterArgs {
    const void *x;               // [T, d] bf16 or fp32
    const float *Wr;             // [d, E]
    const float *logit_bias;     // [E] or null
    const float *sel_bias;       // [E] or null
    int32_t *idx;                // [T, k]
    float *gate;                 // [T, k]
    float *logits_out;           // [T, E] or null
    float *psum;                 // [router_blocks(T, bf16), E]
    int T, d, E, k, score, renorm;
    void *wsplit;                // bf16 layers: [3, E, d] scratch for the split W_r
    float *logits_ws;            // bf16 layers: [router_logit_splits_max(T), T, E] scratch for
                                 // the (partial) logits
    int32_t *status;             // workspace status word
    int num_sms;
    bool pdl;                    // the first launch overlaps the stream's previous kernel
    bool split_ready;            // bf16 layers: wsplit already holds this W_r's split (a frozen router)
};
// W_r -> its exact three-term bf16 split in a.wsplit (bf16 layers).  router_sm100.cu.
cudaError_t launch_router_split(const RouterArgs &a, cudaStream_t st);
// Rows of the per-block score sums: 64 tokens per block for bf16 layers,
// 32 for fp32 layers.
int router_blocks(int T, bool bf16);
size_t router_split_bytes(int d, int E);
// K-split count of the tensor-core logits GEMM: the bound the workspace is
// sized for, and the count used on a GPU with num_sms SMs.
int router_logit_splits_max(int T);
int router_logit_splits(int T, int d, int num_sms);
cudaError_t launch_router(const RouterArgs &a, bool bf16, cudaStream_t st);
cudaError_t launch_router_logits_tc(const RouterArgs &a, float *out, int splits, cudaStream_t st);

struct DispatchArgs {
    const void *x;               // [T, d]
    const int32_t *idx;          // [T, k]
    const float *gate;           // [T, k]
    int32_t *chunk_cnt;          // [E, nchunks] scratch
    int32_t *chunk_base;         // [E, nchunks] scratch
    int32_t *counts, *kept, *offsets;   // [E], [E], [E+1]
    int32_t *row_of;             // [T, k]
    int32_t *row_token;          // [T*k]
    float *row_gate;             // [T*k]
    void *x_perm;                // [T*k, d]
    const float *x_scale;        // [T] per-row scales of e4m3 x, or null
    float *row_scale;            // [T*k]: x_scale of each packed row's token, or null
    int32_t *n_dropped;          // device scalar or null
    int32_t *status;             // workspace status word
    int T, d, E, k, capacity;    // capacity < 0: unlimited
    // Optional (loss != null): the balance statistics, f and P computed in the
    // scan kernel from the router's per-block score sums, the loss added by
    // the permute kernel (or the empty-input kernel).
    const float *psum;           // [nblk, E]
    float *f, *P;                // [E]
    double *loss;                // device scalar
    double *contrib;             // [E] scratch: f_e P_e
    int nblk;
    bool pdl;                    // the first launch overlaps the stream's previous kernel
};
int dispatch_chunks(int T);
// x_bytes: bytes per element of x and x_perm (4 fp32, 2 bf16, 1 e4m3 codes)
cudaError_t launch_dispatch(const DispatchArgs &a, int x_bytes, cudaStream_t st);

// Grouped expert FFN.  Routed group g < n_groups holds rows offsets[g] ..
// offsets[g+1] of x_perm / H / y_perm and uses weight expert g % E (n_groups
// = E: group g is expert g; rows gathered from several sources come as
// n_groups = sources * E runs of all E experts); group n_groups is the shared
// expert (rows 0..T-1 of x, rows shared_base.. of H / y_perm).
struct FfnArgs {
    const void *x_perm;          // [routed_rows, d]
    const void *x;               // [T, d] (shared expert) or null
    const int32_t *offsets;      // [E+1]
    const float *row_gate;       // [T*k]
    const void *W1, *Wu, *W2;    // [E, F, d], [E, F, d] or null, [E, d, F]
    const float *b1, *b2;        // [E, F], [E, d] or null
    const void *Wsg, *Wsu, *Wsd; // [S, d], [S, d] or null, [d, S]
    void *H;                     // [T*k (+T), max(F, S)] scratch, row stride hF
    void *y_perm;                // [T*k (+T), d]
    int32_t *status;
    int T, d, E, k, F, S, act;   // S = d_ff_shared (0: none); E: experts in the weights
    int n_groups;                // routed groups (a multiple of E)
    int64_t routed_rows;         // rows of x_perm / routed rows of H and y_perm
    int hF;                      // row stride of H in elements
    int64_t shared_base;         // = T*k
    int num_sms;
    bool pdl;                    // the first launch overlaps the stream's previous kernel
    // e4m3 experts (bf16 layers): x_perm and x hold e4m3 codes with per-row
    // scales, the weights e4m3 codes with per-output-channel scales; the
    // first GEMM's bf16 H is quantized per row into H8 for the second GEMM
    bool f8;
    const float *xperm_scale;    // [T*k] scale of each packed row
    const float *x_scale;        // [T] (shared expert rows)
    const float *W1s, *Wus, *W2s;      // [E, F], [E, F], [E, d]
    const float *Wsgs, *Wsus, *Wsds;   // [S], [S], [d]
    uint8_t *H8;                 // [T*k (+T), hF] codes
    float *h_scale;              // [T*k (+T)]
    // training forward (bf16 experts): the first GEMM also stores the
    // pre-activations in bf16 -- SwiGLU [rows, 2F] (G | U), GELU [rows, F]
    // (W_1 x + b_1) -- routed rows in pre, the shared expert's T rows in
    // pre_s ([T, 2S] or [T, S]); null for inference
    void *pre, *pre_s;
};
// TMA tile map (128-byte swizzle) of a tensor [outer][mid][inner] (inner
// contiguous) of bf16 (esize 2) or 8-bit codes (esize 1), box {one 128-byte
// row of elements, box_mid(, 1)}; rank 2 maps ignore `outer`.  ffn_sm100.cu.
bool make_map(CUtensorMap *m, int rank, const void *base, uint64_t inner, uint64_t mid, uint64_t outer,
              uint64_t mid_stride_elems, uint64_t outer_stride_elems, uint32_t box_mid, int esize = 2);
cudaError_t launch_ffn_f32(const FfnArgs &a, cudaStream_t st);
cudaError_t launch_ffn_bf16(const FfnArgs &a, cudaStream_t st);

// Block-scaled (MX) e4m3 quantization of bf16 rows (row0 + r for r < rows,
// or fewer when rows_limit points at a smaller device count): codes [.., ld_out]
// and one E8M0 scale byte per 32 values [.., ld_scale].  cols % 32 == 0,
// ld_out % 8 == 0.  mx_sm100.cu.
struct QuantMxArgs {
    const __nv_bfloat16 *in;
    int64_t ld_in;
    uint8_t *out;
    int64_t ld_out;
    uint8_t *scale;
    int64_t ld_scale;
    int64_t rows, row0;
    int cols;
    const int32_t *rows_limit;
    int num_sms;
    bool pdl;
};
cudaError_t launch_quant_mx(const QuantMxArgs &a, cudaStream_t st);
// dst[r] = src[row_token[r]] for r < min(*count, max_rows), rows of ld bytes
// (ld % 16 == 0): the MX scale rows of the packed rows.  mx_sm100.cu.
cudaError_t launch_mx_gather_rows(const uint8_t *src, uint8_t *dst, int64_t ld, const int32_t *row_token,
                                  const int32_t *count, int64_t max_rows, int num_sms, cudaStream_t st);

// The grouped FFN with MX experts (mx_sm100.cu).  Every scale array has rows
// of sld bytes (sld % 16 == 0, at least its K / 32); K dimensions (d, F, S)
// are multiples of 128.
struct FfnMxArgs {
    const uint8_t *x_perm; const uint8_t *xs_perm;    // [routed_rows, d] codes, [routed_rows, sld] scales
    const uint8_t *x; const uint8_t *xs;              // [T, d], [T, sld] (shared expert) or null
    const int32_t *offsets;                           // [E+1]
    const float *row_gate;                            // [routed_rows]
    const uint8_t *W1, *W1s, *Wu, *Wus;               // [E, F, d] codes, [E, F, sld] scales
    const uint8_t *W2, *W2s;                          // [E, d, F], [E, d, sld]
    const float *b1, *b2;                             // GELU biases or null
    const uint8_t *Wsg, *Wsgs, *Wsu, *Wsus, *Wsd, *Wsds;
    __nv_bfloat16 *H;                                 // [routed_rows (+T), hF]
    uint8_t *H8, *Hs;                                 // codes [.., hF], scales [.., sld]
    __nv_bfloat16 *y_perm;                            // [routed_rows (+T), d]
    int32_t *status;
    int T, d, E, F, S, act;
    int64_t routed_rows;
    int hF;
    int64_t shared_base;                              // first shared row of H / y_perm
    int sld;
    int num_sms;
};
cudaError_t launch_ffn_mx(const FfnMxArgs &a, cudaStream_t st);
// INT4 weight-only experts through the same arguments: x_perm / x hold bf16
// rows, W* packed INT4 codes [.., N, K/2] (low nibble = even input, nibble =
// q + 8), W*s bf16 scale bytes [.., N, sld] (one scale per 128 inputs); H
// stays bf16 between the GEMMs.  mx_sm100.cu.
cudaError_t launch_ffn_w4(const FfnMxArgs &a, cudaStream_t st);

// One GEMM of the INT4 weight-only grouped FFN on CTA pairs (M = 256, N =
// 256): every group's 256-row blocks and a last block of more than 128 rows
// (a last block of 1..128 rows is left to the 1-CTA kernel).  A / As: TMA
// maps of the bf16 activations (128-byte swizzle, box 64 x 128).  Packed
// weights: codes [.., N, K/2] bytes and bf16 scale bytes [.., N, sld], read by
// the kernel's decode warps: c / sc routed (SwiGLU: the gate projection),
// c2 / sc2 the SwiGLU up projection, cs* the shared expert's.  out: bf16
// [out_rows, out_cols] with row stride ldo.  mode: 0 SwiGLU, 1 GELU (+ bias),
// 2 down (+ bias, times row_gate).  ffn_sm100.cu.
struct W4PairArgs {
    CUtensorMap A, As;
    const uint8_t *c, *c2, *cs, *cs2;
    const uint8_t *sc, *sc2, *scs, *scs2;
    int64_t sld;
    const int32_t *offsets;
    const float *bias;           // [E, N_routed] or null
    const float *row_gate;       // mode 2: [rows]
    __nv_bfloat16 *out;
    uint64_t out_cols, out_rows;
    int32_t *status;
    int mode, E, T, has_shared, K_routed, K_shared, N_routed, N_shared, ldo;
    int64_t shared_a_row, shared_out_row;
    int num_sms;
    bool pdl;
};
cudaError_t launch_w4_gemm_pair(const W4PairArgs &a, cudaStream_t st);

// Training forward -> backward hand-over of the expert pre-activations
// (moe_api.cu): moe_forward_train records that it left them in a backward
// workspace for a forward workspace and config; moe_backward takes the record
// (true: skip the recompute) and drops any other for its workspace; every
// call that rewrites a forward workspace's packed rows or hidden activation,
// or reinitialises a workspace, forgets the records that involve it.
void note_saved_preacts(const void *bwd_ws, const void *fwd_ws, const moe_config &cfg);
bool take_saved_preacts(const void *bwd_ws, const void *fwd_ws, const moe_config &cfg);
void forget_saved_preacts(const void *ws);
// Where moe_backward keeps the pre-activations in its workspace (bwd_api.cu).
bool bwd_preact_buffers(const moe_config *cfg, void *ws, void **GU, void **GUs);

// Per-row e4m3 quantization of bf16 rows (row0 + r for r < rows, or fewer
// when rows_limit points at a smaller device count): in [.., ld_in] bf16,
// out [.., ld_out] e4m3 codes, scale [..] fp32.  cols % 8 == 0.
struct QuantArgs {
    const __nv_bfloat16 *in;
    int64_t ld_in;
    uint8_t *out;
    int64_t ld_out;
    float *scale;
    int64_t rows, row0;
    int cols;
    const int32_t *rows_limit;   // device count of rows to quantize, or null
    int num_sms;
    bool pdl;                    // the launch overlaps the stream's previous kernel
};
cudaError_t launch_quant_rows(const QuantArgs &a, cudaStream_t st);

struct CombineArgs {
    const void *y_perm;
    const int32_t *row_of;
    void *y;
    int32_t *status;
    int T, d, k, has_shared;
    int64_t rows_routed;         // T*k: valid routed row indices are below it
    int num_sms;
    bool pdl;                    // the launch overlaps the stream's previous kernel
};
cudaError_t launch_combine(const CombineArgs &a, bool bf16, cudaStream_t st);

struct BalanceArgs {
    const int32_t *counts;
    const float *psum;
    float *f, *P;
    double *loss;
    int T, E, k, nblk;
};
cudaError_t launch_balance(const BalanceArgs &a, cudaStream_t st);

cudaError_t launch_bias_update(const int32_t *counts, float *bias, double gamma, int T, int k, int E,
                               cudaStream_t st);
cudaError_t launch_routing_health(const int32_t *counts, const float *P, double *out, int T, int k, int E,
                                  cudaStream_t st);

// ---- backward pass (bwd_sm100.cu, bwd_aux.cu)
// One grouped GEMM C = A B^T on the tensor cores, bf16 operands, fp32
// accumulation.  Group g owns rows offsets[g] .. offsets[g+1]: with kgroup = 0
// they are rows of A and of C (K fixed), with kgroup = 1 they are the
// contraction (A and B both indexed by them, M and N fixed, one C per group).
// Operands are K-major (A rows / B rows of K elements) or MN-major (rows of K
// index holding the M / N elements); a 3-D B map is indexed by expert g.
enum { BW_STORE_BF16 = 0, BW_DGRAD2 = 1, BW_STORE_F32 = 2 };
struct BwdGemmParams {
    const int32_t *offsets;      // [G+1]
    int G;
    int kgroup;
    int M, N, K;                 // kgroup: M, N fixed; else N, K fixed
    int b_per_group;             // 1: B is a 3-D map, expert g; 0: a 2-D map
    int k_split;                 // MN-major B, kgroup 0: K rows >= k_split come from tmB2 (row - k_split)
    int mode;
    // BW_STORE_F32 / BW_STORE_BF16: C row r, column c at out[r * ldo + c]
    // (+ g * out_group_stride when kgroup); BW_STORE_BF16 adds bias[g][c]
    void *out;
    int64_t ldo, out_group_stride;
    const float *bias;
    int64_t bias_group_stride;
    // BW_DGRAD2: C = dH (gate applied) of hidden columns; with H (the forward
    // hidden activation) and GU (pre-activations: G at column c, U at F + c,
    // or the GELU input) of the same rows: dGU = (dG | dU) or dA, and
    // part[r][2 nt + half] = sum over the half-tile's columns of H * C
    float *part;
    int part_ld;
    const __nv_bfloat16 *H;
    int64_t ldh;
    const __nv_bfloat16 *GU;
    int64_t ldgu;
    __nv_bfloat16 *dGU;
    int F, act;
    int32_t *status;
    uint64_t timeout_ns;
};
// Rows of a K-major B box: each CTA of a pair loads half of a 256-column tile.
constexpr uint32_t kBwdBoxRowsB = 128;
cudaError_t launch_bwd_gemm(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &B2, bool a_mn, bool b_mn,
                            const BwdGemmParams &p, int num_sms, cudaStream_t st);

struct BwdAuxArgs {
    const int32_t *offsets;      // [E+1] forward dispatch tables
    const int32_t *row_token;
    const float *row_gate;
    const int32_t *row_of;       // [T, k]
    const int32_t *idx;          // [T, k]
    const float *gate;           // [T, k]
    const float *logits;         // [T, E] forward router logits (with the logit offset)
    const int32_t *counts;       // [E]
    const void *dy;              // [T, d] bf16
    const float *b2;             // [E, d] GELU output bias or null
    const float *part;           // [rows, part_ld] partial <H, dH> of the down dgrad
    int part_ld;
    __nv_bfloat16 *dZ;           // [rows, d]
    float *dh;                   // [T, E]
    __nv_bfloat16 *dh_bf16;      // [T, dh_ld]
    int dh_ld;
    const __nv_bfloat16 *dX_rows;  // [rows, d]
    const float *dX_shared;      // [T, d] or null
    const float *dX_router;      // [T, d]
    void *dx;                    // [T, d] bf16
    float alpha;
    int T, d, E, k, score, renorm, num_sms;
};
cudaError_t launch_scale_rows(const BwdAuxArgs &a, int max_rows, cudaStream_t st);
cudaError_t launch_router_bwd(const BwdAuxArgs &a, cudaStream_t st);
cudaError_t launch_dx_combine(const BwdAuxArgs &a, cudaStream_t st);
// out[g][c] = sum over the rows of group g (offsets, or all `rows` when null) of in[r][c]
struct ColSumArgs {
    const void *in;
    int in_f32;
    int64_t ld;
    const int32_t *offsets;
    int G, rows, cols;
    float *out;
};
cudaError_t launch_column_sums(const ColSumArgs &a, cudaStream_t st);
cudaError_t launch_to_bf16(const float *in, __nv_bfloat16 *out, int64_t rows, int cols, int64_t ldo, cudaStream_t st);
// out[c] = sum of in[r][c] over r < rows, in two deterministic passes (part:
// ceil(rows / 256) x cols fp32 scratch)
cudaError_t launch_col_sums_2pass(const float *in, int64_t rows, int cols, int64_t ld, float *part, float *out,
                                  cudaStream_t st);
cudaError_t launch_set_pair(int32_t *p, int32_t a, int32_t b, cudaStream_t st);     // p[0] = a, p[1] = b

// Host-side helpers shared by the entry points (moe_api.cu).
moe_status validate_config(const moe_config *cfg);        // sets the error detail
void set_error_detail(const char *where, const char *what);

}  // namespace moe
