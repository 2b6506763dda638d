/*
 * moe.h - C ABI of libmoe.so: the single-GPU forward pass of a sparsely-gated
 * Mixture-of-Experts layer on NVIDIA B200 (sm_100a).
 *
 * The layer (Shazeer et al., "Outrageously Large Neural Networks: The Sparsely-Gated
 * Mixture-of-Experts Layer", section "Methode"): y = sum_i G(x)_i E_i(x), where the
 * experts E_i are feed-forward sub-networks and G is a sparse gate that is zero for all
 * but k experts, so only k experts run per token.  The forward pass has five steps:
 *
 *   moe_route      router product x.W_g fused with the gate (softmax top-k, or noisy
 *                  top-k) -> chosen experts and their gate values per token
 *   moe_permute    per-expert histogram, scan, capacity truncation and a stable counting
 *                  sort of the token->expert assignments; gathers the kept token rows
 *   moe_expert_ffn per-expert FFN on the kept rows only (grouped GEMM, tensor cores)
 *   moe_combine    gate-weighted sum of each token's expert outputs (un-permute)
 *   moe_expert_ffn_combine  the last two fused, for top-1 routing in bf16
 *   moe_forward    all of the above on one stream
 *
 * Conventions for every call
 *  - All pointers are DEVICE pointers unless stated, owned by the caller, and must
 *    stay valid until the work queued on `stream` has finished.  The library never
 *    allocates, frees or synchronises, except moe_get_error (which synchronises).
 *  - Work is queued asynchronously on `stream` (NULL = the legacy default stream) on
 *    the current CUDA device.  A call returns once its kernels are queued.
 *  - Arguments are validated on the host before any launch; a bad argument returns
 *    MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED and queues nothing.  A failed launch
 *    returns MOE_ERR_CUDA.  Problems only visible on the device (an expert index out of
 *    range, inconsistent offsets, an expired bounded wait) set bits of the device error
 *    word held in the workspace; read and clear them with moe_get_error.
 *  - Layouts are row-major and contiguous.  Weight matrices are stored K-major (one row
 *    per output feature, contiguous along the contraction): the pages write x.W_g with
 *    W_g as [d_model, E]; w_gate here is its transpose [E, d_model].
 *  - Index tensors are int32.  Assignment a = t*k + j is token t's j-th choice.
 *  - x, the weights, x_perm and h are in cfg->dtype; the expert outputs y_perm, gates,
 *    noise, logit_bias, importance and load are always fp32 (the products accumulate in
 *    fp32 and are not rounded to bf16 on the way out); the layer output y is fp32, or
 *    bf16 with cfg->y_bf16 (the fp32 sum of its row rounded once).
 *  - T == 0 is valid: nothing is launched, the per-expert outputs that are given
 *    (counts, offsets, importance, load) are zero-filled on `stream`, and per-token
 *    pointers may be NULL.
 *  - The workspace `ws` is a device buffer of at least moe_workspace_size() bytes (or
 *    moe_forward_workspace_size() for moe_forward), 256-byte aligned, zero-filled once
 *    by the caller before first use (it holds the sticky device error word).  Calls that
 *    share one workspace must be ordered on one stream.
 *
 * Supported shapes: bf16 needs d_model and d_ff multiples of 64 and E <= 256; fp32
 * needs d_model and d_ff multiples of 4; all need 1 <= k <= min(E, 8), d_model % 8 == 0
 * and T*k < 2^31.  Hierarchical gating also needs groups + E <= 256 (bf16) or <= 1024
 * (fp32) and at most 4 kept per level.  Outside these the call returns
 * MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL selects the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size or enum, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but outside the supported shapes/dtypes */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime/driver call or kernel launch failed */
  MOE_ERR_DEVICE = 4        /* moe_get_error found device error bits set */
} moe_status;

/* Bits of the device error word (see moe_get_error). */
enum {
  MOE_DEVERR_EXPERT_INDEX = 1, /* a topk_idx entry outside [0, E): treated as dropped */
  MOE_DEVERR_OFFSETS = 2,      /* offsets not non-decreasing in [0, T*k]: FFN skipped */
  MOE_DEVERR_SLOT = 4,         /* a slot_pos entry outside [-1, T*k), or a perm_src entry
                                  outside [0, T*k) in moe_expert_ffn_combine: treated as
                                  dropped (that row is not written) */
  MOE_DEVERR_TIMEOUT = 8       /* a bounded wait inside a pipelined kernel expired */
};

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Gating rule.
 * MOE_GATE_SOFTMAX_TOPK: scores l = x.W_g (+ logit_bias); the k largest are chosen.
 *   renorm = 1: gates = Softmax(KeepTopK(l, k)) (Shazeer et al., "Noisy Top-K Gating",
 *               without noise); renorm = 0: each chosen expert's gate is its probability
 *               under the softmax over all E experts (the Switch Transformer top-1 rule).
 * MOE_GATE_NOISY_TOPK: H = x.W_g (+ logit_bias) + noise * Softplus(x.W_noise), the k
 *   largest of H are chosen and gates = Softmax(KeepTopK(H, k)) (Shazeer et al.,
 *   "Noisy Top-K Gating"; renorm is ignored).  `noise` holds the StandardNormal() draws.
 * MOE_GATE_HIERARCHICAL: a two-level gate (Shazeer et al., "Schlüsselbegriffe":
 *   hierarchical MoE, a primary gating network routing to secondary MoE groups; "MoE-H"
 *   in the setups table of the "moe paper models" page).  The E experts form
 *   cfg->groups groups of b = E / groups; w_gate holds groups + E rows: the primary
 *   gating rows, then group i's b secondary rows.  The primary gate Softmax(KeepTopK(.,
 *   k_primary)) keeps k_primary groups; each kept group's gate Softmax(KeepTopK(.,
 *   k / k_primary)) keeps k / k_primary of its experts; expert j of group i is expert
 *   i*b + j and its gate is the product of the two levels' gates.  Chosen groups are
 *   listed largest primary score first, each followed by its chosen experts, largest
 *   first.  No noise; renorm and logit_bias are ignored.
 * Ties go to the lowest expert index; chosen experts are listed largest score first. */
typedef enum {
  MOE_GATE_SOFTMAX_TOPK = 0,
  MOE_GATE_NOISY_TOPK = 1,
  MOE_GATE_HIERARCHICAL = 2
} moe_gating;

/* Expert activation: ReLU, or GELU in its erf form 0.5 z (1 + erf(z / sqrt 2)) (not the
 * tanh approximation).  The bf16 tensor-core path evaluates erf by Abramowitz & Stegun
 * formula 7.1.26 (|error| <= 1.5e-7, far below the 16-bit rounding of h that follows);
 * the fp32 path uses CUDA's erff. */
typedef enum { MOE_ACT_RELU = 0, MOE_ACT_GELU = 1 } moe_act;

typedef struct {
  int64_t T;              /* tokens */
  int32_t d_model;        /* model width d */
  int32_t d_ff;           /* expert hidden width f */
  int32_t E;              /* experts */
  int32_t k;              /* experts per token */
  int32_t gating;         /* moe_gating */
  int32_t renorm;         /* see moe_gating */
  float capacity_factor;  /* > 0: capacity C = ceil(cf*T*k/E) per expert; <= 0: none */
  int32_t act;            /* moe_act */
  int32_t dtype;          /* moe_dtype of x, the weights, x_perm and h */
  int32_t hidden_f16;     /* bf16 only, 0 or 1: 1 stores the hidden activations h in fp16
                             (11 significant bits instead of 8) and takes w2 in fp16, since
                             both operands of one tensor-core product share a type; a bf16
                             w2 converts to fp16 exactly wherever |w| >= 2^-17 (see
                             moe_bf16_to_f16).  Needs |h| < 65504. */
  int32_t groups;         /* MOE_GATE_HIERARCHICAL: expert groups (divides E); else ignored */
  int32_t k_primary;      /* MOE_GATE_HIERARCHICAL: groups kept per token (divides k, and
                             k / k_primary <= E / groups); else ignored */
  int32_t y_bf16;         /* bf16 only, 0 or 1: 1 writes the layer output y in bf16, each
                             row's fp32 sum rounded once to nearest even (y_perm stays
                             fp32; the rounding adds up to 2^-9 relative per value, which
                             a max|err|/RMS bar of 2e-2 does not absorb when a few outputs
                             are many times the RMS); 0 writes y in fp32 */
} moe_config;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status s);

/* Capacity C = ceil(cf * T * k / E), computed exactly from the fp32 value of cf
 * (capacity factors as in the setups table of the "moe paper models" page), or -1 when
 * cfg->capacity_factor <= 0 (no limit).  Returns -2 for an invalid cfg. */
int64_t moe_capacity(const moe_config* cfg);

/* Bytes of workspace the step calls (moe_route ... moe_combine) need; 0 for an invalid
 * or unsupported cfg. */
size_t moe_workspace_size(const moe_config* cfg);

/* Bytes of workspace moe_forward needs: the step workspace plus the intermediates
 * (offsets, slot_pos, perm_src, x_perm, h, y_perm) it keeps there. */
size_t moe_forward_workspace_size(const moe_config* cfg);

/* Router product and gate [Shazeer et al., "Noisy Top-K Gating"; Switch Transformer,
 * switch_routing].
 *  x          [T, d_model] dtype
 *  w_gate     [E, d_model] dtype (W_g transposed)
 *  w_noise    [E, d_model] dtype, required for noisy gating, else ignored (may be NULL)
 *  noise      [T, E] fp32 StandardNormal draws, required for noisy gating
 *  logit_bias [E] fp32 added to the clean logits, or NULL
 *  topk_idx   [T, k] int32 out: chosen experts, largest score first
 *  topk_gate  [T, k] fp32 out: their gates
 *  importance [E] fp32 out or NULL: Importance(X) = sum_t G(x_t) ("Load-Balancing-Losses")
 *  load       [E] fp32 out or NULL: Load(X)_i = sum_t P(x_t, i) with
 *             P(x,i) = Phi(((x.W_g)_i - kth_excluding(H,k,i)) / Softplus((x.W_noise)_i));
 *             noisy gating with k < E only
 *  near_tie   [T] uint8 out or NULL: 1 where the k-th and (k+1)-th scores differ by at
 *             most 1e-4 (there two top-k choices are both correct up to rounding)
 * The scores are accumulated in fp32 (bf16 inputs: exact bf16 products, fp32 sums). */
moe_status moe_route(const moe_config* cfg, const void* x, const void* w_gate,
                     const void* w_noise, const float* noise, const float* logit_bias,
                     int32_t* topk_idx, float* topk_gate, float* importance, float* load,
                     uint8_t* near_tie, void* ws, moe_stream_t stream);

/* Capacity truncation and stable permutation by expert [Switch Transformer,
 * switch_routing: dispatch is a gather of each expert's tokens].
 *  topk_idx [T, k] int32 in
 *  x        [T, d_model] dtype in
 *  counts   [E] int32 out: assignments per expert before the capacity drop
 *  offsets  [E+1] int32 out: expert e's kept rows are x_perm[offsets[e] : offsets[e+1]]
 *  perm_src [T*k] int32 out: perm_src[s] = assignment a held by permuted row s
 *           (entries at s >= offsets[E] are left untouched)
 *  slot_pos [T*k] int32 out: permuted row of assignment a, or -1 if dropped
 *  x_perm   [T*k, d_model] dtype out: x_perm[s] = x[perm_src[s] / k]; or NULL, and then
 *           x may be NULL too: only the index arrays are written and no row is copied
 *           (the expert FFN gathers the rows itself: moe_expert_ffn_gather)
 * Within an expert rows keep ascending a; the first C are kept (C = moe_capacity). */
moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                       int32_t* counts, int32_t* offsets, int32_t* perm_src,
                       int32_t* slot_pos, void* x_perm, void* ws, moe_stream_t stream);

/* Per-expert FFN on the kept rows [Shazeer et al.: experts are feed-forward networks;
 * computation is skipped where G(x)_i = 0]:
 *   h[s] = act(x_perm[s] . W1_e^T),  y_perm[s] = h[s] . W2_e^T  for offsets[e] <= s < offsets[e+1]
 *  x_perm  [T*k, d_model] dtype in (rows >= offsets[E] are never read into outputs)
 *  offsets [E+1] int32 in (as written by moe_permute; any non-decreasing values in
 *          [0, T*k] are accepted)
 *  w1      [E, d_ff, d_model] dtype,  w2 [E, d_model, d_ff] dtype
 *  h       [T*k, d_ff] out (hidden activations; rows < offsets[E] written): dtype, or
 *          fp16 when cfg->hidden_f16
 *  y_perm  [T*k, d_model] fp32 out (rows < offsets[E] written)
 * w2 is fp16 when cfg->hidden_f16, else dtype.  bf16: tcgen05 tensor cores with fp32
 * accumulation; h is rounded once to its storage type.  fp32: FP32 FMA throughout. */
moe_status moe_expert_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                          const void* w1, const void* w2, void* h, void* y_perm, void* ws,
                          moe_stream_t stream);

/* The expert FFN over row groups that share weight blocks: group g (0 <= g < groups) is
 * rows [offsets[g], offsets[g+1]) of x_rows and runs expert g mod E of w1/w2 (E =
 * cfg->E weight blocks).  With the rows that R source ranks sent to this rank's E
 * experts laid out source by source, each source's rows by expert (groups = R E), this is
 * the expert computation of an expert-parallel layer [Shazeer et al., "Kombinierte Daten-
 * und Modellparallelität": each device holds some experts and receives, from every
 * device, the tokens routed to them].  Arithmetic as moe_expert_ffn (bf16 only).
 *  x_rows   [rows_cap, d_model] bf16 in;  offsets [groups+1] int32 in, non-decreasing in
 *           [0, rows_cap] (else MOE_DEVERR_OFFSETS and no output)
 *  w1 [E, d_ff, d_model], w2 [E, d_model, d_ff] (fp16 with cfg->hidden_f16)
 *  h        [rows_cap, d_ff] out;  y_rows [rows_cap, d_model] fp32 out (rows below
 *           offsets[groups] written)
 *  ws       at least moe_workspace_size(cfg) bytes (its device error word is used)
 * cfg->T and cfg->k are not used.  groups <= 1024 and rows_cap < 2^31 (else
 * MOE_ERR_UNSUPPORTED); rows_cap == 0 launches nothing. */
moe_status moe_expert_ffn_grouped(const moe_config* cfg, const void* x_rows, int64_t rows_cap,
                                  const int32_t* offsets, int32_t groups, const void* w1,
                                  const void* w2, void* h, void* y_rows, void* ws,
                                  moe_stream_t stream);

/* moe_expert_ffn with the permuted rows gathered from the token rows instead of read
 * from x_perm [Switch Transformer, switch_routing: dispatch is a gather of each expert's
 * tokens]: permuted row s is x[perm_src[s] / k], fetched by the up-projection's tensor
 * memory accelerator (TMA) straight into the tensor cores' operand tiles, so x_perm is
 * never written or read back.  Results are bit-identical to moe_permute (with x_perm)
 * followed by moe_expert_ffn.
 *  x        [T, d_model] dtype in (the token rows)
 *  perm_src [T*k] int32 in, as written by moe_permute (entries s < offsets[E] are read;
 *           a value outside [0, T*k) reads zeros for that row's operand)
 *  offsets, w1, w2, h, y_perm, ws: as moe_expert_ffn. */
moe_status moe_expert_ffn_gather(const moe_config* cfg, const void* x, const int32_t* perm_src,
                                 const int32_t* offsets, const void* w1, const void* w2, void* h,
                                 void* y_perm, void* ws, moe_stream_t stream);

/* Gate-weighted combine [Shazeer et al., "Methode": y = sum_i G(x)_i E_i(x)]:
 *   y[t] = sum_j topk_gate[t, j] * y_perm[slot_pos[t*k + j]]   (dropped slots add 0)
 *  y_perm [T*k, d_model] fp32, slot_pos [T*k] int32, topk_gate [T, k] fp32 in
 *  y      [T, d_model] fp32 out (bf16 with cfg->y_bf16); accumulated in fp32 in the order
 *         j = 0 .. k-1, then stored. */
moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* slot_pos,
                       const float* topk_gate, void* y, void* ws, moe_stream_t stream);

/* moe_expert_ffn followed by moe_combine as one step, in bf16 for k = 1, and for k = 2
 * with an fp32 y [Switch Transformer, switch_routing: with one expert per token the
 * combine is a scaled copy; Shazeer et al., "Methode": y = sum_i G(x)_i E_i(x)]:
 *   y[t] = sum over t's kept assignments a of topk_gate[a] * (act(x[t] . W1_e^T) . W2_e^T)
 *   (y[t] = 0 for a token all of whose assignments were dropped).
 * The down-projection puts each gate-weighted fp32 row straight into y at its token
 * (token = perm_src[s] / k), so y_perm never exists.  k = 1: a store; the rows of dropped
 * tokens are zeroed by the down-projection's epilogue threads before its first tile.
 * k = 2: the up-projection's epilogue threads zero y (a 16 KB chunk per CTA and tile) and
 * the down-projection adds each rounded product into the row in memory; the two adds of a
 * token commute, so y does not depend on their order.  For k = 1 y is bit-equal to
 * moe_expert_ffn + moe_combine on the same inputs; for k = 2 it differs from it by at most
 * the rounding of one product (moe_combine folds the second product into a fused
 * multiply-add).
 *  x_perm, offsets, w1, w2, h as moe_expert_ffn;  perm_src, slot_pos as written by
 *  moe_permute;  topk_gate [T, k] fp32 in;  y [T, d_model] fp32 out, bf16 with
 *  cfg->y_bf16 for k = 1 (every row written).
 * A perm_src entry outside [0, T*k) sets MOE_DEVERR_SLOT (that row is not written).
 * Returns MOE_ERR_UNSUPPORTED unless dtype is bf16 and k == 1, or k == 2 without
 * cfg->y_bf16. */
moe_status moe_expert_ffn_combine(const moe_config* cfg, const void* x_perm,
                                  const int32_t* offsets, const int32_t* perm_src,
                                  const int32_t* slot_pos, const float* topk_gate,
                                  const void* w1, const void* w2, void* h, void* y, void* ws,
                                  moe_stream_t stream);

/* moe_expert_ffn_combine with the permuted rows gathered from the token rows x (as
 * moe_expert_ffn_gather does) instead of read from x_perm; the same k and dtype rules.
 *  x [T, d_model] bf16 in; the other arguments as moe_expert_ffn_combine.  y is
 *  bit-identical to moe_expert_ffn_combine's on x_perm. */
moe_status moe_expert_ffn_combine_gather(const moe_config* cfg, const void* x,
                                         const int32_t* offsets, const int32_t* perm_src,
                                         const int32_t* slot_pos, const float* topk_gate,
                                         const void* w1, const void* w2, void* h, void* y,
                                         void* ws, moe_stream_t stream);

/* The whole layer forward on one stream: moe_route, moe_permute, moe_expert_ffn,
 * moe_combine (moe_expert_ffn_combine in place of the last two when k = 1 and dtype is
 * bf16; for k = 2 its fused form is not faster, so the two steps run).  Inputs as in the step calls; y [T, d_model] fp32 (bf16 with cfg->y_bf16) out.  topk_idx,
 * topk_gate (both [T, k]) and counts ([E]) are outputs the caller must provide;
 * importance, load and near_tie may be NULL.  The intermediates live in `ws`
 * (moe_forward_workspace_size bytes). */
moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_gate,
                       const void* w_noise, const float* noise, const float* logit_bias,
                       const void* w1, const void* w2, void* y, int32_t* topk_idx,
                       float* topk_gate, int32_t* counts, float* importance, float* load,
                       uint8_t* near_tie, void* ws, moe_stream_t stream);

/* ---------------------------------------------------------------- training
 * The backward pass of the layer for
 *   L = sum(dy * y) + w_importance * CV(Importance(X))^2 + w_load * CV(Load(X))^2
 * [Shazeer et al., "Load-Balancing-Losses": the auxiliary losses are weights times the
 * squared coefficient of variation of Importance and Load; "Fragen": the top-k choice
 * is taken before the softmax, so the chosen experts' gates keep continuous derivatives
 * and gradients reach the gating network].  Which experts are chosen or dropped passes no
 * gradient; the noise draws are inputs; CV uses the population standard deviation;
 * kth_excluding passes its gradient to the entry of H it picks.  bf16 layers with the
 * softmax or noisy gate only (others return MOE_ERR_UNSUPPORTED).  */

/* Bytes of the forward state moe_forward_train writes and moe_backward reads (the kept
 * rows, permutation, expert pre-activations, hidden activations and expert outputs of
 * one batch, and the router's scores as the gate computed them: clean logits, and for
 * noisy gating Softplus(x.W_noise), the noisy scores and each token's k-th and (k+1)-th
 * of them, so that the backward differentiates exactly the forward's choice); 0 for an
 * unsupported cfg.  The layout is internal to the library. */
size_t moe_train_state_size(const moe_config* cfg);

/* Bytes of workspace moe_backward needs (the step workspace, whose device error word it
 * shares, plus its own intermediates). */
size_t moe_backward_workspace_size(const moe_config* cfg);

/* moe_forward that also keeps what the backward pass needs in `state` (a device buffer of
 * moe_train_state_size bytes, 16-byte aligned).  Same arguments and outputs as
 * moe_forward; y is the same function of the inputs.  Pass importance (and load, for
 * noisy gating) when the backward will weight their losses. */
moe_status moe_forward_train(const moe_config* cfg, const void* x, const void* w_gate,
                             const void* w_noise, const float* noise, const float* logit_bias,
                             const void* w1, const void* w2, void* y, int32_t* topk_idx,
                             float* topk_gate, int32_t* counts, float* importance, float* load,
                             uint8_t* near_tie, void* state, void* ws, moe_stream_t stream);

/* Gradients of L with respect to the layer's inputs and parameters.
 *  x, w_gate, w_noise, noise, logit_bias, w1, w2: the inputs of the forward call
 *  topk_idx, topk_gate, importance, load: its outputs; state: its saved state
 *  dy          [T, d_model] fp32: dL/dy of the layer output
 *  w_importance, w_load: loss weights (0 drops a term; w_load needs noisy gating, k < E)
 *  dx          [T, d_model] fp32 out
 *  dw_gate     [E, d_model] fp32 out; dw_noise [E, d_model] fp32 out (noisy gating)
 *  dlogit_bias [E] fp32 out or NULL
 *  dw1         [E, d_ff, d_model] fp32 out; dw2 [E, d_model, d_ff] fp32 out
 *  dgates      [T, k] fp32 out: dL/d of each chosen gate from the layer output (0 where
 *              the assignment was dropped)
 *  losses      [2] fp32 out or NULL: w_importance CV^2 and w_load CV^2
 *  ws          moe_backward_workspace_size bytes
 * The expert products run on the tensor cores in bf16 with fp32 accumulation (the
 * upstream gradient of each expert row is rounded to bf16, or fp16 with hidden_f16);
 * the router's gradients are fp32, from the scores kept in `state` (the router is not
 * recomputed), with every sum over tokens taken in a fixed order. */
moe_status moe_backward(const moe_config* cfg, const void* x, const void* w_gate,
                        const void* w_noise, const float* noise, const float* logit_bias,
                        const void* w1, const void* w2, const int32_t* topk_idx,
                        const float* topk_gate, const float* importance, const float* load,
                        const void* state, const float* dy, float w_importance, float w_load,
                        float* dx, float* dw_gate, float* dw_noise, float* dlogit_bias, float* dw1,
                        float* dw2, float* dgates, float* losses, void* ws, moe_stream_t stream);

/* Synchronises `stream`, then reads the device error word in `ws` into *device_error
 * (may be NULL) and clears it.  Returns MOE_OK if no bit was set, MOE_ERR_DEVICE if
 * some were, MOE_ERR_CUDA if the synchronisation or copy failed. */
moe_status moe_get_error(void* ws, moe_stream_t stream, int32_t* device_error);

/* Re-encodes n bf16 values as fp16 (round to nearest even), e.g. w2 for
 * cfg->hidden_f16.  fp16's 11 significant bits hold every bf16 value of magnitude in
 * [2^-17, 65504] exactly; smaller magnitudes round to fp16's subnormal grid (absolute
 * error <= 2^-25) and larger ones to +-inf.
 *  src        [n] bf16 device in;  dst [n] fp16 device out (may not alias src)
 *  n_inexact  device int32 or NULL: incremented by the number of values not converted
 *             exactly
 * Weight preparation, run once before the forward passes that use it. */
moe_status moe_bf16_to_f16(const void* src, void* dst, int64_t n, int32_t* n_inexact,
                           moe_stream_t stream);

/* moe_permute for callers that cannot allocate device memory.  It takes no workspace:
 * its scratch (a 256-byte counter block, then one int32 per 256-assignment chunk and
 * expert) is a fixed array of MOE_NOALLOC_SCRATCH_BYTES inside libmoe's own device
 * memory, which every GPU that loads the library holds until the process exits.  The
 * pages have no counterpart; this is plumbing for hosts that own all device memory or
 * forbid allocation where they call us: plugins running inside another runtime's memory
 * arena, code on a latency path where cudaMalloc's implicit synchronisation and possible
 * failure are not acceptable, and callbacks in which CUDA allocation calls are not
 * allowed.
 *  Arguments, outputs and results are those of moe_permute, bit for bit.
 *  Sizes: 256 + ceil(T*k / 256) * E * 4 must not exceed MOE_NOALLOC_SCRATCH_BYTES (for
 *  E = 128 that is T*k up to 524,032); larger problems return MOE_ERR_UNSUPPORTED and
 *  queue nothing.
 *  Set-up: the first call in a CUDA context (in practice, the first call on a device, made
 *  with that device current) looks up the array's device address there
 *  (cudaGetSymbolAddress) and caches it under the context's unique id, so a context that
 *  replaces an earlier one (after cudaDeviceReset) gets a fresh lookup; make that first
 *  call before any stream capture.
 *  Sharing: every call uses the same array, which keeps the previous call's contents;
 *  each call clears the counter that must start at zero (cudaMemsetAsync on `stream`) and
 *  rewrites everything else it reads.  Calls whose work overlaps on the GPU (other
 *  streams, other host threads) race on the array and must be serialised by the caller.
 *  Errors: there is no device error word: an out-of-range expert index is treated as
 *  dropped without a report.  Never calls cudaMalloc, cudaFree or any allocating
 *  routine. */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 20)
moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx, const void* x,
                               int32_t* counts, int32_t* offsets, int32_t* perm_src,
                               int32_t* slot_pos, void* x_perm, moe_stream_t stream);

/* Diagnostic: runs the permutation's grid barrier on two blocks with a target that no
 * block ever reaches, so every block's bounded wait expires: after about one second
 * each block sets MOE_DEVERR_TIMEOUT in the workspace's error word and returns, and the
 * last block out resets the barrier counters, as a permutation that lost a block
 * would.  A test reads the error word (moe_get_error) and then runs a normal call on
 * the same workspace.  ws: a workspace as for the step calls (at least 16 bytes).  No
 * counterpart on the pages. */
moe_status moe_wait_timeout_check(void* ws, moe_stream_t stream);

/* Diagnostic: evaluates, for n fp32 inputs x, the erf approximation the GELU epilogue of
 * the tensor-core FFN uses (Abramowitz & Stegun formula 7.1.26, |error| <= 1.5e-7; with its fast fp32 evaluation
 * within 1e-6 of erff) into
 * fast[] and CUDA's erff into ref[], so a test can bound their difference.  No
 * counterpart on the pages (they do not fix the GELU form).  All pointers device. */
moe_status moe_erf_check(const float* x, float* fast, float* ref, int64_t n,
                         moe_stream_t stream);

/* Self-check of the GELU epilogue of the up-projection: writes the epilogue's paired
 * evaluation of GELU(z) = z Phi(z) (erf by Abramowitz & Stegun 7.1.26 on f32x2 pairs
 * (z[2i], z[2i+1]); an odd last value is paired with itself) into fast[] and
 * 0.5 z (1 + erff(z / sqrt 2)) into ref[], so a test can bound their difference.  All
 * pointers device, n >= 0 values; MOE_ERR_INVALID_ARG for n < 0 or a null pointer
 * with n > 0. */
moe_status moe_gelu_check(const float* z, float* fast, float* ref, int64_t n,
                          moe_stream_t stream);

/* Number of kernels the most recent successful call on this host thread queued. */
int32_t moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
