/*
 * cce.h — C ABI of the flash-CCE ORPO language-model head for NVIDIA B200
 * (sm_100a).
 *
 * The head takes final hidden states H[M,D], a frozen output projection
 * W[V,D] and per-row labels y[M].  It computes per-row logp and lse without
 * ever storing the [M,V] logits, the ORPO loss, its cotangent dL/dlogp, and
 * dL/dH.  The operations are those of the mlx-bun design pages:
 *
 *   "Training — design (ORPO, flash-CCE head, prefix sharing, segmented
 *    backward)", mlx-bun 1.0.0: §1 "The objective", §5.1 "The head: from
 *    token-chunking to the flash-CCE kernel", §5.6 "Quantized base";
 *   "ORPO training — design", mlx-bun 0.0.6: "Memory & speed optimization",
 *    ranked lever 1 and its "Implementation spec — fused linear-CE log-prob
 *    head" (forward online softmax, backward recompute from the saved lse);
 *   "flash-CCE host-buffer pin leak — post-mortem", mlx-bun 0.0.6 (why no host
 *    pointer outlives a call).
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - Pointers are DEVICE pointers on the current CUDA device unless a comment
 *   says "host".  Host structs (cce_head, cce_layout) are read during the call
 *   only; their fields go to the kernels by value.  The library keeps no
 *   pointer after a call returns.
 * - Ownership: the caller allocates and frees everything, the workspace
 *   included.  The library never calls cudaMalloc or cudaFree.
 * - Asynchrony: every call enqueues work on `stream` and returns; outputs are
 *   valid once the stream reaches them.  Nothing synchronises except
 *   cce_device_status().
 * - Errors: argument problems are detected before anything is enqueued and
 *   returned synchronously (CCE_ERR_INVALID_ARGUMENT, CCE_ERR_UNSUPPORTED,
 *   CCE_ERR_WORKSPACE_TOO_SMALL).  A failed launch returns CCE_ERR_CUDA.
 *   Problems only the device can see (a label >= V, an empty response
 *   segment, a mean log-prob outside the domain of log1mexp, a bounded wait
 *   that ran out) set a bit in the status word at the start of the workspace;
 *   the kernels then finish without trapping, and cce_device_status() reports
 *   and clears the bits.  No C++ exception crosses this interface.
 * - Labels: y < 0 marks an ignored row (logp = 0, no loss term, dH row
 *   exactly 0; lse is still computed).  y >= V is an error.
 * - Tensor-core path requirements: D % 64 == 0; 16-byte aligned pointers.
 * - Size limits: M <= 2^30, V <= 2^30, D <= 2^16, and the kernels' tile count
 *   ceil(M/128) * max(ceil(V/256), 32*ceil(D/256)) below 2^31; larger
 *   problems return CCE_ERR_UNSUPPORTED (split them by rows).
 */
#ifndef CCE_H_
#define CCE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* cce_stream_t;

typedef enum {
  CCE_OK = 0,
  CCE_ERR_INVALID_ARGUMENT = 1,
  CCE_ERR_UNSUPPORTED = 2,
  CCE_ERR_CUDA = 3,
  CCE_ERR_WORKSPACE_TOO_SMALL = 4,
  CCE_ERR_LABEL_OUT_OF_RANGE = 5,  /* device: some y >= V                    */
  CCE_ERR_DEVICE_TIMEOUT = 6,      /* device: a bounded wait ran out          */
  CCE_ERR_EMPTY_SEGMENT = 7,       /* device: no labelled chosen/rejected row */
  CCE_ERR_DOMAIN = 8,              /* device: mean logp >= 0 (log1mexp)       */
  CCE_ERR_FP16_RANGE = 9           /* device: a 4/8-bit head's fp16 path met a
                                      hidden value |h| > 65504, or a scale or
                                      bias outside the fp16 normal range        */
} cce_status;

typedef enum { CCE_F32 = 0, CCE_BF16 = 1 } cce_dtype;

typedef enum {
  CCE_W_DENSE = 0,         /* w: [V, D] row-major, dtype f32 or bf16          */
  CCE_W_AFFINE_Q4_G64 = 1, /* w: uint32 [V, D/8]; element 8k+j of a row is bits
                              4j..4j+3 of word k (low nibble first);
                              scales, biases: bf16 [V, D/64]; the weight is
                              q*scale + bias (Training design §5.6).          */
  CCE_W_AFFINE_Q8_G64 = 2  /* w: uint32 [V, D/4]; element 4k+j of a row is byte
                              j of word k (low byte first); scales, biases as
                              for the 4-bit head.  Quantised heads compute in
                              fp16: H is converted once, and each weight is
                              dequantised by this library's kernels (inside
                              the GEMM, or into a staged fp16 chunk of the
                              workspace; see cce_set_quant_staging) and
                              rounded once to fp16.  fp16 holds these values
                              exactly only for |h| <= 65504 and scales and
                              biases that are 0 or of magnitude in
                              [2^-14, 65504]; anything else completes but sets
                              CCE_ERR_FP16_RANGE in the status word.  The
                              coefficient tile G'' is fp16 on this path and is
                              stored times 2^14 (|G''| <= 1), so softmax
                              probabilities down to about 4e-12 stay normal
                              or representable (a flat softmax over 128k
                              entries is 5e-6); the dH step divides it out in
                              fp32.                                           */
} cce_wformat;

/* The frozen head (host struct; device pointers inside). */
typedef struct {
  cce_wformat format;
  cce_dtype dtype;       /* dense: dtype of w; 4/8-bit: CCE_BF16 (scales) */
  int64_t V, D;
  const void* w;
  const void* scales;    /* 4/8-bit heads only, else NULL (2-byte aligned) */
  const void* biases;    /* 4/8-bit heads only, else NULL (2-byte aligned) */
  float softcap;         /* > 0: logits are softcap * tanh(h.W_v / softcap)
                            (Gemma-style final-logit capping; the backward
                            applies 1 - tanh^2); 0 = none */
} cce_head;

/* Disjoint head-row ranges [begin, end) of one ORPO pair (host struct).
 * prompt rows feed the NLL term in "full" scope; chosen rows give the
 * length-normalised mean lw, rejected rows lr (Training design §1). */
typedef struct {
  int64_t prompt_begin, prompt_end;
  int64_t chosen_begin, chosen_end;
  int64_t rejected_begin, rejected_end;
} cce_layout;

/* NLL scope of the ORPO objective (Training design §1, `sft_scope`). */
enum { CCE_SCOPE_FULL = 0, CCE_SCOPE_RESPONSE = 1 };

/* Width of one vocab block of the per-block statistics (and of one vocab
 * tile of the kernels). */
#define CCE_VOCAB_BLOCK 256

/* Number of vocab blocks: ceil(V / CCE_VOCAB_BLOCK). */
int64_t cce_blockmax_cols(int64_t V);

/* Bytes of workspace that cce_forward and cce_backward_dh need for this
 * problem with the default backward chunk.  A larger workspace lets the
 * backward use wider vocab chunks (fewer passes); a smaller one (down to
 * cce_workspace_min_bytes: one 256-column chunk, no K split of the dH GEMM)
 * narrower ones and fewer K splits.  Returns 0 for invalid input. */
size_t cce_workspace_bytes(int64_t M, cce_dtype h_dtype, const cce_head* W);
size_t cce_workspace_min_bytes(int64_t M, cce_dtype h_dtype, const cce_head* W);

/*
 * Forward of the head (Training design §5.1; ORPO design 0.0.6, fused-head
 * spec "Forward (online-softmax over vocab tiles)"):
 *   lse[m]  = logsumexp_v (H[m] . W[v])
 *   logp[m] = H[m] . W[y_m] - lse[m]      (0 when y_m < 0)
 * H: [M, D] row-major, f32 or bf16.  labels: int32 [M].
 * logp, lse: fp32 [M] outputs.
 * tgt_logit: optional fp32 [M] output of H[m] . W[y_m] (untouched when y < 0).
 * blockmax: optional fp32 [cce_blockmax_cols(V), M] output, block-major:
 *   blockmax[b*M + m] = max over v in block b of H[m] . W[v]; the backward's
 *   block skip reads it.
 * ws: workspace of ws_bytes (see cce_workspace_bytes); its first 256 bytes
 *   hold the device status word and must be zeroed once before first use.
 */
cce_status cce_forward(const void* H, cce_dtype h_dtype, int64_t M,
                       const cce_head* W, const int32_t* labels, float* logp,
                       float* lse, float* tgt_logit, float* blockmax, void* ws,
                       size_t ws_bytes, cce_stream_t stream);

/*
 * ORPO loss from per-row log-probs (Training design §1, orpoLossFromLogps):
 *   lw, lr, pm = means of logp over the labelled chosen, rejected, prompt rows
 *   NLL  = -(sum_prompt + sum_chosen)/(n_prompt + n_chosen)   (full scope;
 *          equal to combineFullNll) or -lw (response scope)
 *   z    = (lw - lr) - (log1mexp(lw) - log1mexp(lr))
 *   L_OR = -log sigmoid(z);  L = NLL + lambda * L_OR
 * out8 (device, fp64 [8]): L, NLL, L_OR, lw, lr, pm, z, sigmoid(z).
 * Only the first 256 bytes of ws are used (status word).
 */
cce_status orpo_loss_from_logps(const float* logp, const int32_t* labels,
                                int64_t M, const cce_layout* layout,
                                double lambda, int sft_scope, double* out8,
                                void* ws, size_t ws_bytes,
                                cce_stream_t stream);

/*
 * Cotangent of the ORPO loss with respect to logp (the "1/(1-P)"-scaled OR
 * gradient plus the NLL term; ORPO design 0.0.6, regularization notes):
 *   chosen:   lambda (sigmoid(z) - 1) / (1 - e^lw) / n_chosen + s_C
 *   rejected: -lambda (sigmoid(z) - 1) / (1 - e^lr) / n_rejected
 *   prompt:   s_P;   ignored rows and rows outside the layout: 0
 * with s_C = s_P = -1/(n_prompt + n_chosen) (full) or s_C = -1/n_chosen,
 * s_P = 0 (response).  coeff: fp32 [M] output.
 */
cce_status orpo_grad_coeffs(const float* logp, const int32_t* labels,
                            int64_t M, const cce_layout* layout, double lambda,
                            int sft_scope, float* coeff, void* ws,
                            size_t ws_bytes, cce_stream_t stream);

/*
 * One pair split by rows over several processes (one per GPU).  The
 * objective (Training design §1) reads the rows only through three segment
 * means, i.e. through the sums and counts of logp over the labelled prompt,
 * chosen and rejected rows, so the shards need one exchange of six numbers
 * between the forward and the backward.  No counterpart on the pages.
 *
 * orpo_partial_sums: sums6 (device fp64 [6], 8-byte aligned) = (sum of logp
 *   over the labelled prompt, chosen, rejected rows of this shard; the three
 *   counts), for an all-reduce (sum) across the shards.
 * orpo_from_sums: from the all-reduced sums6, the loss out8 (as in
 *   orpo_loss_from_logps; nullable) and dL/dlogp coeff for this shard's rows
 *   (nullable, not both null).  Identical across shards for out8.
 * layout: this shard's rows in its own row numbering; a shard may hold no
 *   chosen or rejected row (an empty pair-wide segment sets
 *   CCE_ERR_EMPTY_SEGMENT in the status word, as the unsharded call).
 * Otherwise as orpo_loss_from_logps / orpo_grad_coeffs.
 */
cce_status orpo_partial_sums(const float* logp, const int32_t* labels, int64_t M,
                             const cce_layout* layout, double* sums6, void* ws,
                             size_t ws_bytes, cce_stream_t stream);
cce_status orpo_from_sums(const double* sums6, const int32_t* labels, int64_t M,
                          const cce_layout* layout, double lambda, int sft_scope,
                          double* out8, float* coeff, void* ws, size_t ws_bytes,
                          cce_stream_t stream);

/*
 * Objective siblings on the same log-prob engine (Training design §8.3
 * "Objective variants"; the UltraFeedback research notes §6.1-6.3):
 *   CCE_OBJ_ORPO        the ORPO loss above (lambda, sft_scope; beta, gamma
 *                       unused)
 *   CCE_OBJ_SIMPO       L = -log sigmoid(beta (lw - lr) - gamma), no NLL term
 *   CCE_OBJ_ORPO_MARGIN L = NLL + lambda * [-log sigmoid(beta (lw - lr) - gamma)]
 *                       (ORPO's NLL anchor with SimPO's target margin)
 * For the SimPO kinds out8 holds L, NLL, the SimPO term, lw, lr, pm,
 * u = beta (lw - lr) - gamma, sigmoid(u); the cotangent follows by the chain
 * rule (d/du softplus(-u) = sigmoid(u) - 1).  Host struct, read during the
 * call.  lambda >= 0, beta >= 0, gamma finite.
 */
typedef enum { CCE_OBJ_ORPO = 0, CCE_OBJ_SIMPO = 1, CCE_OBJ_ORPO_MARGIN = 2 } cce_objective_kind;
typedef struct {
  cce_objective_kind kind;
  double lambda, beta, gamma;
  int sft_scope;
} cce_objective;

cce_status pref_loss_from_logps(const float* logp, const int32_t* labels,
                                int64_t M, const cce_layout* layout,
                                const cce_objective* obj, double* out8,
                                void* ws, size_t ws_bytes,
                                cce_stream_t stream);
cce_status pref_grad_coeffs(const float* logp, const int32_t* labels,
                            int64_t M, const cce_layout* layout,
                            const cce_objective* obj, float* coeff, void* ws,
                            size_t ws_bytes, cce_stream_t stream);

/*
 * Backward of the head (ORPO design 0.0.6, fused-head spec "Backward
 * (recompute vocab tiles from the saved LSE)"; Training design §5.1):
 *   dH[m] = coeff[m] * sum_v (onehot(y_m)_v - p_mv) W[v],
 *   p_mv  = exp(H[m].W[v] - lse[m]) recomputed tile by tile.
 * coeff: fp32 [M], the cotangent dL/dlogp (e.g. from orpo_grad_coeffs).
 * lse: fp32 [M] from cce_forward on the same H and W.
 * filter_eps > 0 drops p_mv < filter_eps on non-target columns (the coeff
 *   filter, Training design §5.1); 0 disables it.
 * blockmax: optional; when given (with filter_eps > 0) a 128-row x 256-vocab
 *   tile is skipped when every row's block probability exp(blockmax - lse) is
 *   below filter_eps and no label of a row with coeff != 0 falls in the
 *   block, which is exact relative to the filter.
 * dH: fp32 [M, D] output, overwritten.
 * skip_stats: optional device uint64 [2] incremented by (skipped tiles,
 *   total tiles).
 * ws: as for cce_forward.  A dense bf16 head runs the fused backward: one
 *   persistent kernel recomputes every vocab tile, forms the coefficient
 *   tile from the TMEM accumulator and contracts it with W into a dH
 *   accumulator held in TMEM for a whole sweep of the vocabulary; the
 *   coefficient tiles pass between the CTAs sharing a row tile through a
 *   small ring of tiles in ws (two rounds per group, tens of MB, L2-
 *   resident), never as a whole.  ws then holds the block-skip plan, the
 *   ring and its flags, and O(M*D) partial dH buffers when row tiles are
 *   shared between groups (cce_workspace_bytes sizes it).  Other heads (fp32,
 *   4/8-bit, or a workspace too small for the fused layout) run two GEMMs per
 *   vocab chunk, G'' of one chunk living in ws (chunks as wide as ws allows,
 *   see cce_query_plan).  Deterministic in both forms.
 */
cce_status cce_backward_dh(const void* H, cce_dtype h_dtype, int64_t M,
                           const cce_head* W, const int32_t* labels,
                           const float* lse, const float* coeff,
                           float filter_eps, const float* blockmax, float* dH,
                           unsigned long long* skip_stats, void* ws,
                           size_t ws_bytes, cce_stream_t stream);

/*
 * Prefix-shared ORPO pair (Training design §5.4, "Shared prompt-prefix
 * forward"): one forward over [prompt(P); chosen(Rc); rejected(Rr)] gives
 * H_cat [P+Rc+Rr, D], and the head gathers chosen[k] <- H_cat[P-1+k],
 * rejected[0] <- H_cat[P-1], rejected[k>=1] <- H_cat[P+Rc+k-1]; prompt row m
 * (the position predicting prompt token m) <- H_cat[m-1], and the unlabelled
 * head row 0 <- H_cat[0].
 * cce_prefix_gather writes those head rows, in the layout [prompt | chosen |
 * rejected] used by every other call, into H_head [P+Rc+Rr, D] (dtype f32 or
 * bf16, row bytes a multiple of 16).
 * cce_prefix_scatter is its adjoint for the backward: dH_cat [P+Rc+Rr, D]
 * fp32 (overwritten) = the sum of dH_head rows that read each row, so row
 * P-1 receives the gradients of the first chosen and the first rejected
 * token (the two branches' cotangents meet in the shared prefix).
 * Deterministic, bandwidth-bound; P, Rc, Rr >= 1.
 */
cce_status cce_prefix_gather(const void* H_cat, cce_dtype dtype, int64_t P,
                             int64_t Rc, int64_t Rr, int64_t D, void* H_head,
                             cce_stream_t stream);
cce_status cce_prefix_scatter(const float* dH_head, int64_t P, int64_t Rc,
                              int64_t Rr, int64_t D, float* dH_cat,
                              cce_stream_t stream);

/*
 * Backward of a trainable head: cce_backward_dh plus the weight gradient
 *   dW[v] = sum_m coeff[m] (onehot(y_m)_v - p_mv) H[m]   (times 1 - tanh^2
 *   under a softcap, with the same coefficient filter),
 * for when the head stops being frozen (ORPO design 0.0.6, fused-head spec:
 * the head's explicit VJP inputs and the "dC"/head-LoRA follow-on).  It reuses
 * each vocab chunk of the backward: dW[chunk] = -(G''^T . (coeff * H)), a
 * tensor-core GEMM over the rows.  dW: fp32 [V, D] output, overwritten.
 * Dense heads only (quantised heads return CCE_ERR_UNSUPPORTED).  Other
 * arguments as for cce_backward_dh.
 */
cce_status cce_backward_dh_dw(const void* H, cce_dtype h_dtype, int64_t M,
                              const cce_head* W, const int32_t* labels,
                              const float* lse, const float* coeff,
                              float filter_eps, const float* blockmax,
                              float* dH, float* dW,
                              unsigned long long* skip_stats, void* ws,
                              size_t ws_bytes, cce_stream_t stream);

/* Synchronises `stream`, reads and clears the status word in ws, and
 * returns the first error it holds (CCE_OK when none). */
cce_status cce_device_status(void* ws, cce_stream_t stream);

/* Human-readable name of a status. */
const char* cce_status_string(cce_status s);

/* Upper bound, in nanoseconds, of every bounded wait inside the kernels
 * (default 2e9).  0 restores the default.  Process-wide; meant for tests of
 * the timeout path. */
void cce_set_wait_limit_ns(uint64_t ns);

/* Dense heads run the tensor-core GEMMs on CTA pairs (clusters of two
 * CTAs on one TPC, tcgen05 cta_group::2, 256x256 tiles) by default; 0 selects
 * single-CTA 128x256 tiles.  Both give the same results to rounding.
 * Process-wide; a workspace sized under one setting fits the other. */
void cce_set_cta_pairs(int on);

/* How the GEMMs read a 4- or 8-bit head (the dequantisation step of the
 * quantised-head design, Training design, MLX affine quantisation):
 *   0  choose (default): staged when M spans at least 3 row tiles of 128 in
 *      the forward, 2 in the backward, and the workspace holds chunks of at
 *      least 8,192 head rows; else in-kernel;
 *   1  in-kernel: extra warps of the GEMM kernels dequantise each B tile into
 *      shared memory (reads 4.25 or 8.25 bits per weight; the small-M choice);
 *   2  staged: each vocabulary chunk is first dequantised once into an fp16
 *      [chunk, D] buffer in the workspace, then the dense fp16 GEMMs (CTA
 *      pairs) run on it, so the dequantisation is not repeated per row tile.
 * Both produce the same fp16 weights (w = q*scale + bias rounded once), so
 * results agree to accumulation order.  Process-wide.  Any other value is
 * taken as 0.  A workspace of cce_workspace_bytes() under 0 fits every mode
 * (staged falls back to in-kernel when the chunk would be too narrow). */
void cce_set_quant_staging(int mode);

/* Backward of dense bf16 heads:
 *   0  choose (default): the grouped fused kernel from M = 1024 rows when ws
 *      holds its layout (where it measured at least as fast); else two GEMMs
 *      per vocab chunk;
 *   1  the grouped fused kernel at any M (CCE_ERR_WORKSPACE_TOO_SMALL when ws
 *      cannot hold its layout);
 *   2  two GEMMs per vocab chunk;
 *   3  the sliced kernel (M <= 64, D <= 2048; CCE_ERR_UNSUPPORTED outside
 *      that, CCE_ERR_WORKSPACE_TOO_SMALL when ws cannot hold its layout):
 *      clusters of up to 8 CTAs, each owning 256 columns of D, sum their
 *      partial logits through distributed shared memory, so W is read from
 *      HBM once (at D = 2048, V = 262,144 and M <= 64 it measured 0.51 ms
 *      against 0.344 ms for the two GEMMs, so 0 does not choose it).
 * cce_workspace_bytes sizes ws for the form the current setting takes.  All
 * forms give the same results to accumulation order (the sliced kernel sums
 * the logits of its D slices in fp32 in a fixed order).  Process-wide; any
 * other value is taken as 0.  No counterpart on the pages: it selects
 * between schedules of the same backward. */
void cce_set_backward_mode(int mode);

/* Which kernel the forward of a 4-bit or 8-bit head runs (dense heads and
 * staged 4/8-bit heads are not affected):
 *   0  choose: up to 240 head rows, with D a multiple of 512 and 16-byte
 *      aligned scale and bias arrays, a transposed small-M kernel (the
 *      logits as S^T = W_t H^T, the dequantised head tile written into
 *      tensor memory as the MMA's A operand, H the shared-memory B operand
 *      of N = M rounded up to 16, one CTA per SM over blocks of 256 vocab
 *      rows): up to 128 rows both 128-row halves of a block share each K
 *      step, from 129 rows they run one after the other; otherwise the
 *      tiled GEMM with in-kernel dequantisation;
 *   1  the tiled GEMM with in-kernel dequantisation at every M;
 *   2  the second transposed form for 1 to 256 rows (from 241 rows it
 *      measured no faster than the tiled GEMM, whose 256-row tile costs the
 *      same from 129 rows on).
 * Both forms compute the same logits (the same fp16 weights and products,
 * fp32 accumulation), so the results agree to accumulation order: the
 * online softmax of the flash-CCE forward (ORPO design 0.0.6, fused-head
 * implementation spec, "Forward") reduced over the vocabulary in another
 * order.  Process-wide; any other value is taken as 0.  No counterpart on
 * the pages: it selects between schedules of the same forward. */
void cce_set_forward_mode(int mode);

/* The execution plan cce_forward and cce_backward_dh would take for this
 * problem and workspace size under the current settings (host-only: no
 * launch, no device memory; with no device visible the SM count is taken as
 * 148).  No counterpart on the pages: it exposes how the workspace size
 * shapes the chunking, for sizing workspaces and for tests.
 *   fwd_ok / bwd_ok   1 when the workspace is large enough for the call;
 *   fwd_chunk         vocab rows per forward launch (the padded vocabulary
 *                     when the forward runs as one launch);
 *   bwd_chunk         vocab rows per backward G'' chunk;
 *   bwd_ksplit        K splits of the dH GEMM (fp32 partial buffers);
 *   *_staged          1 when a 4/8-bit head runs as staged fp16 chunks;
 *   *_cta_pairs       1 when the GEMMs are planned on CTA pairs (used if the
 *                     device can co-schedule them);
 *   bwd_fused         1 when the backward runs the fused kernel (bwd_chunk
 *                     is then 0);
 *   bwd_fused_groups  groups of CTAs (pairs) that each sweep a row tile;
 *   bwd_fused_members CTAs (pairs) per group, one per 256 columns of dH;
 *   bwd_fused_buffers dH buffers (1 + partial buffers in ws);
 *   bwd_sliced        1 when the backward runs the sliced kernel (bwd_chunk
 *                     and bwd_fused are then 0);
 *   bwd_sliced_clusters  clusters it launches (each sweeps every
 *                     bwd_sliced_clusters-th vocab tile of 128 rows);
 *   bwd_sliced_ctas   CTAs per cluster, one per 256 columns of D;
 *   fwd_q_small_m     the transposed small-M forward a 4/8-bit head runs
 *                     (cce_set_forward_mode): 1 at most 128 head rows, 2
 *                     129 to 240 (1 to 256 in mode 2); 0 the tiled GEMM.
 * Returns CCE_ERR_INVALID_ARGUMENT / UNSUPPORTED as the calls would. */
typedef struct {
  int fwd_ok, bwd_ok;
  int64_t fwd_chunk, bwd_chunk;
  int bwd_ksplit;
  int fwd_staged, bwd_staged;
  int fwd_cta_pairs, bwd_cta_pairs;
  int bwd_fused, bwd_fused_groups, bwd_fused_members, bwd_fused_buffers;
  int bwd_sliced, bwd_sliced_clusters, bwd_sliced_ctas;
  int fwd_q_small_m;
} cce_plan;
cce_status cce_query_plan(int64_t M, cce_dtype h_dtype, const cce_head* W, size_t ws_bytes,
                          cce_plan* out);

/* The work schedule of the fused backward for this problem under the current
 * settings (host-only: no launch, no device memory).  A unit is one round of
 * a group's sweep: a row tile (256 rows on CTA pairs, 128 on single CTAs)
 * against C = ceil(D/256) vocab tiles.  For every unit, group by group and
 * in the order each group runs them, six int32 go to out[6n .. 6n+5]: group,
 * row tile, round, first unit of a segment (a run of units on one row tile),
 * last unit of a segment, and the dH buffer the segment writes (0 = dH,
 * b >= 1 = partial buffer b-1, summed into dH in buffer order).  Writes at
 * most `cap` units (out may be NULL) and returns the total number of units,
 * or -1 when the fused backward does not take the problem.  No counterpart
 * on the pages; it exposes the partition for tests. */
int64_t cce_query_fused_schedule(int64_t M, cce_dtype h_dtype, const cce_head* W,
                                 int32_t* out, int64_t cap);

/* Self-test of the timeout path: launches one CTA that waits, with the
 * current wait limit, on an mbarrier nothing arrives on.  The wait runs out,
 * the kernel sets CCE_ERR_DEVICE_TIMEOUT in the status word and returns;
 * the caller reads it with cce_device_status(). */
cce_status cce_selftest_wait_timeout(void* ws, size_t ws_bytes,
                                     cce_stream_t stream);


/* Optional per-kernel timing for benchmarks.  While enabled, every kernel the
 * library launches is bracketed by a pair of CUDA events recorded on its own
 * launch stream.  cce_profile_enable(1) starts (and clears) a recording,
 * cce_profile_enable(0) stops it.  cce_profile_read() waits for the recorded
 * events, writes per kernel kind the summed milliseconds and the number of
 * launches into ms[0..n) and launches[0..n) (host arrays, either may be
 * NULL), clears the records and returns the number of kinds.
 * cce_profile_kind_name() names a kind.  Process-wide; not for concurrent
 * use from several host threads. */
void cce_profile_enable(int on);
int cce_profile_read(double* ms, long long* launches, int n);
const char* cce_profile_kind_name(int kind);

/*
 * Forward without a caller workspace (no counterpart on the pages; it is a
 * convenience of this library).
 *
 * For callers that cannot allocate device memory: plugins and plain-C hosts
 * that receive only input and output pointers from a framework owning every
 * device allocation, and runtimes whose device-memory budget is fixed at
 * start-up.  Computes exactly what cce_forward computes, for bf16 H and a
 * dense bf16 head, with the forward's scratch (per-block partials, gathered
 * target logits, status word) in a fixed device array of
 * CCE_NOALLOC_SCRATCH_BYTES inside the library.  Every GPU that loads the
 * library holds that array until the process exits.
 *
 * - Needs 256 + 8*ceil(V/256)*M + 4*M bytes of scratch (each term rounded up
 *   to 256) when tgt_logit and blockmax are NULL; a non-NULL blockmax or
 *   tgt_logit is written directly and its share is unused.  Larger problems
 *   return CCE_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - All calls share the one array and it keeps the last call's contents.
 *   Calls whose work overlaps on the GPU (several streams, several host
 *   threads) race on it; serialise them.
 * - status: optional device uint32 output; it is zeroed, then receives the
 *   device error bits (bit 0: a label >= V, bit 1: a bounded wait ran out).
 *   With NULL the bits go to the array and are not reported.
 * - Other arguments as for cce_forward; H is bf16 [M, D], W dense bf16.
 */
#define CCE_NOALLOC_SCRATCH_BYTES (32u << 20)
cce_status cce_forward_noalloc(const void* H, int64_t M, const cce_head* W,
                               const int32_t* labels, float* logp, float* lse,
                               float* tgt_logit, float* blockmax,
                               uint32_t* status, cce_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CCE_H_ */
