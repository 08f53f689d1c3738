/*
 * kda.h -- KDA (Kimi Delta Attention) forward, and its gradient, on NVIDIA B200 (sm_100a).
 *
 * A C-ABI library (libkda_b200.so).  Plain pointers and sizes only; every
 * pointer is a DEVICE pointer unless its name ends in _host.  The caller owns
 * every buffer.  All work is enqueued asynchronously on `stream`; the
 * functions never allocate device memory and never synchronise the stream.
 *
 * The layer (Kimi K3 report explainer, affta.cn, section
 * "第一关：KDA 解决算得动"): per (sequence n, head h) a fixed-size state
 * S in R^{dk x dv} (fp32 here), and for every token t, in this order:
 *   1. forget        S <- Diag(alpha_t) S,  alpha_t = exp(g_t) per key channel
 *                    (channel-wise forget gate: each state direction decays at
 *                    its own rate)
 *   2. delta write   u = beta_t (v_t - S^T k_t);  S <- S + k_t u^T
 *                    (read the state with the key, compare with the value,
 *                    write only the error, scaled by the update strength)
 *   3. read          o_t = S^T (scale q_t)
 *   4. output gate   y_t = gate_t (.) o_t   (full-rank: one gate per channel)
 *
 * Decay floor (same page and section): a channel keeps at least about 0.67%
 * of its state per step, i.e. ln(0.0067) <= g <= 0.  This is a PRECONDITION
 * of kda_chunk_fwd (it is what keeps every decay ratio inside a 16-token
 * chunk within BF16/FP32 range -- prism.simon-ai.net, "从架构创新出发：K3的MoE
 * 与混合注意力设计", section "数值稳定性与 Co-Design：BF16 约束下的衰减控制策略").
 * It is not checked on the device; values below the floor may overflow to
 * inf/NaN in the output.  g must also be finite and <= 0.
 *
 * Layouts ("THD", packed variable length):
 *   q, k, g   [total_tokens][H][dk]   contiguous, element type = dtype
 *   v, gate   [total_tokens][H][dv]   contiguous, element type = dtype
 *   beta      [total_tokens][H]       contiguous, element type = dtype
 *   out       [total_tokens][H][dv]   contiguous, element type = dtype
 *   cu_seqlens[num_seqs + 1] int32, cu_seqlens[0] = 0, non-decreasing,
 *             cu_seqlens[num_seqs] = total_tokens.  Sequence n is tokens
 *             [cu_seqlens[n], cu_seqlens[n+1]).  Chunks never cross a
 *             sequence boundary.
 *   states    [num_seqs][H][dk][dv]   fp32, dv contiguous.
 *
 * Supported sizes: dk, dv in {64, 128}; H >= 1; dtype BF16 or F32 (all of q,
 * k, v, g, beta, gate, out share it; states are always fp32).  Arithmetic:
 * fp32 accumulation and an fp32 state; BF16 inputs feed the tensor cores as
 * bf16; F32 inputs are computed in fp32 throughout.  Output is rounded to
 * nearest-even into dtype.
 *
 * Alignment: q, k, v, g, gate, out, states and workspace must be 16-byte
 * aligned; beta must be aligned to its element size.  KDA_ERR_ALIGNMENT
 * otherwise.
 *
 * Errors: every function validates its arguments on the host before launching
 * anything; on a validation error nothing is launched.  After launching, the
 * return value also reports cudaGetLastError() (KDA_ERR_CUDA).  Errors in
 * kernels that run later are reported by later CUDA calls on the stream.
 */
#ifndef KDA_B200_H
#define KDA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kda_stream_t; /* == cudaStream_t; NULL = legacy default stream */

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1, /* null pointer, negative size, inconsistent sizes */
    KDA_ERR_UNSUPPORTED = -2, /* dk/dv/dtype outside the supported set */
    KDA_ERR_ALIGNMENT = -3,   /* a pointer breaks the alignment rule above */
    KDA_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than required */
    KDA_ERR_CUDA = -5,        /* a CUDA runtime call failed (launch, attribute) */
    KDA_ERR_TIMEOUT = -6      /* reserved: a bounded device-side wait gave up */
} kda_status;

typedef enum { KDA_DTYPE_F32 = 0, KDA_DTYPE_BF16 = 1 } kda_dtype;

/* Human-readable name of a kda_status value (static string, never NULL). */
const char *kda_status_string(int status);

/* Bytes of device workspace kda_chunk_fwd needs for these sizes on the
 * current CUDA device (the plan depends on its SM count).  0 is never
 * returned for a valid call; returns 0 for invalid sizes. */
size_t kda_chunk_fwd_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H,
                                    int32_t dk, int32_t dv, kda_dtype dtype);

/* The prefill plan for these sizes on the current CUDA device: the piece
 * length (tokens; sequences longer than this are split into pieces whose
 * states are combined by a prefix scan), an upper bound on the number of
 * pieces, and the number of kernel launches one kda_chunk_fwd call makes.
 * Any output pointer may be NULL.  Returns KDA_OK or KDA_ERR_INVALID_ARG. */
int kda_chunk_fwd_plan(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t *piece_len,
                       int32_t *max_pieces, int32_t *launches);

/* Sub-pieces of the same plan (bf16, dk = dv = 128, the 16-token tcgen05
 * kernels): the summary pass cuts every piece that has a successor into this
 * many equal parts, summarised by separate CTAs so that the pass's waves fill
 * the GPU, and composes their affine maps into the piece's before the scan
 * (the piece states of the prefix scan, Kimi K3 report explainer, affta.cn,
 * section "KDA 上下文并行，让上下文的交接变薄", at two levels).  1 = none.
 * Returns the count (>= 1) or KDA_ERR_INVALID_ARG. */
int32_t kda_chunk_fwd_sub_pieces(int32_t total_tokens, int32_t num_seqs, int32_t H);

/*
 * Prefill: the layer over packed variable-length sequences, computed in
 * 16-token chunks (within a chunk by whole-block matrix products, between
 * chunks by carrying the state -- prism.simon-ai.net page, section
 * "计算范式演进：从递归低效到 GPU 友好的 Chunk Recurrent"), with long
 * sequences split into pieces whose state hand-offs are combined by a prefix
 * scan (affta.cn page, section "KDA 上下文并行，让上下文的交接变薄";
 * prism.simon-ai.net page, section "Linear Attention 的分层 Chunking 策略").
 *
 *   gate            may be NULL: y = o.
 *   cu_seqlens      device copy (required).
 *   cu_seqlens_host optional host copy; when given it is validated
 *                   (monotone, ends at total_tokens) -> KDA_ERR_INVALID_ARG.
 *   scale           multiplies q (1.0 = none).
 *   qk_l2norm       0: q, k used as given.  1: each q_t and k_t is divided
 *                   by sqrt(sum x^2 + 1e-6) first.
 *   initial_state   NULL = zeros.
 *   final_state     NULL = not written.  May alias initial_state exactly
 *                   (in-place state update); no other aliasing is allowed.
 *   workspace       >= kda_chunk_fwd_workspace_size(...) bytes; contents on
 *                   entry are ignored and on exit unspecified.
 * num_seqs == 0 or total_tokens == 0 with num_seqs > 0 is valid (empty
 * sequences copy initial_state to final_state).
 */
int kda_chunk_fwd(const void *q, const void *k, const void *v, const void *g, const void *beta,
                  const void *gate, void *out, const int32_t *cu_seqlens,
                  const int32_t *cu_seqlens_host, int32_t num_seqs, int32_t total_tokens,
                  int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, float scale,
                  int32_t qk_l2norm, const float *initial_state, float *final_state,
                  void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * Errors found on the device by kda_chunk_fwd / kda_chunk_fwd_ex are kept in
 * the first bytes of the workspace they ran with (cleared by each call):
 * offsets that are not monotone or do not end at total_tokens; a bounded
 * device wait that gave up; and, in the checked build of the library
 * (libkda_b200_checked.so, compiled with -DKDA_CHECK_G), a log-decay value
 * outside the precondition ln(0.0067) <= g <= 0 (with KDA_FLAG_CLAMP_DECAY
 * only g <= 0 is required), or NaN.  The release build does not check g.
 *
 * kda_chunk_fwd_check: waits for `stream` (this call, unlike the others,
 * synchronises), then reads those words.  Returns KDA_OK, KDA_ERR_INVALID_ARG
 * (bad offsets, or g out of range in the checked build; also for a NULL or
 * too-small workspace argument), KDA_ERR_TIMEOUT, or KDA_ERR_CUDA.  Call it
 * after the prefill and before the workspace is reused.
 *
 * kda_build_checks_g: 1 in the checked build, 0 in the release build.
 */
int kda_chunk_fwd_check(const void *workspace, size_t workspace_bytes, kda_stream_t stream);
int kda_build_checks_g(void);

/*
 * kda_chunk_fwd without a workspace argument, for callers that cannot
 * allocate device memory when they run the layer (code running inside an
 * allocator or memory-pool callback, runtimes that hand out only fixed
 * buffers, hosts that forbid allocation after start-up).  The pages have no
 * counterpart to this; it is a deployment convenience.
 *
 * Same arguments, semantics, argument checks and results as kda_chunk_fwd,
 * minus workspace.  The scratch the prefill needs (piece plan, per-piece
 * transitions and states) lives in a fixed 32 MiB array of device memory
 * owned by the library: it exists on every GPU that loads this code and is
 * held until the process exits.  The piece length is the usual one or, when
 * that plan does not fit, the shortest one that does; sizes whose plan does
 * not fit even with one piece per sequence are rejected with
 * KDA_ERR_WORKSPACE.  A call allocates nothing (no cudaMalloc/cudaFree,
 * directly or through a library).
 *
 * The array is placed on a device when the library's device code is loaded
 * there; under CUDA's lazy module loading (the default) that happens on the
 * first call into the library on that device, and is the one device
 * allocation this entry point implies.  Callers that may not allocate later
 * make one call at start-up (kda_chunk_fwd_noalloc_check(NULL) is enough),
 * and before any stream capture.  Each call looks the array's address up on
 * the current device.  All calls on a device share the array and its
 * contents persist between calls: calls that overlap on the GPU (other
 * streams, other host threads) race on it and must be serialised by the
 * caller.  No entry needs to start at zero; each call writes what it reads.
 *
 * Device-side errors (inconsistent device offsets, a bounded wait that gave
 * up, g out of range in the checked build) land in the array's first words,
 * as in a kda_chunk_fwd workspace; kda_chunk_fwd_noalloc_check waits for
 * `stream` and maps the words of the last call on the current device to a
 * status exactly as kda_chunk_fwd_check does (KDA_OK, KDA_ERR_INVALID_ARG,
 * KDA_ERR_TIMEOUT, or KDA_ERR_CUDA if the synchronisation or the 12-byte
 * copy fails).  It allocates nothing.
 */
int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *g,
                          const void *beta, const void *gate, void *out,
                          const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                          int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                          int32_t dv, kda_dtype dtype, float scale, int32_t qk_l2norm,
                          const float *initial_state, float *final_state, kda_stream_t stream);
int kda_chunk_fwd_noalloc_check(kda_stream_t stream);

/*
 * Decode: one token per sequence, the recurrence above applied once, state
 * updated in place.  Decode cost is this per-token state update
 * (prism.simon-ai.net page, section "推理瓶颈与Kimi K3的针对性优化").
 *
 *   q, k, g    [num_seqs][H][dk];  v, gate, out [num_seqs][H][dv];
 *   beta       [num_seqs][H];  gate may be NULL.
 *   state      [num_seqs][H][dk][dv] fp32, read and overwritten.
 * Same dtype, alignment and decay-floor rules as kda_chunk_fwd.  No
 * workspace.  qk_l2norm as for kda_chunk_fwd.
 */
int kda_decode_step(const void *q, const void *k, const void *v, const void *g, const void *beta,
                    const void *gate, void *out, float *state, int32_t num_seqs, int32_t H,
                    int32_t dk, int32_t dv, kda_dtype dtype, float scale, int32_t qk_l2norm,
                    kda_stream_t stream);

/*
 * Flags of the extended entry points (kda_chunk_fwd_ex, kda_decode_step_ex).
 * The preprocessing that the FlashKDA preparation stage folds into its kernel
 * (affta.cn page, section "FlashKDA ，让线性计算也能沾上并行的光"): q/k
 * normalisation, the squashing of the write strength and of the output gate,
 * and the decay floor of the forget gate (affta.cn page, section
 * "第一关：KDA 解决算得动": at least about 0.67% of the state survives a step).
 */
#define KDA_FLAG_QK_L2NORM 1    /* q_t, k_t divided by sqrt(sum x^2 + 1e-6) (= qk_l2norm) */
#define KDA_FLAG_BETA_LOGITS 2  /* beta holds logits: beta = 1 / (1 + exp(-x)) */
#define KDA_FLAG_GATE_LOGITS 4  /* gate holds logits: gate = 1 / (1 + exp(-x)) (when not NULL) */
#define KDA_FLAG_CLAMP_DECAY 8  /* g = max(g, ln 0.0067) per element */

/*
 * kda_chunk_fwd with a flags word instead of qk_l2norm, and optional state
 * snapshots (prefix caching at block granularity: the state at fixed token
 * boundaries of each sequence, so that a later call can resume from any of
 * them -- prism.simon-ai.net page, section "推理瓶颈与Kimi K3的针对性优化").
 *
 *   flags             any OR of the KDA_FLAG_* bits; other bits ->
 *                     KDA_ERR_INVALID_ARG.
 *   snapshot_tokens   0 = no snapshots.  Otherwise a multiple of 16: for
 *                     each sequence n of length L_n the state after tokens
 *                     m * snapshot_tokens, m = 1 .. (L_n - 1) / snapshot_tokens
 *                     (the state at L_n itself is the final state), is
 *                     written to
 *                     snapshots[((snapshot_offsets[n] + m - 1) * H + h) * dk * dv],
 *                     laid out [dk][dv] like the states.  Not a multiple of 16,
 *                     or negative -> KDA_ERR_INVALID_ARG.
 *   snapshots         device fp32, 16-byte aligned, at least
 *                     snapshot_offsets[num_seqs] * H * dk * dv floats; must not
 *                     overlap any other argument.  Required when
 *                     snapshot_tokens > 0.
 *   snapshot_offsets  device int32 [num_seqs + 1]: the caller's running sums
 *                     of (L_n - 1) / snapshot_tokens (0 for empty sequences).
 *                     Required when snapshot_tokens > 0.
 * Everything else as kda_chunk_fwd (same workspace size).
 */
int kda_chunk_fwd_ex(const void *q, const void *k, const void *v, const void *g, const void *beta,
                     const void *gate, void *out, const int32_t *cu_seqlens,
                     const int32_t *cu_seqlens_host, int32_t num_seqs, int32_t total_tokens,
                     int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, float scale, int32_t flags,
                     const float *initial_state, float *final_state, int32_t snapshot_tokens,
                     float *snapshots, const int32_t *snapshot_offsets, void *workspace,
                     size_t workspace_bytes, kda_stream_t stream);

/* kda_decode_step with a flags word (KDA_FLAG_*) instead of qk_l2norm. */
int kda_decode_step_ex(const void *q, const void *k, const void *v, const void *g, const void *beta,
                       const void *gate, void *out, float *state, int32_t num_seqs, int32_t H,
                       int32_t dk, int32_t dv, kda_dtype dtype, float scale, int32_t flags,
                       kda_stream_t stream);

/*
 * Context parallelism (affta.cn page, section "KDA 上下文并行，让上下文的交接变薄";
 * prism.simon-ai.net page, section "Linear Attention 的分层 Chunking 策略"):
 * the tokens of a sequence segment act on an incoming state as one affine
 * map S -> transition * S + zero_state, of fixed size whatever the segment's
 * length.  A sequence split over devices exchanges only these maps; each
 * device folds the maps of the segments before its own into its incoming
 * state (kda_state_compose) and runs kda_chunk_fwd from there.
 *
 * kda_chunk_fwd_summary: the map of every sequence of a packed batch.
 *   k, v, g, beta, cu_seqlens, cu_seqlens_host, sizes, dtype: as kda_chunk_fwd
 *                 (q and gate are not needed: the map does not depend on them).
 *   flags         KDA_FLAG_* (the gate flag has no effect here).
 *   transition    device fp32 [num_seqs][H][dk][dk], written.
 *   zero_state    device fp32 [num_seqs][H][dk][dv], written: the state the
 *                 sequence's tokens produce from zero.
 *   workspace     >= kda_chunk_fwd_workspace_size(total_tokens, num_seqs, H,
 *                 dk, dv, dtype) bytes.
 * An empty sequence has the identity map.  Errors as kda_chunk_fwd.
 */
int kda_chunk_fwd_summary(const void *k, const void *v, const void *g, const void *beta,
                          const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                          int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                          kda_dtype dtype, int32_t flags, float *transition, float *zero_state,
                          void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_state_compose: state_out = map[count-1]( ... map[0](state_in) ...) for
 * every (sequence, head), map[i](S) = transitions[i] S + zero_states[i], fp32.
 *   transitions   device fp32 [count][num_seqs][H][dk][dk].
 *   zero_states   device fp32 [count][num_seqs][H][dk][dv].
 *   state_in      device fp32 [num_seqs][H][dk][dv]; NULL = zeros.
 *   state_out     device fp32 [num_seqs][H][dk][dv]; may alias state_in
 *                 exactly, no partial overlap (KDA_ERR_INVALID_ARG).
 * count = 0 copies state_in (or writes zeros).  All pointers 16-byte aligned.
 */
int kda_state_compose(const float *transitions, const float *zero_states, int32_t count,
                      const float *state_in, float *state_out, int32_t num_seqs, int32_t H,
                      int32_t dk, int32_t dv, kda_stream_t stream);

/* ------------------------------------------------------------------ backward
 * Gradients of the plain forward (kda_chunk_fwd with qk_l2norm = 0: beta and
 * gate as given, the delta-rule write) for the loss
 *   L = sum dy (.) y + sum d_final_state (.) final_state.
 * The pages state the forward only (Kimi K3 report explainer, affta.cn,
 * section "第一关：KDA 解决算得动": forget, corrective write with an update
 * strength, read, output gate); this is its 16-token chunk form
 * (prism.simon-ai.net, section "计算范式演进：从递归低效到 GPU 友好的 Chunk
 * Recurrent") differentiated by the chain rule: per-chunk operands in
 * parallel, a forward pass over the chunks storing the state entering each,
 * a reverse pass carrying dL/dS, then the per-chunk gradients in parallel
 * (three launches on `stream`; the two passes over the chunks share one).
 * fp32 accuracy (products with a whole state on split-tf32 tensor-core
 * tiles); every output element is written once, so results are
 * deterministic.
 *
 * kda_bwd_workspace_size: bytes of workspace kda_bwd needs (0 for
 *   unsupported sizes).  With ch = (total_tokens / 16 + num_seqs) * H chunk
 *   slots: ch * (49 dk + 16 dv + 256 + 2 dk dv + 32 dv) floats (per-chunk
 *   operands, the state entering and dL/d(state leaving) each chunk, U and
 *   dL/dU), each region rounded up to 256 bytes.
 *
 * kda_bwd:
 *   q, k, g       device [total_tokens][H][dk], dtype; v, gate, dy device
 *                 [total_tokens][H][dv], dtype (gate may be NULL: y = o);
 *                 beta device [total_tokens][H], dtype.  Element-aligned.
 *   cu_seqlens, cu_seqlens_host, num_seqs, total_tokens, H, dk, dv, dtype,
 *                 scale: as kda_chunk_fwd (dk, dv in {64, 128}).  The device
 *                 offsets are clamped into [0, total_tokens] in the kernel.
 *   initial_state device fp32 [num_seqs][H][dk][dv] or NULL (zeros).
 *   d_final_state device fp32 [num_seqs][H][dk][dv] or NULL (zeros).
 *   dq, dk_out, dg  device fp32 [total_tokens][H][dk], written.
 *   dv_out          device fp32 [total_tokens][H][dv], written.
 *   dbeta           device fp32 [total_tokens][H], written.
 *   dgate           device fp32 [total_tokens][H][dv] or NULL (must be NULL
 *                   when gate is NULL -> KDA_ERR_INVALID_ARG).
 *   d_initial_state device fp32 [num_seqs][H][dk][dv] or NULL.
 *   workspace       >= kda_bwd_workspace_size(...) bytes, 256-byte aligned.
 * Gradient outputs are 4-byte aligned; all device buffers stay owned by the
 * caller.  Errors: as kda_chunk_fwd.
 */
size_t kda_bwd_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                              int32_t dv);

int kda_bwd(const void *q, const void *k, const void *v, const void *g, const void *beta,
            const void *gate, const void *dy, const int32_t *cu_seqlens,
            const int32_t *cu_seqlens_host, int32_t num_seqs, int32_t total_tokens, int32_t H,
            int32_t dk, int32_t dv, kda_dtype dtype, float scale, const float *initial_state,
            const float *d_final_state, float *dq, float *dk_out, float *dv_out, float *dg,
            float *dbeta, float *dgate, float *d_initial_state, void *workspace,
            size_t workspace_bytes, kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_H */
