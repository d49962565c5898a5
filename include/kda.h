/*
 * kda.h — C ABI of libkda.so: the Kimi Delta Attention (KDA) gated delta rule on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (one head; dk x dv fp32 state S; per token t):
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 * i.e. the state is decayed per key channel by exp(g_t) (g_t <= 0), corrected by
 * the delta rule with strength beta_t along k_t, written with k_t v_t^T and read
 * with q_t after the write.  The query scale is 1.  Sources: the open-model-atlas
 * page "Kimi-K3 ?inspect=blocks" (self.layers: 69 KDA layers keep a state of fixed
 * size between calls) and maxtext PR #5548's review, item 2 (KDA tensors A_log,
 * dt_bias, conv weights and o_norm kept in F32; exp(A_log) drives the decay).
 *
 * Entry points
 *   kda_forward_chunked          chunked prefill: outputs and final state
 *   kda_forward_chunked_varlen   the same over N packed sequences (cu_seqlens)
 *   kda_decode_step              one token per sequence, state in place
 *   kda_layer_forward            the layer core (conv + SiLU, L2-norm, gate, beta,
 *                                recurrence, RMSNorm x sigmoid gate); _noalloc and
 *                                _varlen variants
 *   kda_layer_decode_step        one decode step of the layer core with a conv cache
 *   kda_backward_chunked         gradients of the recurrence's inputs
 *   kda_*_workspace_size, kda_check_device_error, kda_status_string, kda_abi_version
 *   kda_set_wait_test_hooks      wait limit and failure injection for the failure path
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless a comment says otherwise; the caller owns
 *     and allocates every buffer.  The library allocates no device memory in any call
 *     (kda_layer_forward_noalloc uses a fixed array the library holds from load time).
 *   - Layouts are dense and row-major (last index fastest):
 *       q, k, g : [B, T, H, dk]      v, out : [B, T, H, dv]      beta : [B, T, H]
 *       state   : [B, H, dk, dv] fp32
 *   - Every tensor pointer must be 16-byte aligned (KDA_ERR_MISALIGNED otherwise).
 *   - Calls are asynchronous on `stream` and never synchronise it.  KDA_OK means the
 *     arguments were valid and the kernels were launched.  Arguments are validated
 *     before anything is launched; on any error nothing is launched and no output
 *     is touched.  Faults inside kernels and bounded-wait timeouts surface through
 *     kda_check_device_error() (which synchronises the stream).
 *   - The library never aborts, exits or prints.  It is reentrant; concurrent calls
 *     on different streams must not share output buffers.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null required pointer, non-positive size, bad enum  */
    KDA_ERR_UNSUPPORTED = 2,  /* valid but not built: head dims, chunk size, dtype    */
    KDA_ERR_MISALIGNED = 3,   /* a tensor pointer is not 16-byte aligned              */
    KDA_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, attribute, ...)  */
    KDA_ERR_TIMEOUT = 5,      /* a kernel's bounded wait gave up (device error word)  */
    KDA_ERR_WORKSPACE = 6     /* workspace missing or smaller than required           */
} kda_status_t;

typedef enum {
    KDA_F32 = 0,  /* q, k, v, g, beta, out (and the layer's raw inputs) are float32  */
    KDA_BF16 = 1  /* ... are bfloat16; the state is always float32                   */
} kda_dtype_t;

/* Static, NUL-terminated description of a status code (never NULL). */
const char *kda_status_string(kda_status_t status);

/* Version of this ABI (major * 100 + minor). */
int kda_abi_version(void);

/*
 * Chunked prefill (chunkwise-parallel form of the recurrence; results equal the
 * token-by-token recurrence up to rounding).
 *   q, k, g       [B, T, H, dk]   io dtype; g is the per-channel log-decay (<= 0)
 *   v             [B, T, H, dv]   io dtype
 *   beta          [B, T, H]       io dtype, the delta-rule strength in [0, 1]
 *   initial_state [B, H, dk, dv]  fp32, or NULL for a zero initial state
 *   out           [B, T, H, dv]   io dtype (written)
 *   final_state   [B, H, dk, dv]  fp32, or NULL to skip; may equal initial_state
 *                                 (in-place state passing)
 *   chunk         must be 64.
 * Supported: dk, dv in {64, 128} in either io dtype.  io KDA_BF16 with dk = dv = 128 runs
 * on the tcgen05 tensor-core kernel only: on a device or driver where that kernel cannot
 * run the call returns KDA_ERR_UNSUPPORTED (no slower kernel is substituted).  io KDA_F32
 * and the other bf16 head-dim pairs run exact fp32 CUDA-core kernels.  T = 0 is valid: out
 * is untouched and final_state receives initial_state (or zeros).
 */
kda_status_t kda_forward_chunked(const void *q, const void *k, const void *v, const void *g,
                                 const void *beta, const float *initial_state, void *out,
                                 float *final_state, int B, int T, int H, int dk, int dv,
                                 int chunk, kda_dtype_t io, kda_stream_t stream);

/*
 * Bytes of device workspace kda_backward_chunked needs: for every 16-token chunk, the fp32
 * state at its start (d * d floats) and the chunk's forward quantities U and X = V - K^ S
 * (2 * 16 * d floats) and its three 16 x 16 matrices, so
 * B * H * ceil(T / 16) * (d * d + 32 * d + 768) * 4 with d = dk.  dk must equal dv
 * (KDA_ERR_UNSUPPORTED otherwise).  *bytes is written on KDA_OK.
 */
kda_status_t kda_backward_workspace_size(int B, int T, int H, int dk, int dv, kda_dtype_t io,
                                         size_t *bytes);

/*
 * kda_backward_chunked — gradients of the recurrence of kda_forward_chunked (training;
 * the pages' runs differentiate the KDA layer: maxtext PR #5550, its jax.grad test and the
 * C4 training steps).  Given d_out = dL/dout and d_final_state = dL/dS_T, writes dL/d of
 * every input.  Computed in fp32 from the io-dtype inputs: a forward sweep stores each
 * 16-token chunk's start state and forward quantities in `workspace`, then a reverse sweep
 * reloads them and applies the chain rule (pairwise decays exp(G_i - G_j), j <= i, so no
 * gate overflows).
 *   q, k, g, v, beta, initial_state   as kda_forward_chunked (inputs, unchanged)
 *   d_out          [B, T, H, dv] io dtype
 *   d_final_state  [B, H, dk, dv] fp32 or NULL (zero)
 *   d_q, d_k, d_g  [B, T, H, dk] io dtype (written; d_g is the gradient of the log-decay g)
 *   d_v            [B, T, H, dv] io dtype (written)
 *   d_beta         [B, T, H] io dtype (written)
 *   d_initial_state [B, H, dk, dv] fp32 (written) or NULL; may equal d_final_state
 *   workspace      device buffer of kda_backward_workspace_size() bytes, 256-byte aligned
 * Supported: dk = dv in {64, 128}, both dtypes.  T = 0: d_initial_state receives
 * d_final_state (or zeros).
 */
kda_status_t kda_backward_chunked(const void *q, const void *k, const void *v, const void *g,
                                  const void *beta, const float *initial_state, const void *d_out,
                                  const float *d_final_state, void *d_q, void *d_k, void *d_v,
                                  void *d_g, void *d_beta, float *d_initial_state, void *workspace,
                                  size_t workspace_bytes, int B, int T, int H, int dk, int dv,
                                  kda_dtype_t io, kda_stream_t stream);

/*
 * kda_forward_chunked_varlen — chunked prefill of N packed sequences of different lengths
 * (the variable-length batches that segment ids or a padding mask describe; the MaxText
 * port of the Kimi-K3 model rejects packing for KDA).  Each sequence runs the recurrence
 * from its own initial state; no state crosses a sequence boundary.
 *   q, k, g       [T_total, H, dk]  io dtype, the sequences' tokens back to back
 *   v             [T_total, H, dv]  io dtype
 *   beta          [T_total, H]      io dtype
 *   cu_seqlens    [N + 1] int32, DEVICE memory: sequence n is tokens cu_seqlens[n] ..
 *                 cu_seqlens[n + 1] - 1.  Expected non-decreasing from 0 to T_total.  The
 *                 values are read on the device only and are not checked; every offset is
 *                 clamped into [0, T_total] (and each end to at least its start), so no
 *                 access leaves the buffers, but other malformed arrays give unspecified
 *                 results.  A zero-length sequence passes its initial state through.
 *   initial_state [N, H, dk, dv]  fp32 or NULL (zeros)
 *   out           [T_total, H, dv]  io dtype (written at every token of the N sequences)
 *   final_state   [N, H, dk, dv]  fp32 or NULL; may equal initial_state
 *   chunk         must be 64.
 * Supported: as kda_forward_chunked.  T_total = 0: final_state receives initial_state.
 */
kda_status_t kda_forward_chunked_varlen(const void *q, const void *k, const void *v, const void *g,
                                        const void *beta, const float *initial_state, void *out,
                                        float *final_state, const int *cu_seqlens, int N,
                                        int T_total, int H, int dk, int dv, int chunk,
                                        kda_dtype_t io, kda_stream_t stream);

/*
 * One decode step: the recurrence for a single new token per sequence, with the
 * state updated in place (read once, written once).
 *   q, k, g [B, H, dk] io dtype; v, out [B, H, dv] io dtype; beta [B, H] io dtype;
 *   state [B, H, dk, dv] fp32, read and overwritten.
 * Supported: dk, dv in {64, 128}, both dtypes.
 */
kda_status_t kda_decode_step(const void *q, const void *k, const void *v, const void *g,
                             const void *beta, float *state, void *out, int B, int H, int dk,
                             int dv, kda_dtype_t io, kda_stream_t stream);

/*
 * Bytes of device workspace kda_layer_forward needs for these sizes.  0 for bf16 at
 * dk = dv = 128, whose prologue, chunked step and epilogue run as one tensor-core kernel;
 * otherwise the fp32 prologue outputs and the chunked step's output (q, k, g, v, beta, o in
 * fp32, each rounded up to 256 bytes).  *bytes is written on KDA_OK.
 */
kda_status_t kda_layer_workspace_size(int B, int T, int H, int dk, int dv, kda_dtype_t io,
                                      size_t *bytes);

/*
 * KDA layer core: prologue -> chunked gated delta rule -> epilogue.
 *   prologue  q = l2norm(SiLU(conv_q * q_raw)), k = l2norm(SiLU(conv_k * k_raw)),
 *             v = SiLU(conv_v * v_raw)   (depthwise causal conv, kernel 4, zero history,
 *                                          PyTorch Conv1d tap order; l2norm eps 1e-6)
 *             g = max(-exp(A_log[h]) * softplus(g_raw + dt_bias), gate_lower_bound),
 *             beta = sigmoid(b_raw)
 *   epilogue  out = o_norm_w * cast_io(o * rsqrt(mean_dv(o^2) + norm_eps)) * sigmoid(o_gate_raw)
 * (open-model-atlas "Kimi-K3" linear_attn_config: short_conv_kernel_size 4;
 *  atlas.klimoza.dev KimiRMSNorm excerpt; maxtext PR #5543 sigmoid output gate.)
 *   q_raw, k_raw  [B, T, H*dk]  io dtype      v_raw       [B, T, H*dv]  io dtype
 *   conv_q, conv_k [H*dk, 4] fp32             conv_v      [H*dv, 4]     fp32
 *   g_raw         [B, T, H, dk] io dtype      A_log       [H]           fp32
 *   dt_bias       [H*dk] fp32 or NULL (zero)  b_raw       [B, T, H]     io dtype
 *   gate_lower_bound  a lower bound on every log-decay g, <= 0; -INFINITY for none.  (The
 *                 Kimi-K3 linear-attention config sets gate_lower_bound = -5.0 and gives no
 *                 formula; it is read as a bound on g itself, so that no token decays the
 *                 state by more than exp(bound) per channel.)  NaN or > 0: KDA_ERR_INVALID_ARG.
 *   o_gate_raw    [B, T, H, dv] io dtype      o_norm_w    [dv] fp32 or NULL (ones)
 *   initial_state / final_state as in kda_forward_chunked.
 *   out           [B, T, H, dv] io dtype (written)
 *   workspace     device buffer of at least kda_layer_workspace_size() bytes, 256-byte
 *                 aligned (may be NULL when that size is 0).
 * Supported: dk, dv in {64, 128}, both dtypes (as kda_forward_chunked).
 */
kda_status_t kda_layer_forward(const void *q_raw, const void *k_raw, const void *v_raw,
                               const float *conv_q, const float *conv_k, const float *conv_v,
                               const void *g_raw, const float *A_log, const float *dt_bias,
                               float gate_lower_bound, const void *b_raw, const void *o_gate_raw,
                               const float *o_norm_w, float norm_eps, const float *initial_state,
                               void *out, float *final_state, void *workspace, size_t workspace_bytes,
                               int B, int T, int H, int dk, int dv, kda_dtype_t io,
                               kda_stream_t stream);

/*
 * kda_layer_forward_varlen — kda_layer_forward over N packed sequences of different lengths
 * (the padding-mask / segment-id case; see kda_forward_chunked_varlen).  Every raw tensor is
 * token-major over T_total tokens ([T_total, H*dk], [T_total, H, dk], [T_total, H], ...);
 * states are [N, H, dk, dv]; cu_seqlens is the device int32 [N + 1] offsets array (same
 * rules as kda_forward_chunked_varlen).  The short conv's history is zero before each
 * sequence's first token, so no input of one sequence reaches another's outputs.
 * Workspace: kda_layer_workspace_size(1, T_total, H, dk, dv, io) bytes.
 */
kda_status_t kda_layer_forward_varlen(const void *q_raw, const void *k_raw, const void *v_raw,
                                      const float *conv_q, const float *conv_k, const float *conv_v,
                                      const void *g_raw, const float *A_log, const float *dt_bias,
                                      float gate_lower_bound, const void *b_raw, const void *o_gate_raw,
                                      const float *o_norm_w, float norm_eps, const float *initial_state,
                                      void *out, float *final_state, const int *cu_seqlens, void *workspace,
                                      size_t workspace_bytes, int N, int T_total, int H, int dk, int dv,
                                      kda_dtype_t io, kda_stream_t stream);

/* Size in bytes of the built-in scratch that kda_layer_forward_noalloc uses (64 MiB). */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * kda_layer_forward_noalloc — kda_layer_forward for callers that cannot allocate device
 * memory on their call path: a serving loop whose device memory is planned once at
 * start-up, a plugin or callback interface that provides no allocator, or code that
 * cannot pay for cudaMalloc (which may synchronise the device).  The paper has no
 * counterpart to this entry point; it exists for those callers only.
 *   Arguments, layouts and results are those of kda_layer_forward without the workspace
 *   pair.  The caller still owns and passes every input and output.
 *   Scratch: a library-owned device array of KDA_NOALLOC_SCRATCH_BYTES, held by every GPU
 *   that loads the library until the process exits.  Sizes whose workspace
 *   (kda_layer_workspace_size) exceeds it are rejected with KDA_ERR_WORKSPACE before
 *   anything runs.  All calls share the array and it keeps the last call's contents;
 *   each call writes every scratch byte it reads, so nothing needs clearing.  Calls that
 *   overlap on the GPU (other streams or host threads) race on it and must be serialised
 *   by the caller.
 *   The first call on each device looks up the array's device address (with that device
 *   current); make that first call before any stream capture begins.
 */
kda_status_t kda_layer_forward_noalloc(const void *q_raw, const void *k_raw, const void *v_raw,
                                       const float *conv_q, const float *conv_k,
                                       const float *conv_v, const void *g_raw, const float *A_log,
                                       const float *dt_bias, float gate_lower_bound, const void *b_raw,
                                       const void *o_gate_raw, const float *o_norm_w,
                                       float norm_eps, const float *initial_state, void *out,
                                       float *final_state, int B, int T, int H, int dk, int dv,
                                       kda_dtype_t io, kda_stream_t stream);

/*
 * kda_layer_decode_step — one decode step of the layer core for B sequences: the prologue,
 * the gated delta rule and the epilogue of kda_layer_forward for the single new token t,
 * with the conv history kept in a cache instead of recomputed.
 *   y = SiLU(w[c,0] x[t-3] + w[c,1] x[t-2] + w[c,2] x[t-1] + w[c,3] x[t])  per channel, for q,
 *   k and v, x[t-3..t-1] read from the cache, which then shifts in x[t]; then as
 *   kda_layer_forward: q, k L2-normalised, g, beta, the state update
 *   S <- (I - beta k k^T) Diag(exp g) S + beta k v^T, o = S^T q, RMSNorm x gain x sigmoid gate.
 * (The Kimi-K3 linear-attention config's short conv of kernel 4; the pages note that KDA
 *  decode with a cached state is not yet implemented in the MaxText port.)
 *   q_raw, k_raw  [B, H*dk] io dtype         v_raw        [B, H*dv] io dtype
 *   cache_q, cache_k [B, 3, H*dk] io dtype   cache_v      [B, 3, H*dv] io dtype
 *                 updated in place; tap 0 is the oldest token (t-3); zeros = empty history
 *   conv_q, conv_k [H*dk, 4] fp32            conv_v       [H*dv, 4] fp32
 *   g_raw         [B, H, dk] io dtype        A_log        [H] fp32
 *   dt_bias       [H*dk] fp32 or NULL        b_raw        [B, H] io dtype
 *   gate_lower_bound  as in kda_layer_forward (-INFINITY for none)
 *   o_gate_raw    [B, H, dv] io dtype        o_norm_w     [dv] fp32 or NULL (ones)
 *   state         [B, H, dk, dv] fp32, updated in place
 *   out           [B, H, dv] io dtype (written)
 * Supported: dk = dv = 128 (KDA_ERR_UNSUPPORTED otherwise), both dtypes.  Every pointer
 * 16-byte aligned.  n calls from an empty cache and state give the outputs of
 * kda_layer_forward over the same n tokens.
 */
kda_status_t kda_layer_decode_step(const void *q_raw, const void *k_raw, const void *v_raw,
                                   const float *conv_q, const float *conv_k, const float *conv_v,
                                   void *cache_q, void *cache_k, void *cache_v, const void *g_raw,
                                   const float *A_log, const float *dt_bias, float gate_lower_bound,
                                   const void *b_raw, const void *o_gate_raw, const float *o_norm_w,
                                   float norm_eps, float *state, void *out, int B, int H, int dk, int dv,
                                   kda_dtype_t io, kda_stream_t stream);

/*
 * kda_set_wait_test_hooks — the failure path of the tensor-core kernels, made testable
 * without a GPU fault.  Those kernels wait on their own mbarriers (tile loads, MMA
 * completion) with a time limit; a wait that runs out sets the device error word, makes
 * the whole CTA stop, wait for everything it already issued (loads, MMAs, copies, stores),
 * free its tensor memory and return, so the context stays usable and the next
 * kda_check_device_error returns KDA_ERR_TIMEOUT.  The paper has no counterpart to this
 * entry point.
 *   wait_limit_ns    limit of each such wait, in ns of %globaltimer; 0 restores the
 *                    default of 2 s
 *   skip_load_chunk  >= 0: in every later launch, the tile load of that chunk index is
 *                    never issued, so the wait for it runs out after the limit (the
 *                    kernel's outputs from that chunk on are then unspecified); -1: off
 * The settings are process-wide and read at each launch of those kernels; change them only
 * while no call is being made from another host thread.  Always returns KDA_OK.
 */
kda_status_t kda_set_wait_test_hooks(unsigned long long wait_limit_ns, int skip_load_chunk);

/*
 * Synchronises `stream`, then reports and clears the library's device error word
 * (set by a kernel whose bounded wait gave up) and any sticky CUDA error.
 * Returns KDA_OK, KDA_ERR_TIMEOUT or KDA_ERR_CUDA.
 */
kda_status_t kda_check_device_error(kda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
