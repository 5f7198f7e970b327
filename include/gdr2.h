/*
 * gdr2.h -- C ABI of libgdr2.so, the B200 (sm_100a) implementation of the
 * Gated Delta Rule-2 (GDR-2) token mixer from "Gated DeltaNet-2: Decoupling
 * Erase and Write in Linear Attention" (Hatamizadeh, Choi, Kautz).
 *
 * The operation (per batch index b and head h, independently):
 *
 *   e_t = b_t (.) k_t,   z_t = w_t (.) v_t,   a_t = exp(log_alpha_t)
 *   S_t = (I - k_t e_t^T) Diag(a_t) S_{t-1} + k_t z_t^T          (dk x dv state)
 *   o_t = S_t^T q_t
 *
 * Sources: the note's sec. 3 forward-pass paragraph (gated key and value,
 * decay, read), sec. 2 fast-weight objective and the sec. 3 gate-aware
 * backward paragraph (erase outer product along k: the asymmetric factor
 * (I - k_t e_t^T)); sec. 3 chunkwise paragraph (decay-normalised state and
 * WY form used by the forward kernel); sec. 1 (constant-memory recurrent
 * decoding).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers:   all tensor pointers are DEVICE pointers (CUDA global memory) of
 *             the current device, contiguous in the layouts below, 16-byte
 *             aligned. The caller owns every buffer; the library allocates no
 *             device memory. Scratch, where an entry point needs any, is a
 *             caller buffer sized by the matching *_workspace_bytes query
 *             (gdr2_backward_noalloc instead uses a fixed array inside the
 *             library; see there).
 * Layouts:    token tensors are token-major:
 *               q, k, log_alpha, b          [B, T, H, dk]
 *               v, w, o                     [B, T, H, dv]
 *             states are [B, H, dk, dv] fp32, row = key channel c,
 *             column = value channel j (dv contiguous).
 * Dtypes:     q, k, v, b, w, o and their gradients have the dtype `dt`
 *             (fp32 or bf16); log_alpha, its gradient and every state are
 *             fp32. Arithmetic is fp32 throughout; bf16 outputs are rounded
 *             to nearest even from fp32.
 * Decay:      log_alpha must not be NaN; values below -64 are treated as
 *             -64 (alpha = 1.6e-28, a reset to fp32 precision).
 * Streams:    `stream` is a cudaStream_t (NULL = legacy default stream).
 *             Every call is asynchronous on that stream and returns once
 *             the work is enqueued.
 * Errors:     argument errors are detected on the host before any launch and
 *             return GDR2_ERR_INVALID_ARG or GDR2_ERR_UNSUPPORTED with no
 *             work enqueued; launch failures return GDR2_ERR_CUDA. Kernels
 *             that wait on hardware barriers bound every wait; a kernel that
 *             gives up records it in a device status word that
 *             gdr2_sync_status() reports as GDR2_ERR_TIMEOUT. No exception
 *             or abort crosses the ABI. gdr2_last_error() describes the last
 *             non-OK status of the calling thread.
 * Sizes:      dk and dv must each be 64 or 128; B, T, H >= 0 (an empty
 *             problem is a no-op apart from copying S0 to S_T).
 */
#ifndef GDR2_H
#define GDR2_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDR2_ABI_VERSION 9
#define GDR2_CHUNK 64 /* tokens per chunk of the chunkwise forward */

typedef enum {
    GDR2_OK = 0,
    GDR2_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, ... */
    GDR2_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. dk = 96)   */
    GDR2_ERR_CUDA = 3,        /* launch or runtime failure                  */
    GDR2_ERR_TIMEOUT = 4      /* a kernel gave up a bounded device wait     */
} gdr2_status;

typedef enum {
    GDR2_F32 = 0,
    GDR2_BF16 = 1
} gdr2_dtype;

/*
 * Gate layouts for the *_gated entry points and gdr2_forward_varlen (bits of
 * `gates`): by default the erase gate b has d_k entries per token-head and the
 * write gate w d_v; with a bit set that gate is one value per token-head
 * ([B, T, H], or [T, H] packed, or [N, H] for decode), the same value in every
 * channel -- the scalar-gate ablations of the Gated DeltaNet-2 note (sec. 4),
 * and with both bits and b = w = beta the KDA / Gated DeltaNet gates (sec. 2).
 */
#define GDR2_GATE_SCALAR_B 1
#define GDR2_GATE_SCALAR_W 2

/* ABI version of the loaded library (GDR2_ABI_VERSION it was built with). */
int gdr2_abi_version(void);

/* Human-readable description of the calling thread's last non-OK status
 * (empty string if none). The pointer stays valid until the next call from
 * the same thread. */
const char *gdr2_last_error(void);

/* Bytes of device scratch gdr2_forward needs for this problem (0 when the
 * call runs on CUDA cores: fp32 inputs, or dk/dv other than 128). */
size_t gdr2_forward_workspace_bytes(int B, int T, int H, int dk, int dv, gdr2_dtype dt);

/*
 * gdr2_forward -- chunkwise forward over whole sequences (prefill/training).
 *   Computes o_t for every token and the final state S_T, starting from S0.
 *   Gated DeltaNet-2 note sec. 3: per chunk of GDR2_CHUNK tokens the decay
 *   is absorbed into the gated keys (decay-normalised state), the
 *   strictly-lower system (I + A) is solved in UT form, the WY factors give
 *   the chunk's pseudo-values, and the state is carried between chunks in
 *   fp32.
 * in:  q, k [B,T,H,dk] dt; v [B,T,H,dv] dt; log_alpha [B,T,H,dk] fp32;
 *      b [B,T,H,dk] dt; w [B,T,H,dv] dt;
 *      S0 [B,H,dk,dv] fp32 or NULL (zero initial state).
 * out: o [B,T,H,dv] dt; S_T [B,H,dk,dv] fp32 or NULL (not written);
 *      saved_states [B,H,ceil(T/64),dk,dv] fp32 or NULL: the state entering
 *      each chunk (chunk 0 receives S0), for gdr2_backward.
 * scratch: workspace of at least gdr2_forward_workspace_bytes(...) bytes,
 *      256-byte aligned (may be NULL when that size is 0); contents on entry
 *      do not matter. The bf16 path at d = 128 keeps each chunk's
 *      state-independent intermediates there (88.5 KiB per (b, h, chunk)),
 *      then a task queue counter and one ready flag per chunk for the fused
 *      kernel (chunk tasks and the per-(b, h) scans in one launch, used when
 *      B H leaves at least 32 SMs to the chunk tasks; the call clears them).
 * Input and output buffers must not overlap (S0 == S_T is allowed).
 */
gdr2_status gdr2_forward(int B, int T, int H, int dk, int dv, gdr2_dtype dt,
                         const void *q, const void *k, const void *v,
                         const float *log_alpha, const void *b, const void *w,
                         const float *S0, void *o, float *S_T, float *saved_states,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr2_forward_gated -- gdr2_forward with the gate layouts of `gates`
 * (GDR2_GATE_* bits); a scalar gate is [B, T, H] in the dtype dt, any element
 * alignment. Everything else as gdr2_forward; gates = 0 is gdr2_forward.
 */
gdr2_status gdr2_forward_gated(int B, int T, int H, int dk, int dv, gdr2_dtype dt, int gates,
                               const void *q, const void *k, const void *v, const float *log_alpha,
                               const void *b, const void *w, const float *S0,
                               void *o, float *S_T, float *saved_states,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr2_decode_step -- one recurrent token for N*H resident states
 *   (constant-memory decoding, Gated DeltaNet-2 note sec. 1; the per-token
 *   steps of sec. 3). One read and one write of S: with r = S^T(a (.) e) and
 *   s = S^T(a (.) q) taken from the old state, o = s + (z - r)(k . q) and
 *   S <- Diag(a) S + k (z - r)^T.
 * in:  q, k, b [N,H,dk] dt; v, w [N,H,dv] dt; log_alpha [N,H,dk] fp32.
 * in/out: S [N,H,dk,dv] fp32, updated in place.
 * out: o [N,H,dv] dt.
 */
gdr2_status gdr2_decode_step(int N, int H, int dk, int dv, gdr2_dtype dt,
                             const void *q, const void *k, const void *v,
                             const float *log_alpha, const void *b, const void *w,
                             float *S, void *o, void *stream);

/*
 * gdr2_decode_step_gated -- gdr2_decode_step with the gate layouts of `gates`
 * (GDR2_GATE_* bits); a scalar gate is [N, H]. gates = 0 is gdr2_decode_step.
 */
gdr2_status gdr2_decode_step_gated(int N, int H, int dk, int dv, gdr2_dtype dt, int gates,
                                   const void *q, const void *k, const void *v,
                                   const float *log_alpha, const void *b, const void *w,
                                   float *S, void *o, void *stream);

/* Bytes of device scratch gdr2_forward_varlen needs (N sequences, T tokens in all). */
size_t gdr2_forward_varlen_workspace_bytes(int N, int T, int H, int dk, int dv, gdr2_dtype dt);

/*
 * gdr2_forward_varlen -- gdr2_forward over N packed sequences of different
 * lengths. The pages' chunkwise forward applied to each sequence on its own:
 * each starts from its own S0 and stops at its own end, and no state or
 * product crosses from one sequence to the next. (The pages train on
 * sequences of one length; packing is how such layers are fed mixed lengths.)
 * in:  cu_seqlens [N + 1] int32, DEVICE memory: 0 = cu_seqlens[0] <=
 *      cu_seqlens[1] <= ... <= cu_seqlens[N] = T; sequence i is tokens
 *      cu_seqlens[i] .. cu_seqlens[i+1] - 1 (empty sequences are allowed).
 *      q, k, b [T, H, dk] (= [1, T, H, dk]) bf16; v, w [T, H, dv] bf16;
 *      log_alpha [T, H, dk] fp32; S0 [N, H, dk, dv] fp32 or NULL (zeros).
 * out: o [T, H, dv] bf16; S_T [N, H, dk, dv] fp32 or NULL.
 *      saved_states or NULL: the state entering each chunk, [C_total][dk][dv]
 *      fp32 with C_total <= H * (ceil(T / 64) + N) (allocate that many);
 *      sequence i's entries start at H * sum_{j<i} ceil(len_j / 64), head
 *      by head, its chunks in order within a head.
 * scratch: workspace of at least gdr2_forward_varlen_workspace_bytes(...)
 *      bytes, 256-byte aligned.
 * gates: GDR2_GATE_* bits (0 = vector gates); a scalar gate is [T, H].
 * Supported: bf16 inputs with dk = dv = 128 (GDR2_ERR_UNSUPPORTED otherwise).
 * cu_seqlens is read on the device only: if it breaks the rule above, the call
 * computes nothing and the next gdr2_sync_status returns GDR2_ERR_INVALID_ARG.
 */
gdr2_status gdr2_forward_varlen(int N, int T, int H, int dk, int dv, gdr2_dtype dt, int gates, const int *cu_seqlens,
                                const void *q, const void *k, const void *v, const float *log_alpha,
                                const void *b, const void *w, const float *S0,
                                void *o, float *S_T, float *saved_states,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr2_forward_ex -- the forward with every option in one call: dense
 * ([B, T, H, .], cu_seqlens = NULL; B = batch) or packed sequences
 * (cu_seqlens as in gdr2_forward_varlen; B = N sequences), the gate layouts of
 * `gates`, and the output epilogue of the Gated DeltaNet-2 block (note sec. 3,
 * block data-flow paragraph: the mixer output goes through an RMSNorm combined
 * with a SiLU output gate), applied to the bf16 o in fp32 arithmetic by a pass
 * over o and out_gate after the forward's kernels, on the same stream:
 *
 *   o[t, j] <- o[t, j] / sqrt(mean_j' o[t, j']^2 + norm_eps) * norm_weight[j]
 *              * silu(out_gate[t, j]),        silu(x) = x / (1 + exp(-x))
 *
 * with the mean over the dv channels of one token and head. Each factor is
 * optional: norm_weight = NULL skips the normalisation, out_gate = NULL the
 * gate. S_T and saved_states are the recurrence's own states, untouched by
 * the epilogue.
 * in:  out_gate same layout and dtype as o ([B, T, H, dv], or [T, H, dv]
 *      packed), 16-byte aligned, or NULL; norm_weight [dv] fp32 (4-byte
 *      aligned) or NULL; norm_eps finite and >= 0 (used only with
 *      norm_weight; with 0, a token whose o is all zero gives NaN).
 * scratch: gdr2_forward_workspace_bytes(...) dense,
 *      gdr2_forward_varlen_workspace_bytes(...) packed.
 * Supported: any case gdr2_forward_gated runs; packed sequences or an
 * epilogue need bf16 inputs with dk = dv = 128 (GDR2_ERR_UNSUPPORTED
 * otherwise). With cu_seqlens = NULL and no epilogue this is
 * gdr2_forward_gated; with cu_seqlens and no epilogue, gdr2_forward_varlen.
 */
gdr2_status gdr2_forward_ex(int B, int T, int H, int dk, int dv, gdr2_dtype dt, int gates, const int *cu_seqlens,
                            const void *q, const void *k, const void *v, const float *log_alpha,
                            const void *b, const void *w, const float *S0,
                            const void *out_gate, const float *norm_weight, float norm_eps,
                            void *o, float *S_T, float *saved_states,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Block prologue (Gated DeltaNet-2 note sec. 3, block data-flow paragraph: query and
 * key go linear -> conv -> SiLU -> L2 norm, the value linear -> conv -> SiLU, and three
 * separate branches give the decay and the erase and write gates). The linear
 * projections are the caller's; these two calls take their outputs to the mixer's
 * inputs. The note gives neither the convolution width nor the activation laws; the
 * readings taken are stated with each call.
 *
 * gdr2_short_conv_silu -- y = SiLU(causal depthwise convolution of x), then, with
 *   l2norm, y / sqrt(sum over the head's d channels of y^2 + l2_eps) per token and head.
 *   The convolution has the tap layout of a depthwise Conv1d weight [C, 1, W] left-padded
 *   by W - 1: y[t, c] = sum_i weight[c][i] x[t - (W - 1) + i, c] (the last tap is the
 *   current token); inputs before a sequence's first token come from state_in, or are 0.
 * in:  x [N, T, H, d] dt (dense; N sequences of T tokens), or [T, H, d] with cu_seqlens
 *      ([N + 1] int32 on the device, as for gdr2_forward_varlen; T = all tokens);
 *      weight [H * d][width] fp32 (channel c = h * d + j); width 1 .. 4;
 *      state_in [N][width - 1][H][d] dt or NULL: the width - 1 inputs before each
 *      sequence, oldest first.
 * out: y in x's layout (must not be x); state_out in state_in's layout or NULL: the last
 *      width - 1 inputs of [state_in; sequence] (a sequence without tokens keeps its
 *      state). state_out may be state_in only for T = 1 without cu_seqlens (a decode step,
 *      updated in place); otherwise the two must not overlap.
 * d is 64 or 128; dt fp32 or bf16 (arithmetic fp32); l2_eps finite and >= 0.
 * cu_seqlens is not checked here (gdr2_forward_varlen checks it): an array that breaks
 * the rule gives unspecified outputs, but every access stays inside the buffers above.
 * A bounded device wait that gives up is reported by gdr2_sync_status (TIMEOUT).
 */
gdr2_status gdr2_short_conv_silu(int N, int T, int H, int d, gdr2_dtype dt, int width, int l2norm, float l2_eps,
                                 const int *cu_seqlens, const void *x, const float *weight,
                                 const void *state_in, void *state_out, void *y, void *stream);

/*
 * gdr2_gate_activations -- the decay and gate branches' activations, element by element
 * over flat arrays (any layout: vector or scalar gates alike):
 *   log_alpha = -softplus(a) = -log(1 + e^a)   (so alpha = sigmoid(-a), in (0, 1))
 *   b = sigmoid(b_pre),  w = sigmoid(w_pre)
 * in:  a [n_alpha], b_pre [n_b], w_pre [n_w] in dt; any of them NULL (with its output) to
 *      skip it. out: log_alpha [n_alpha] fp32; b [n_b], w [n_w] in dt. 16-byte aligned.
 */
gdr2_status gdr2_gate_activations(gdr2_dtype dt, long long n_alpha, const void *a, float *log_alpha,
                                  long long n_b, const void *b_pre, void *b,
                                  long long n_w, const void *w_pre, void *w, void *stream);

/*
 * gdr2_segment_states -- the states entering the G segments of split sequences, for a
 * forward whose segments run at the same time (on one GPU as a batch, or one segment per
 * GPU). Across a segment the recurrence is affine in the entering state:
 * S_out = A_g S_in + B_g, with A_g the product of the segment's (I - k e^T) Diag(alpha)
 * factors -- the segment's final state from S0 = I with the write gate w = 0 -- and B_g its
 * final state from S0 = 0 (both from gdr2_forward). This call scans them in order:
 *   S_starts[g = 0] = S0,  S_starts[g + 1] = A_g S_starts[g] + B_g,  S_T = after the last.
 * in:  A [B][G][H][dk][dk] fp32, Bst [B][G][H][dk][dv] fp32 (the layout of a batched
 *      forward's S_T over B * G segments, segment index inside the batch index);
 *      S0 [B][H][dk][dv] fp32 or NULL (zeros).
 * out: S_starts [B][G][H][dk][dv] fp32; S_T [B][H][dk][dv] fp32 or NULL.
 * dk and dv are 64 or 128; fp32 arithmetic; buffers must not overlap.
 */
gdr2_status gdr2_segment_states(int B, int G, int H, int dk, int dv, const float *A, const float *Bst,
                                const float *S0, float *S_starts, float *S_T, void *stream);

/* Bytes of device scratch gdr2_backward needs for this problem. */
size_t gdr2_backward_workspace_bytes(int B, int T, int H, int dk, int dv, gdr2_dtype dt);

/*
 * gdr2_backward -- gate-aware backward (Gated DeltaNet-2 note sec. 3):
 *   gradients of L = <o, dO> + <S_T, dS_T> with respect to q, k, v,
 *   log_alpha, b, w and S0, through the asymmetric factor (I - k_t e_t^T).
 * in:  forward inputs as in gdr2_forward (S0 NULL = zeros); dO [B,T,H,dv] dt;
 *      dS_T [B,H,dk,dv] fp32 or NULL (zero);
 *      saved_states as written by gdr2_forward for the same inputs, or NULL
 *      (the states are recomputed).
 * out: dq, dk_, db [B,T,H,dk] dt; dv_, dw [B,T,H,dv] dt;
 *      dlog_alpha [B,T,H,dk] fp32; dS0 [B,H,dk,dv] fp32 or NULL.
 * scratch: workspace of at least gdr2_backward_workspace_bytes(...) bytes,
 *      256-byte aligned; its contents on entry do not matter.
 * Paths: bf16 inputs with dk = dv = 128 run the chunkwise tensor-core backward
 *      (the forward's chunk kernel again, a reverse scan of the state gradient
 *      over the chunks, then the chunk gradients of every chunk in parallel;
 *      deterministic, bf16 tensor-core operands with fp32 accumulation and an
 *      fp32 state gradient). Other inputs run a token-level kernel in fp32,
 *      whose per-key-channel gradients (dq, dk, db, dlog_alpha) are summed over
 *      the value columns with fp32 atomics, so their last bits may differ
 *      between calls.
 */
gdr2_status gdr2_backward(int B, int T, int H, int dk, int dv, gdr2_dtype dt,
                          const void *q, const void *k, const void *v,
                          const float *log_alpha, const void *b, const void *w,
                          const float *S0, const void *dO, const float *dS_T,
                          const float *saved_states,
                          void *dq, void *dk_, void *dv_, float *dlog_alpha,
                          void *db, void *dw, float *dS0,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr2_backward_gated -- gdr2_backward with the gate layouts of `gates`
 * (GDR2_GATE_* bits): a scalar gate b or w is [B, T, H] in the dtype dt (one
 * value per token-head, the scalar-erase and scalar-write ablations of the
 * note's sec. 4; both scalar and equal are the KDA and Gated DeltaNet gates of
 * sec. 2), and its gradient db or dw has the same layout: the sum over the
 * channels of the vector gate's gradient. Everything else as gdr2_backward;
 * gates = 0 is gdr2_backward. Scalar gates need bf16 inputs with
 * dk = dv = 128 (GDR2_ERR_UNSUPPORTED otherwise).
 */
gdr2_status gdr2_backward_gated(int B, int T, int H, int dk, int dv, gdr2_dtype dt, int gates,
                                const void *q, const void *k, const void *v,
                                const float *log_alpha, const void *b, const void *w,
                                const float *S0, const void *dO, const float *dS_T,
                                const float *saved_states,
                                void *dq, void *dk_, void *dv_, float *dlog_alpha,
                                void *db, void *dw, float *dS0,
                                void *workspace, size_t workspace_bytes, void *stream);

/* Size of the device scratch array behind gdr2_backward_noalloc (64 MiB). */
#define GDR2_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * gdr2_backward_noalloc -- gdr2_backward without a caller workspace and
 * without any device allocation. The paper has no counterpart: this is a
 * deployment variant for callers that may not allocate device memory, such as
 * a serving engine that reserves nearly all of HBM for its own pool at start-up
 * (a fresh cudaMalloc would fail or fragment that pool, and cudaFree
 * synchronises the device), or a host component that only receives device
 * pointers from another runtime and has no allocator of its own.
 * Scratch: a file-scope device array of GDR2_NOALLOC_SCRATCH_BYTES inside the
 *      library. Every GPU on which the library's backward module is loaded
 *      holds one such array until the process exits. The first call on a
 *      device looks up the array's device address (once per device, with that
 *      device current); make that first call before any stream capture.
 * Sharing: all calls on a device share the one array and it keeps the last
 *      call's contents (nothing in it needs to start at zero). Calls that
 *      overlap on the GPU -- on different streams, or from different host
 *      threads -- race on it; serialise them.
 * Limit: a problem whose scratch (gdr2_backward's workspace minus the chunk
 *      states when saved_states is given) exceeds GDR2_NOALLOC_SCRATCH_BYTES
 *      returns GDR2_ERR_UNSUPPORTED before any work is enqueued. At
 *      dk = dv = 128 with saved_states that is about 4.2 MiB per (batch, head)
 *      plus 2 KiB per (batch, head, token).
 * Arguments, layouts and results are those of gdr2_backward. The call itself
 * makes no cudaMalloc, cudaFree or other allocating call.
 */
gdr2_status gdr2_backward_noalloc(int B, int T, int H, int dk, int dv, gdr2_dtype dt,
                                  const void *q, const void *k, const void *v,
                                  const float *log_alpha, const void *b, const void *w,
                                  const float *S0, const void *dO, const float *dS_T,
                                  const float *saved_states,
                                  void *dq, void *dk_, void *dv_, float *dlog_alpha,
                                  void *db, void *dw, float *dS0, void *stream);

/*
 * gdr2_sync_status -- wait for `stream`, then report and clear the device
 * status word: GDR2_ERR_TIMEOUT if any kernel of this library gave up a
 * bounded wait since the last call, GDR2_ERR_CUDA on an asynchronous CUDA
 * error, GDR2_OK otherwise.
 */
gdr2_status gdr2_sync_status(void *stream);

/*
 * Test hooks. None has a counterpart in the paper; they exist so that tests
 * can reach code that normal inputs never run, or compare two paths bit for bit.
 *
 * gdr2_debug_force_timeout -- while `enable` is nonzero, the chunk kernel of
 * every tensor-core forward launch (also the one inside gdr2_backward) first
 * waits, with a 1 us limit, on an mbarrier that nothing arrives on, before it
 * issues any copy or MMA. The wait runs out and the kernel takes its normal
 * give-up path: it frees its tensor memory, records the timeout in the device
 * status word and returns. The call's outputs are then undefined, and the next
 * gdr2_sync_status returns GDR2_ERR_TIMEOUT. The setting is process-wide;
 * concurrent callers see it too. 0 (the default) turns it off.
 */
void gdr2_debug_force_timeout(int enable);

/*
 * gdr2_debug_forward_unfused -- while `enable` is nonzero, every dense bf16
 * forward runs as its two kernels (all chunk tasks, then one scan per
 * (sequence, head)) even where it would otherwise run as the fused kernel
 * (chunk tasks and scans in one cooperative launch), and gdr2_backward with
 * saved states runs its chunk tasks and reverse scans as two launches instead
 * of one. Both ways give the same bits; the hook lets a test compare them.
 * Process-wide; 0 (the default) turns it off.
 */
void gdr2_debug_forward_unfused(int enable);

/*
 * gdr2_debug_recip -- y[i] = the device reciprocal the kernels use in place of
 * 1 / x[i] for positive normal x below 2^125 (a bit-pattern seed and two
 * Newton steps, relative error at most 6.6e-6). x and y are device arrays of
 * n floats; asynchronous on `stream`. INVALID_ARG for a NULL pointer or n < 0.
 */
gdr2_status gdr2_debug_recip(const float *x, float *y, long long n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDR2_H */
