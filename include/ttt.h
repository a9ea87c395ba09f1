/*
 * ttt.h -- C ABI of the B200 (sm_100a) TTT-KV fast-weight layer library
 *          (libttt_b200.so).
 *
 * The layer: fast weights trained at test time by one gradient step per token
 * (linear case) or per chunk (LaCT case) on the key->value binding loss
 * l_t(W) = -<f_W(k_t), v_t>, read by the queries.
 *
 *   * "Test-Time Training with KV Binding Is Secretly Linear Attention"
 *     (summary page, "B. Reformulación Teórica"): with a linear fast weight
 *     the recurrence W_t = W_{t-1} + eta_t v_t k_t^T, o_t = W_t q_t is causal
 *     linear attention and admits a chunked / prefix-scan form
 *     ("Formulación Paralela").
 *     Its backward pass is ttt_linear_bwd.
 *   * "Test-Time Training Done Right" (LaCT review): a SwiGLU memory with
 *     three matrices, chunk gradients summed with per-token learning rates,
 *     GD / momentum / Muon (Newton-Schulz) updates followed by L2
 *     normalisation ("Memoria no lineal y atención local"); causal chunks read
 *     the memory of earlier chunks before updating it, posed-image sets are
 *     written first and queried afterwards ("El orden de lectura evita
 *     información futura").  The language layer adds causal sliding-window
 *     attention on the same q, k, v (ttt_window_attn_fwd, lact_layer_fwd).
 *
 * General conventions for every entry point
 *   * Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *     library never allocates device memory (lact_chunk_fwd_noalloc uses a
 *     file-scope device array instead of a workspace).  Its other state is a
 *     per-process cache of kernel attributes and, per host thread and
 *     device, helper streams and events created on first use, on which the
 *     independent kernels of a call run beside each other (forked from and
 *     joined back into `stream`).
 *   * Token tensors are [B, H, T, D], contiguous, D innermost.  Learning
 *     rates are float32 [B, H, T].  Pointers must be 16-byte aligned and
 *     D * sizeof(element) a multiple of 16 bytes (TMA rule).
 *   * Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and runs asynchronously.  Arguments are
 *     validated on the host before anything is enqueued; a negative
 *     ttt_status is returned and nothing runs when validation fails.
 *   * Kernels never trap.  Every wait inside a kernel is bounded; when a
 *     bound is exceeded the kernel writes a code into the status word at the
 *     start of the workspace and returns.  ttt_check_device_status() reads it.
 *   * Functions are thread-safe for distinct buffers.
 */
#ifndef TTT_B200_H
#define TTT_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_OK = 0,
  TTT_ERR_ARG = -1,          /* null pointer / bad enum / non-positive size     */
  TTT_ERR_SHAPE = -2,        /* inconsistent or out-of-range shapes            */
  TTT_ERR_ALIGN = -3,        /* pointer or row pitch not 16-byte aligned        */
  TTT_ERR_DTYPE = -4,        /* unsupported dtype combination                  */
  TTT_ERR_UNSUPPORTED = -5,  /* head dims outside the compiled tile set        */
  TTT_ERR_WORKSPACE = -6,    /* workspace too small                            */
  TTT_ERR_CUDA = -7,         /* a CUDA runtime/driver call failed               */
  TTT_ERR_TIMEOUT = -8       /* a bounded in-kernel wait ran out               */
} ttt_status;

typedef enum { TTT_F32 = 0, TTT_BF16 = 1 } ttt_dtype;
typedef enum { TTT_CAUSAL = 0, TTT_BIDIRECTIONAL = 1 } ttt_order;
typedef enum { TTT_OPT_GD = 0, TTT_OPT_MOMENTUM = 1, TTT_OPT_MUON = 2 } ttt_opt;

/* Bytes of the device status word block at the start of every workspace. */
#define TTT_STATUS_BYTES 256

/* ------------------------------------------------------------------------
 * Case (a): linear fast weight == linear attention.
 * "Test-Time Training with KV Binding Is Secretly Linear Attention",
 * summary "B. Reformulación Teórica" and "Formulación Paralela".
 *
 *   state S = W^T, float32 [B, H, dk, dv]
 *   causal:  for t in 0..N-1:  S += lr_t k_t v_t^T ;  out_t = S^T q_t
 *            (include_diag = 0: out_t is read before token t's own update)
 *   bidirectional:  S += sum_t lr_t k_t v_t^T over all N tokens, then
 *            out_t = S^T q_t for every t with that final S.  This is linear
 *            attention with no causal mask, the X A X^T X B form of the
 *            xiaoxiang.io post on the same paper (section "线性注意力视角"),
 *            and the write-then-read order that the "Test-Time Training Done
 *            Right" review gives posed-image sets ("El orden de lectura
 *            evita información futura"); include_diag is ignored.
 *
 * `chunk` is the blocking of the chunked form.  Because the gradient of the
 * binding loss does not depend on W, the result is the same for every chunk
 * size up to rounding; the tensor-core kernel processes 128-token tiles.
 * ---------------------------------------------------------------------- */
typedef struct {
  int B, H, N;          /* batch, heads, tokens (N >= 0)                     */
  int dk, dv;           /* key/query dim, value dim                          */
  int chunk;            /* > 0                                               */
  ttt_order order;      /* TTT_CAUSAL or TTT_BIDIRECTIONAL                   */
  int include_diag;     /* causal: 1 = token reads after its own update     */
  ttt_dtype in_dtype;   /* q, k, v element type (TTT_F32 or TTT_BF16)        */
  ttt_dtype out_dtype;  /* out element type                                  */
} ttt_linear_desc;

/* Workspace bytes for ttt_linear_fwd at full speed (same summary,
 * "Formulación Paralela": the state after a token is S0 plus the sum of the
 * updates before it, a prefix scan).  The status block, plus, on the
 * tensor-core path (bf16, dk = dv = 64), room for partial state sums:
 *   causal: the start states of the sequence segments that run on separate
 *     SMs (a pre-pass sums each segment's updates);
 *   bidirectional: the per-unit sums of the whole-sequence state pass.
 * The size depends on the device's SM count.  A workspace of only
 * TTT_STATUS_BYTES is accepted: a causal call then runs each head unsplit,
 * a bidirectional one runs on CUDA cores.  Errors: TTT_ERR_ARG (null
 * pointers), the shape and dtype errors of ttt_linear_fwd. */
int ttt_linear_workspace_bytes(const ttt_linear_desc* desc, size_t* bytes);

/* The state before the first token (same summary, "B. Reformulación
 * Teórica": the fast weight the recurrence starts from, W0 = S0^T).
 * S <- S0 (device float32 [B,H,dk,dv], caller-owned); S0 == NULL zero-fills
 * S.  Enqueued on `stream`; TTT_ERR_CUDA if the copy cannot be enqueued. */
int ttt_linear_state_init(const ttt_linear_desc* desc, const float* S0, float* S, void* stream);

/* Readout of the fast weight after a call (same summary: the state the next
 * call of a streamed sequence continues from).  dst <- S, float32
 * [B,H,dk,dv]; dst may be a device pointer or pinned/registered host memory.
 * Enqueued on `stream`; TTT_ERR_CUDA if the copy cannot be enqueued. */
int ttt_linear_state_readout(const ttt_linear_desc* desc, const float* S, float* dst, void* stream);

/* One call over N tokens.  q, k: [B,H,N,dk]; v: [B,H,N,dv]; lr: [B,H,N];
 * S: in = state before the first token, out = state after the last token;
 * out: [B,H,N,dv].  Supported: in_dtype F32 (any dk, dv <= 128) and BF16
 * (dk = dv = 64 on tensor cores; other dims <= 128 on CUDA cores), in
 * either order.  A bidirectional call on tensor cores first sums the whole
 * sequence's updates into S, then reads every query with that S.
 * ws (>= TTT_STATUS_BYTES, device, caller-owned) holds the status block and
 * the segment states (see ttt_linear_workspace_bytes); it must not be shared
 * by calls that overlap in time. */
int ttt_linear_fwd(const ttt_linear_desc* desc, const void* q, const void* k, const void* v,
                   const float* lr, float* S, void* out, void* ws, size_t ws_bytes, void* stream);

/* Backward pass of ttt_linear_fwd: the gradients of
 *   L = sum_t <dout_t, out_t> + <dS_end, S_end>
 * with respect to q, k, v, lr and the start state S0, for training through
 * the layer ("Test-Time Training with KV Binding Is Secretly Linear
 * Attention", summary "Resultados Experimentales": the training-time result).
 * With R_s = dS_end + sum of q_t dout_t^T over the reads t that see token s,
 *   dq_t = S_t dout_t,  dk_s = lr_s R_s v_s,  dv_s = lr_s R_s^T k_s,
 *   dlr_s = k_s^T R_s v_s,  dS0 = dS_end + sum_t q_t dout_t^T,
 * where S_t is the state token t read (desc->include_diag as in the forward
 * call).  Each is computed as a forward-time causal scan with the roles of
 * q, k, v and dout exchanged, on the kernels of ttt_linear_fwd.  Causal order
 * only: a bidirectional desc returns TTT_ERR_UNSUPPORTED.
 * Inputs (device): q, k [B,H,N,dk], v [B,H,N,dv], lr [B,H,N] as given to the
 * forward call; S0 [B,H,dk,dv] float32, the forward call's start state (NULL =
 * zeros); dout [B,H,N,dv] in desc->in_dtype; dS_end [B,H,dk,dv] float32 (NULL =
 * zeros).  Outputs (device, float32, written in full): dq, dk [B,H,N,dk],
 * dv [B,H,N,dv], dlr [B,H,N], dS0 [B,H,dk,dv]; desc->out_dtype is not used.
 * ws: device workspace of at least ttt_linear_bwd_workspace_bytes, status
 * block first; it must not be shared by calls that overlap in time.
 * Errors as ttt_linear_fwd; nothing is enqueued when validation fails. */
int ttt_linear_bwd_workspace_bytes(const ttt_linear_desc* desc, size_t* bytes);
int ttt_linear_bwd(const ttt_linear_desc* desc, const void* q, const void* k, const void* v,
                   const float* lr, const float* S0, const void* dout, const float* dS_end,
                   float* dq, float* dk, float* dv, float* dlr, float* dS0, void* ws,
                   size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Case (b): LaCT, SwiGLU fast-weight memory with large chunks.
 * "Test-Time Training Done Right" review, "Memoria no lineal y atención
 * local" and "El orden de lectura evita información futura".
 *
 * Per (b,h): W1, W3 in R^{dh x d}, W2 in R^{d x dh};
 *   f_W(x) = W2 (silu(W1 x) * (W3 x)),  l_t = -<f_W(k_t), v_t>.
 * For each chunk of `chunk` input tokens (the last may be shorter):
 *   causal:        out = f_W(q) for the chunk's tokens with the weights left
 *                  by earlier chunks, then update;
 *   bidirectional: update only; after the last chunk the N_q queries read.
 * Update: G = sum_t lr_t grad_W l_t (all at the chunk-start W), then
 *   GD:       W -= G
 *   MOMENTUM: M = beta M + G;  W -= M
 *   MUON:     M = beta M + G;  W -= NS(M)  (ns_steps quintic Newton-Schulz
 *             steps with ns_coef on M/(||M||_F + ns_eps), wide orientation)
 * then, if normalize_rows, every row of each updated matrix is rescaled to
 * unit L2 norm: W[i,:] /= max(||W[i,:]||, norm_eps).
 * update_mask selects the updated matrices: bit0 W1, bit1 W3, bit2 W2.
 * ---------------------------------------------------------------------- */
typedef struct {
  int B, H;
  int N_in;             /* input (key/value) tokens                          */
  int N_q;              /* query tokens; must equal N_in when causal         */
  int d, dh;            /* head dim (multiple of 64), hidden dim (mult. 64)  */
  int chunk;            /* > 0                                               */
  ttt_order order;
  ttt_opt opt;
  float beta;           /* momentum (MOMENTUM, MUON)                         */
  int ns_steps;         /* Newton-Schulz steps (MUON), >= 0                  */
  float ns_coef[3];     /* (a, b, c) of a*X + (b*A + c*A^2) X                */
  float ns_eps;
  int normalize_rows;
  float norm_eps;
  int update_mask;      /* 1..7                                              */
  ttt_dtype in_dtype;   /* q, k, v: TTT_BF16                                 */
  ttt_dtype out_dtype;  /* out: TTT_F32 or TTT_BF16                          */
  int split_operands;   /* 0: bf16 tensor-core operands; 1: every weight,
                           gradient intermediate and Newton-Schulz operand is
                           carried as bf16 hi + lo (x = hi + lo), which keeps
                           ~16 significant bits at 2-3x the MMA work.  Needed
                           by MUON, whose update amplifies operand rounding */
} lact_desc;

/* Bytes of the state: W1, W3, W2 float32 per (b,h) (+ M1, M3, M2 for
 * MOMENTUM and MUON).  Layout: [W1 | W3 | W2 | M1 | M3 | M2], each block
 * [B*H, rows, cols] row-major. */
int lact_state_bytes(const lact_desc* desc, size_t* bytes);

/* Workspace bytes for lact_chunk_fwd (status word, bf16 operand copies of
 * the weights, per-chunk intermediates, split-K partial sums, NS buffers):
 * the size at which the call takes its fastest form. */
int lact_workspace_bytes(const lact_desc* desc, size_t* bytes);

/* The smallest workspace lact_chunk_fwd accepts.  It equals
 * lact_workspace_bytes except for the W2-only layer of "Test-Time Training
 * with KV Binding Is Secretly Linear Attention", summary "Resultados
 * Experimentales" (component ablation) and "Formulación Paralela" (causal, GD,
 * update_mask = 4, normalize_rows = 0, no split operands, d and dh
 * multiples of 128, chunk a multiple of 128 dividing N_in): that layer is
 * block-causal linear attention on silu(W1 x) * (W3 x) and runs in parallel
 * over chunks when the workspace holds every chunk's features and W2
 * increment (lact_workspace_bytes); with less, down to this size, it runs the
 * chunk loop.  Both give the same result up to rounding. */
int lact_workspace_bytes_min(const lact_desc* desc, size_t* bytes);

/* Initialise the state from float32 device weights.  w_per_batch = 0: W1,
 * W3 are [H,dh,d] and W2 [H,d,dh], shared by every batch entry; 1: they are
 * [B,H,...].  Momentum buffers are zeroed. */
int lact_state_init(const lact_desc* desc, const float* W1, const float* W3, const float* W2,
                    int w_per_batch, void* state, void* stream);

/* Copy the state out: W1, W3 [B,H,dh,d], W2 [B,H,d,dh]; M (nullable) gets
 * [M1 | M3 | M2] when the optimizer keeps momentum.  Destinations may be
 * device pointers or pinned host memory. */
int lact_state_readout(const lact_desc* desc, const void* state, float* W1, float* W3, float* W2,
                       float* M, void* stream);

/* One call of the layer.  q: causal [B,H,N_in,d], bidirectional [B,H,N_q,d];
 * k, v: [B,H,N_in,d]; lr: [B,H,N_in]; state in/out; out: [B,H,N_in,d]
 * (causal) or [B,H,N_q,d] (bidirectional).  A causal call may be followed by
 * another call on the continuation of the sequence with the same state;
 * chunk boundaries restart at every call.  A causal call with d = 128, GD
 * or momentum and no split operands runs every chunk in one cooperative
 * launch that takes every SM of the device (its CTAs wait on one another
 * through counters in the workspace, each wait bounded); the environment
 * variable TTT_LACT_CHUNK_LOOP=0, read once per process, keeps one launch
 * per chunk.  Both give the same result (bit for bit when every chunk is
 * full). */
int lact_chunk_fwd(const lact_desc* desc, const void* q, const void* k, const void* v,
                   const float* lr, void* state, void* out, void* ws, size_t ws_bytes,
                   void* stream);

/* ------------------------------------------------------------------------
 * Context parallelism: the tokens of one chunk split across devices.
 * "Test-Time Training Done Right" review, "Vídeo y cálculo distribuido":
 * every device computes the gradient of its share of a chunk's tokens, the
 * shares are summed across devices, and every device applies the same
 * update to its copy of the weights.  These three calls are the per-device
 * pieces of lact_chunk_fwd; the sum between them is the caller's collective
 * (an all-reduce into each device's own G).  Per chunk of a causal call:
 *   lact_read (the chunk's queries, current weights), lact_chunk_grad (this
 *   device's tokens of the chunk), all-reduce of G, lact_apply_grad;
 * a bidirectional call does the last three per chunk and lact_read of the
 * queries at the end.  desc, state and ws are as for lact_chunk_fwd (ws of
 * at least lact_workspace_bytes_min); the calls keep no state of their own.
 * ---------------------------------------------------------------------- */

/* Bytes of a chunk gradient G: [G1 | G3 | G2], each [B,H,rows,cols] float32,
 * laid out like the weights of the state. */
int lact_grad_bytes(const lact_desc* desc, size_t* bytes);

/* G <- sum over tokens t in [t0, t0 + n) of lr_t times the gradient of
 * -<f_W(k_t), v_t> at the state's current weights (no update; G is
 * overwritten).  k, v: [B,H,N_in,d]; lr: [B,H,N_in]; n <= desc->chunk
 * (a share of one chunk), t0 + n <= N_in, else TTT_ERR_SHAPE.  n = 0 writes
 * zeros. */
int lact_chunk_grad(const lact_desc* desc, int t0, int n, const void* k, const void* v,
                    const float* lr, const void* state, float* G, void* ws, size_t ws_bytes,
                    void* stream);

/* The update of one chunk with the (summed) chunk gradient G: GD / momentum /
 * Muon as in lact_chunk_fwd, then the row normalisation, on `state`. */
int lact_apply_grad(const lact_desc* desc, const float* G, void* state, void* ws,
                    size_t ws_bytes, void* stream);

/* out rows [t0, t0 + n) <- f_W(q rows [t0, t0 + n)) with the state's current
 * weights ("El orden de lectura evita información futura": a causal chunk
 * reads the weights left by earlier chunks, queries of a posed-image set read
 * the final ones).  q, out: [B,H,R,d] with R = N_in (causal) or N_q
 * (bidirectional); n at most one chunk (causal) or N_q, else TTT_ERR_SHAPE. */
int lact_read(const lact_desc* desc, int t0, int n, const void* q, const void* state, void* out,
              void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Backward pass of lact_chunk_fwd, for training through the layer ("Test-Time
 * Training Done Right" review, "Lenguaje: calidad y velocidad no son
 * equivalentes": the layer's training throughput with GD, momentum and Muon
 * updates).  The gradients of
 *   L = sum <dout, out> + sum_m <dW_end[m], W_m after the call>
 * with respect to q, k, v, lr and the weights at the start of the call,
 * through every chunk's update (chunk gradients at the chunk-start weights,
 * optimizer step, row normalisation) and every read.  GD and MOMENTUM (the
 * momentum buffers start at zero, as after lact_state_init); MUON returns
 * TTT_ERR_UNSUPPORTED.  The call replays the forward chunk loop to keep each
 * chunk's start weights, then walks the chunks in reverse.
 * state0: the state the forward call started from (its W1, W3, W2 are read);
 * dout: [B,H,R,d] bf16 with R = N_in (causal) or N_q (bidirectional);
 * dW_end: nullable [dW1 | dW3 | dW2] float32 in the state's weight layout.
 * Outputs, float32, written in full: dq [B,H,R,d], dk, dv [B,H,N_in,d],
 * dlr [B,H,N_in], dW0 [dW1 | dW3 | dW2] (the state's weight layout).
 * ws: device workspace of at least lact_bwd_workspace_bytes, status block
 * first. */
int lact_bwd_workspace_bytes(const lact_desc* desc, size_t* bytes);
int lact_chunk_bwd(const lact_desc* desc, const void* q, const void* k, const void* v,
                   const float* lr, const void* state0, const void* dout, const float* dW_end,
                   float* dq, float* dk, float* dv, float* dlr, float* dW0, void* ws,
                   size_t ws_bytes, void* stream);

/* Same computation as lact_chunk_fwd for callers that cannot allocate device
 * memory (code hosted by a program that owns all device allocations and
 * hands it only its tensors; paths where cudaMalloc/cudaFree and their
 * possible device synchronisation are not allowed).  The pages have no
 * counterpart: this is a deployment variant, not part of the method.
 * The workspace is a file-scope device array of 64 MiB held by every GPU
 * that loads the library until exit; problems needing more (see
 * lact_workspace_bytes_min) return TTT_ERR_WORKSPACE and nothing runs.  The
 * first call on a device looks up the array's address with that device
 * current (make that first call before any stream capture); a
 * cudaDeviceReset of the device invalidates it, so do not call the entry
 * point after one.  `stream` must belong to the current device
 * (TTT_ERR_ARG otherwise).  All calls share the array: each call clears its
 * status block on `stream`; calls whose GPU work overlaps race and must not
 * be issued.  Read the status block with lact_noalloc_check_status. */
int lact_chunk_fwd_noalloc(const lact_desc* desc, const void* q, const void* k, const void* v,
                           const float* lr, void* state, void* out, void* stream);

/* ttt_check_device_status for the scratch array of lact_chunk_fwd_noalloc
 * on the current device: synchronises `stream` (which must belong to the
 * current device), then reads and clears the status block of the last call.
 * Returns TTT_OK, TTT_ERR_TIMEOUT (a bounded wait of that call ran out),
 * TTT_ERR_ARG (stream of another device) or TTT_ERR_CUDA.  Like the entry
 * point it serves, it has no counterpart in the pages. */
int lact_noalloc_check_status(void* stream);

/* ------------------------------------------------------------------------
 * Local branch of the LaCT language layer: causal sliding-window attention.
 * "Test-Time Training Done Right" review, "Memoria no lineal y atención
 * local", "El orden de lectura evita información futura" and "Lenguaje"
 * (window 2048 for the 760M model, 4096 for the 3B one):
 *
 *   o_i = sum over j in (i - window, i] of softmax_j(scale q_i . k_j) v_j
 *
 * The window counts the token itself; scale <= 0 selects 1 / sqrt(d).
 * ---------------------------------------------------------------------- */
typedef struct {
  int B, H, N;          /* N >= 0                                            */
  int d;                /* head dim of q, k and v: 128                       */
  int window;           /* >= 1                                              */
  float scale;
  ttt_dtype in_dtype;   /* TTT_BF16                                          */
  ttt_dtype out_dtype;  /* TTT_F32 or TTT_BF16                               */
  int accumulate;       /* 0: out = attention; 1: out += attention           */
} ttt_window_desc;

/* q, k, v: device [B,H,N,d] bf16; out: device [B,H,N,d] in out_dtype (read
 * as well when accumulate = 1).  ws: at least TTT_STATUS_BYTES (status
 * block).  Tensor cores (tcgen05), one CTA per 128-query tile. */
int ttt_window_attn_fwd(const ttt_window_desc* desc, const void* q, const void* k, const void* v,
                        void* out, void* ws, size_t ws_bytes, void* stream);

/* The LaCT language layer in causal order: the fast-weight memory of
 * lact_chunk_fwd and the sliding-window attention above on the same q, k, v,
 * outputs summed into out (the window branch adds its output in its
 * epilogue).  desc as for lact_chunk_fwd (causal, d = 128); window and scale
 * as in ttt_window_desc; ws as for lact_chunk_fwd. */
int lact_layer_fwd(const lact_desc* desc, int window, float scale, const void* q, const void* k,
                   const void* v, const float* lr, void* state, void* out, void* ws,
                   size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Status and diagnostics
 * ---------------------------------------------------------------------- */

/* Synchronises `stream`, then reads and clears the status word of `ws`.
 * Returns TTT_OK, TTT_ERR_TIMEOUT (a bounded wait ran out) or TTT_ERR_CUDA. */
int ttt_check_device_status(void* ws, void* stream);

/* Launch a one-CTA kernel that waits, with a bound of `timeout_us`
 * microseconds, on an mbarrier that nothing ever completes; it must record
 * TTT_ERR_TIMEOUT in the status word of `ws` and return.  Exercises the
 * failure path of every bounded wait without faulting the GPU. */
int ttt_selftest_wait_timeout(void* ws, size_t ws_bytes, int timeout_us, void* stream);

/* Optional per-kernel timing.  Between ttt_profile_begin() and
 * ttt_profile_end() every kernel launch of this library is bracketed by two
 * CUDA events recorded on its launch stream.  ttt_profile_end() waits for
 * them and returns, per kernel kind, the number of launches and the summed
 * event time; `entries` (nullable) receives up to `max_entries` of them and
 * `*n_entries` the number of kinds seen.  Process-wide; not for concurrent
 * use from several threads. */
typedef struct {
  char name[32];
  int launches;
  double total_ms;
} ttt_prof_entry;
int ttt_profile_begin(void);
int ttt_profile_end(ttt_prof_entry* entries, int max_entries, int* n_entries);

/* Human-readable name of a ttt_status value. */
const char* ttt_status_string(int status);

/* Library build string (compiler, arch). */
const char* ttt_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_B200_H */
