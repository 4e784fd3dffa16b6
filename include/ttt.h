/*
 * ttt.h -- C ABI of the B200 (sm_100a) TTT forward-scan library (libttt_b200.so).
 *
 * The library computes the causal forward scan of a Test-Time-Training layer
 * ("Learning to (Learn at Test Time): RNNs with Expressive Hidden States").
 * Every (batch, head) pair carries a hidden state that is itself a model f
 * with weights W.  Over the sequence, in mini-batches of b tokens, the scan
 * takes gradient steps on the reconstruction loss
 *     l(W; t) = || f(K_t; W) - V_t ||^2            (sum of squares)
 * with a per-token learning rate eta_t, and emits z_t = f(Q_t; W_t).
 *   - State, update rule and output rule: literature record of the paper
 *     (dmarx.github.io lit-801), Key takeaways, bullet 1.
 *   - Inner loss and the token-dependent learning rate: same record, bullet 2.
 *   - Mini-batch updates (b = 16) and LayerNorm + residual inside f: bullet 5.
 *   - Theorem 1 (linear f, batch GD, eta = 1/2, W0 = 0 is causal linear
 *     attention): bullet 3.  TTT_PLAIN mode is that linear f.
 *   - TTT-Linear and TTT-MLP hidden states: the paper's abstract
 *     (codewithpapers.app record).
 *
 * Mini-batch rule: inside a mini-batch every token's gradient is taken at the
 * state the mini-batch started from; the state used for the output of token t
 * subtracts eta_s * grad_s for every token s <= t of the mini-batch (t
 * included).  At the end of the mini-batch that state becomes the next start
 * state.  If b does not divide T, the last mini-batch holds T mod b tokens.
 *
 * Inner models (row vectors, W stored [in][out] row-major):
 *   TTT_LN_RESIDUAL  f(x) = x + LN(x W + b)
 *   TTT_PLAIN        f(x) = x W              (no bias, no LN, no residual)
 *   TTT-MLP          f(x) = x + LN(GELU(x W1 + b1) W2 + b2)
 * LN(y) = gamma * (y - mean(y)) / sqrt(var(y) + eps) + beta over the d features
 * of one token, biased variance.  gamma and beta are fixed; the scan updates
 * W and b (W1, b1, W2, b2 for the MLP).  GELU is the tanh form
 * 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
 *
 * Conventions shared by every entry point
 *   Memory      All data pointers are DEVICE pointers on the current CUDA
 *               device, owned by the caller.  The library allocates no memory
 *               and keeps no state between calls.
 *   Layout      Q, K, V, Z: [B][H][T][d] contiguous.  eta: [B][H][T] fp32.
 *               Per-(batch, head) state: W [B][H][d_in][d_out] fp32, b [B][H][d_out].
 *               gamma, beta: [H][d] fp32, shared by all batch rows.
 *   Types       Q, K, V are bf16 (TTT_BF16) or fp32 (TTT_F32); everything else
 *               is fp32, and the state is carried in fp32.  Z is fp32.
 *   Alignment   Every pointer must be 16-byte aligned (TTT_ERR_ALIGN).
 *   Aliasing    W_T may be the same pointer as W0 (and b_T as b0) for an
 *               in-place state update; any other overlap between an output
 *               (Z, W_T, b_T) and any other buffer is TTT_ERR_ALIAS.
 *   Shapes      B, H >= 1; T >= 0; mini_batch >= 1 and either a multiple of
 *               16 or one of 1, 2, 4, 8.  T = 0 copies the state; the token
 *               buffers (Q, K, V, eta, Z) are then empty and may be NULL.
 *   Stream      Work is enqueued on `stream` (0 = legacy default stream); the
 *               call does not synchronise.
 *   Errors      Argument errors are detected on the host before anything is
 *               launched, and return without side effects.  A launch failure
 *               returns TTT_ERR_CUDA (from cudaPeekAtLastError).  With the
 *               environment variable TTT_CHECK=1 the call synchronises the
 *               stream after the launch and returns TTT_ERR_CUDA on an
 *               asynchronous error, or TTT_ERR_TIMEOUT if a kernel abandoned a
 *               bounded wait (its outputs are then undefined).  The kernels
 *               record an abandoned wait in an error word per process, not
 *               per call: a checked call clears it before its launch, so its
 *               status covers that call alone, but checked calls that overlap
 *               on several streams may see each other's timeouts.  Both
 *               environment variables are read once per process.
 *   Fault injection  TTT_DEBUG_DROP_CHUNK=<c> (a test hook, read once per
 *               process) makes the tensor-core TTT-Linear kernels skip the
 *               loads of chunk c, so their bounded waits give up.  While it is
 *               set every call runs as if TTT_CHECK=1 and such a call returns
 *               TTT_ERR_TIMEOUT; leave it unset in normal use.
 *   Threads     Entry points are re-entrant.
 *   Continuation  Feeding W_T (b_T) back as W0 (b0) continues the sequence
 *               when the split falls on a mini-batch boundary (bit for bit in
 *               the generic family; the tensor-core family reaches the first
 *               chunk after a split by an algebraically equal route, so the
 *               results agree up to rounding).
 */
#ifndef TTT_B200_TTT_H
#define TTT_B200_TTT_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t. */
typedef struct CUstream_st* ttt_stream_t;

typedef enum {
    TTT_OK = 0,
    TTT_ERR_NULL = 1,        /* a required pointer is NULL                         */
    TTT_ERR_SHAPE = 2,       /* B, H, T, mini_batch out of range                   */
    TTT_ERR_DTYPE = 3,       /* unknown ttt_dtype                                  */
    TTT_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned                   */
    TTT_ERR_ALIAS = 5,       /* an output overlaps an input other than as allowed  */
    TTT_ERR_UNSUPPORTED = 6, /* d, hidden, mode or implementation not built       */
    TTT_ERR_CUDA = 7,        /* CUDA launch or execution error                     */
    TTT_ERR_TIMEOUT = 8,     /* a kernel gave up a bounded wait (TTT_CHECK=1 only) */
    TTT_ERR_WORKSPACE = 9    /* workspace NULL or smaller than its size query returns */
} ttt_status;

typedef enum { TTT_BF16 = 0, TTT_F32 = 1 } ttt_dtype;

typedef enum { TTT_LN_RESIDUAL = 0, TTT_PLAIN = 1 } ttt_mode;

/* Kernel family.  TTT_IMPL_AUTO picks the fastest one built for the shape. */
typedef enum {
    TTT_IMPL_AUTO = 0,
    TTT_IMPL_GENERIC = 1,    /* fp32 SIMT scan: every supported shape, dtype and mode */
    TTT_IMPL_TENSORCORE = 2, /* tensor-core scan: bf16 Q/K/V, b = 16, T a multiple of 16;
                                TTT-Linear d = 64 in LN mode, TTT-MLP d = 64, hidden = 256 */
    TTT_IMPL_TENSORCORE_SPLIT = 3, /* TTT-MLP only, same shapes as TTT_IMPL_TENSORCORE: each
                                      scan's hidden units split over the two CTAs of a
                                      cluster (two SMs per scan) */
    TTT_IMPL_TCGEN05 = 4, /* TTT-Linear only, same shapes as TTT_IMPL_TENSORCORE: the products
                            with the state run on the 5th-generation tensor cores (tcgen05,
                            fp32 accumulators in tensor memory, one issuing thread), the
                            sequential per-chunk chain on warp-level mma; the state is kept
                            centred on its per-row means, which are added back to W_T, b_T */
} ttt_impl;

/*
 * TTT-Linear forward scan.
 *   d          head dimension: 16, 32 or 64 (TTT_ERR_UNSUPPORTED otherwise)
 *   mini_batch b of the mini-batch rule above
 *   qkv_dtype  element type of Q, K, V
 *   mode       TTT_LN_RESIDUAL or TTT_PLAIN
 *   ln_eps     LayerNorm epsilon (> 0 in LN mode)
 *   Q, K, V    [B][H][T][d]
 *   eta        [B][H][T] per-token inner learning rate
 *   W0, b0     initial state [B][H][d][d], [B][H][d]; b0 may be NULL in TTT_PLAIN
 *   ln_gamma, ln_beta  [H][d]; may be NULL in TTT_PLAIN
 *   Z          [B][H][T][d] fp32 output z_t
 *   W_T, b_T   final state (same shapes as W0, b0); b_T may be NULL in TTT_PLAIN
 */
ttt_status ttt_linear_forward(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                              ttt_mode mode, float ln_eps, const void* Q, const void* K,
                              const void* V, const float* eta, const float* W0,
                              const float* b0, const float* ln_gamma, const float* ln_beta,
                              float* Z, float* W_T, float* b_T, ttt_stream_t stream);

/* As ttt_linear_forward, with an explicit kernel family (TTT_ERR_UNSUPPORTED if
 * that family does not cover the arguments). */
ttt_status ttt_linear_forward_impl(int B, int H, int T, int d, int mini_batch,
                                   ttt_dtype qkv_dtype, ttt_mode mode, float ln_eps,
                                   const void* Q, const void* K, const void* V,
                                   const float* eta, const float* W0, const float* b0,
                                   const float* ln_gamma, const float* ln_beta, float* Z,
                                   float* W_T, float* b_T, ttt_impl impl, ttt_stream_t stream);

/* Kernel family TTT_IMPL_AUTO would run for these arguments (TTT_IMPL_AUTO if
 * no family covers them).  Pure host query; launches nothing. */
ttt_impl ttt_linear_pick_impl(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                              ttt_mode mode);

/*
 * TTT-Linear decode: the scan of ttt_linear_forward continued by T >= 0 more
 * tokens, the first of them at position pos0 of its mini-batch
 * (0 <= pos0 < mini_batch, else TTT_ERR_SHAPE).  T = 1 is single-token decode;
 * T need not fill or end a mini-batch.  The caller keeps the position:
 * the next call's pos0 is (pos0 + T) % mini_batch.
 *   W, b       running state W_t, b_t [B][H][d][d], [B][H][d]: read, then
 *              overwritten with the state after the call's last token
 *   W_mb, b_mb state the current mini-batch started from, at which its
 *              gradients are taken: read when pos0 > 0, then overwritten with
 *              the start state of the mini-batch the next token falls in
 *              (equal to W, b when the call ends on a mini-batch boundary)
 *   b, b_mb, ln_gamma, ln_beta may be NULL in TTT_PLAIN.  The four state
 *   buffers, Z and the inputs must not overlap (TTT_ERR_ALIAS).  Other
 *   arguments as ttt_linear_forward.  d = 64 runs a decode kernel that keeps
 *   the state in registers for the whole call (token-serial, fp32); d = 16 and
 *   32 run the generic fp32 family.  Results equal a ttt_linear_forward over
 *   the whole stream up to rounding.
 */
ttt_status ttt_linear_decode(int B, int H, int T, int d, int mini_batch, int pos0,
                             ttt_dtype qkv_dtype, ttt_mode mode, float ln_eps, const void* Q,
                             const void* K, const void* V, const float* eta, float* W, float* b,
                             float* W_mb, float* b_mb, const float* ln_gamma,
                             const float* ln_beta, float* Z, ttt_stream_t stream);

/*
 * TTT-MLP forward scan, f(x) = x + LN(GELU(x W1 + b1) W2 + b2).
 *   d = 64 and hidden = 256 are built (TTT_ERR_UNSUPPORTED otherwise).
 *   W1_0 [B][H][d][hidden], b1_0 [B][H][hidden], W2_0 [B][H][hidden][d], b2_0 [B][H][d]
 *   W1_T, b1_T, W2_T, b2_T: final state, same shapes; each may be the same
 *   pointer as its initial-state counterpart.  When mini_batch > 16, W1_T and
 *   W2_T also hold the mini-batch start state while the scan runs.
 */
ttt_status ttt_mlp_forward(int B, int H, int T, int d, int hidden, int mini_batch,
                           ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K,
                           const void* V, const float* eta, const float* W1_0,
                           const float* b1_0, const float* W2_0, const float* b2_0,
                           const float* ln_gamma, const float* ln_beta, float* Z, float* W1_T,
                           float* b1_T, float* W2_T, float* b2_T, ttt_stream_t stream);

/* As ttt_mlp_forward, with an explicit kernel family (TTT_ERR_UNSUPPORTED if
 * that family does not cover the arguments).  The tensor-core families keep the
 * state in shared memory in fp32 and run every product on the tensor cores
 * (bf16 hi/lo operands, fp32 accumulation); their results agree with the
 * generic family's, and with each other's, up to rounding. */
ttt_status ttt_mlp_forward_impl(int B, int H, int T, int d, int hidden, int mini_batch,
                                ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K,
                                const void* V, const float* eta, const float* W1_0,
                                const float* b1_0, const float* W2_0, const float* b2_0,
                                const float* ln_gamma, const float* ln_beta, float* Z,
                                float* W1_T, float* b1_T, float* W2_T, float* b2_T, ttt_impl impl,
                                ttt_stream_t stream);

/*
 * TTT-MLP decode: the scan of ttt_mlp_forward continued by T >= 0 more tokens,
 * the first at position pos0 of its mini-batch (0 <= pos0 < mini_batch, else
 * TTT_ERR_SHAPE), as ttt_linear_decode for the linear model.
 *   W1, b1, W2, b2          running state (shapes of ttt_mlp_forward's W1_0 ...),
 *                           read, then overwritten with the state after the
 *                           call's last token
 *   W1_mb, b1_mb, W2_mb, b2_mb  state the current mini-batch started from: read
 *                           when pos0 > 0, then overwritten with the start state
 *                           of the mini-batch the next token falls in
 * The eight state buffers, Z and the inputs must not overlap (TTT_ERR_ALIAS).
 * Runs a decode kernel that keeps the running state in registers for the
 * whole call (token-serial, fp32).
 */
ttt_status ttt_mlp_decode(int B, int H, int T, int d, int hidden, int mini_batch, int pos0,
                          ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K,
                          const void* V, const float* eta, float* W1, float* b1, float* W2,
                          float* b2, float* W1_mb, float* b1_mb, float* W2_mb, float* b2_mb,
                          const float* ln_gamma, const float* ln_beta, float* Z,
                          ttt_stream_t stream);

/* As ttt_mlp_decode with an explicit family: TTT_IMPL_AUTO (the decode kernel)
 * or TTT_IMPL_GENERIC (the generic fp32 scan run from inside a mini-batch);
 * TTT_ERR_UNSUPPORTED for any other. */
ttt_status ttt_mlp_decode_impl(int B, int H, int T, int d, int hidden, int mini_batch, int pos0,
                               ttt_dtype qkv_dtype, float ln_eps, const void* Q, const void* K,
                               const void* V, const float* eta, float* W1, float* b1, float* W2,
                               float* b2, float* W1_mb, float* b1_mb, float* W2_mb, float* b2_mb,
                               const float* ln_gamma, const float* ln_beta, float* Z, ttt_impl impl,
                               ttt_stream_t stream);

/* Kernel family TTT_IMPL_AUTO would run for these TTT-MLP arguments
 * (TTT_IMPL_AUTO if no family covers them).  Pure host query.  Among the
 * tensor-core families it picks TTT_IMPL_TENSORCORE_SPLIT while the doubled
 * grid, 2 B H CTAs of one SM each, fits in one wave (B H <= 74), else
 * TTT_IMPL_TENSORCORE. */
ttt_impl ttt_mlp_pick_impl(int B, int H, int T, int d, int hidden, int mini_batch,
                           ttt_dtype qkv_dtype);

/*
 * The layer's prologue: the scan's inputs from the layer input x, in one kernel
 * (literature record, Key takeaways bullets 1 and 2: the scan sees the views
 * theta_K x_t, theta_V x_t, theta_Q x_t of each token and a learning rate that
 * depends on the token; the codewithpapers.app record names the official
 * code's rotate_half helper).  Per head h and token t (readings of the pages,
 * which give no formulas):
 *   Q = x theta_q[h], K = x theta_k[h], V = x theta_v[h]        (no bias)
 *   eta = eta_base * sigmoid(x . theta_lr[h] + b_lr[h]) / d
 *   rotary (when rotary != 0), on Q and K: features i and i + d/2 rotate
 *   together by the angle p * rope_base^(-2 i / d), p = pos0 + t the token's
 *   absolute position.
 *   x         [B][T][d_model] bf16
 *   theta_q, theta_k, theta_v  [H][d_model][d] bf16;  theta_lr [H][d_model] bf16
 *   b_lr      [H] fp32
 *   Q, K, V   [B][H][T][d] bf16 outputs (the layout ttt_linear_forward reads),
 *             rounded to nearest from the fp32 accumulation
 *   eta       [B][H][T] fp32 output
 * Built for d = 64, d_model a multiple of 64, H a multiple of 4 up to 256
 * (TTT_ERR_UNSUPPORTED otherwise); T >= 1.  Runs on the tcgen05 tensor cores
 * (bf16 products, fp32 accumulation).  Outputs may not overlap the inputs or
 * each other (TTT_ERR_ALIAS).  Other conventions as ttt_linear_forward.
 */
ttt_status ttt_prologue_forward(int B, int T, int H, int d, int d_model, int pos0, float eta_base,
                                float rope_base, int rotary, const void* x, const void* theta_q,
                                const void* theta_k, const void* theta_v, const void* theta_lr,
                                const float* b_lr, void* Q, void* K, void* V, float* eta,
                                ttt_stream_t stream);

/*
 * TTT-Linear layer backward: the gradients an outer training loop needs
 * (literature record, Key takeaways bullet 2: the outer loop trains the views
 * theta_K, theta_V, theta_Q, the initial weights and the learning rate).
 * Given the forward arguments of ttt_linear_forward and the upstream gradient
 * dZ of its output (and, optionally, dW_T, db_T of its final state), returns
 * the gradients of   sum(Z * dZ) + sum(W_T * dW_T) + sum(b_T * db_T)
 * with respect to every forward input:
 *   dQ, dK, dV   [B][H][T][d] fp32 (whatever qkv_dtype is)
 *   deta         [B][H][T]
 *   dW0, db0     [B][H][d][d], [B][H][d]
 *   dgamma, dbeta [H][d], summed over the batch in a fixed order
 *   dW_T, db_T   may be NULL (zero)
 * Built for TTT_LN_RESIDUAL, d = 16, 32 or 64, mini_batch 1, 2, 4, 8 or 16,
 * any T (TTT_ERR_UNSUPPORTED otherwise; TTT_PLAIN is not built).
 * workspace    caller-owned device scratch of at least
 *              ttt_linear_backward_workspace_size(B, H, T, d, mini_batch)
 *              bytes (16-byte aligned), else TTT_ERR_WORKSPACE.  The call
 *              first runs the forward scan and records there the state every
 *              mini-batch starts from (d*d + d floats per mini-batch and
 *              head), then sweeps the mini-batches in reverse, recomputing
 *              each one's intermediates from its recorded state.  Its contents
 *              are undefined afterwards; calls that may overlap need separate
 *              workspaces.
 * Outputs may not overlap each other, the inputs or the workspace
 * (TTT_ERR_ALIAS).  Other conventions as ttt_linear_forward.
 */
size_t ttt_linear_backward_workspace_size(int B, int H, int T, int d, int mini_batch);

ttt_status ttt_linear_backward(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                               ttt_mode mode, float ln_eps, const void* Q, const void* K,
                               const void* V, const float* eta, const float* W0, const float* b0,
                               const float* ln_gamma, const float* ln_beta, const float* dZ,
                               const float* dW_T, const float* db_T, float* dQ, float* dK, float* dV,
                               float* deta, float* dW0, float* db0, float* dgamma, float* dbeta,
                               void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * ttt_linear_backward without a workspace argument, for callers that cannot
 * allocate device memory: for example a host program whose own allocator owns
 * all device memory and grants a library nothing at call time, or a loop with a
 * latency budget that an allocation (and the synchronisation it may bring)
 * would break.  The pages define no such call; it exists only for this reason.
 *   The workspace is a fixed array inside the library,
 *   TTT_BACKWARD_STATIC_WORKSPACE_BYTES (32 MiB) long, which every GPU that
 *   loads the library holds until the process exits.  Arguments whose
 *   ttt_linear_backward_workspace_size exceeds it return TTT_ERR_WORKSPACE
 *   before anything runs (for d = 64 it holds about 2000 mini-batch states,
 *   summed over batch and heads).
 *   The call allocates nothing: no cudaMalloc, no library allocator.  The
 *   first call on a device looks up the array's device address (one
 *   cudaGetSymbolAddress with that device current) and keeps it; make that
 *   first call before any stream capture.
 *   Every call on a device shares the one array, and the array keeps the last
 *   call's contents; the kernels write every word of it they later read, so
 *   nothing needs to start at zero.  Calls that may overlap on the GPU (on
 *   several streams, or from several host threads) race on it: run them one
 *   after another.
 *   Arguments, outputs and errors otherwise as ttt_linear_backward.
 */
#define TTT_BACKWARD_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)

ttt_status ttt_linear_backward_static(int B, int H, int T, int d, int mini_batch, ttt_dtype qkv_dtype,
                                      ttt_mode mode, float ln_eps, const void* Q, const void* K,
                                      const void* V, const float* eta, const float* W0, const float* b0,
                                      const float* ln_gamma, const float* ln_beta, const float* dZ,
                                      const float* dW_T, const float* db_T, float* dQ, float* dK,
                                      float* dV, float* deta, float* dW0, float* db0, float* dgamma,
                                      float* dbeta, ttt_stream_t stream);

/* Static string naming a status code; never NULL. */
const char* ttt_status_string(ttt_status status);

/* ABI version of the library (major * 100 + minor). */
int ttt_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_B200_TTT_H */
