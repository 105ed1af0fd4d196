/*
 * kla.h -- C ABI of libkla.so: Kaczmarz Linear Attention (KLA) on NVIDIA B200 (sm_100a).
 *
 * KLA ("Kaczmarz Linear Attention", arXiv 2605.08587) is a gated delta rule whose write
 * is normalised by the key energy.  Per head, with state S in R^{Dk x Dv}:
 *
 *     beta_t = eta_t / (||k_t||^2 + eps)          section 3.1, Eq. (3)
 *     alpha_t = exp(g_t)                           (g is the log-decay)
 *     Sbar = alpha_t S_{t-1};  e_t = v_t - Sbar^T k_t
 *     S_t  = Sbar + beta_t k_t e_t^T               Algorithm 1 (left panel)
 *     o_t  = S_t^T q_t                             section 2 readout
 *
 * The readout uses q exactly as passed.  Algorithm 1's readout divides by ||q_t||; because o
 * is linear in q, a caller who wants that form passes q_t / ||q_t||.  No 1/sqrt(Dk) scale
 * and no key normalisation is applied (normalising k would turn KLA into GDN).
 * When ||k_t||^2 + eps == 0 the write is skipped (beta_t = 0); the paper is silent there.
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers owned by the caller; the library allocates nothing
 *     and keeps no pointer after the call returns.  Buffers must be contiguous in the
 *     layouts given below and 16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream) and never synchronise the host.
 *   - Arguments are validated on the host before any launch; an invalid call returns an
 *     error status and launches nothing.  A failed launch returns KLA_ERR_CUDA.
 *     kla_last_error() gives a one-line description of the last failure on this thread.
 *   - Kernels never wait without a bound: if an internal wait expires the kernel stops,
 *     records it, and kla_check_device_error() reports KLA_ERR_TIMEOUT.
 *   - Supported shapes: Dk, Dv in {64, 128}; chunk == 64; B, H >= 1; T >= 0 (T == 0 copies
 *     S0 to S_T).  The last chunk may be partial.  eps >= 0.  g <= 0 is the intended range
 *     (the decay factors exp(G_i - G_j) are then <= 1); g > 0 is accepted without an
 *     accuracy guarantee.
 *   - dtype selects the element type of the inputs q, k, v (and dO): KLA_F32 or KLA_BF16,
 *     optionally OR-ed with KLA_BETA_DIRECT.  That flag takes the write strength as given,
 *     beta_t = eta_t (the Gated DeltaNet update, or any beta the caller computes), instead of
 *     the Kaczmarz step beta_t = eta_t / (||k_t||^2 + eps); eps is then unused (it must still
 *     be >= 0).  Every entry point taking dtype accepts the flag (the workspace and launch-count
 *     queries ignore it); the backward then differentiates the direct map.
 *     out_dtype selects the element type of the outputs o (and dq, dk, dv): KLA_F32 or
 *     KLA_BF16.  eta, g, S0, S_T, S, dS_T, deta, dg, dS0 are always fp32, as is the state.
 *     Outputs are computed in fp32 and rounded once on store; with heavy-tailed outputs a
 *     bf16 store alone moves the largest elements by 2^-9 of their magnitude.
 *   - NaN or Inf inputs propagate; they are not checked.
 *
 * Layouts (row-major):
 *   q, k, dq, dk : [B, T, H, Dk]          v, o, dO, dv : [B, T, H, Dv]
 *   eta, g, deta, dg : [B, T, H]          S0, S_T, dS_T, dS0 : [B, H, Dk, Dv]
 *   decode: q, k : [B, H, Dk]; v, o : [B, H, Dv]; eta, g : [B, H]; S : [B, H, Dk, Dv]
 */
#ifndef KLA_H_
#define KLA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KLA_OK = 0,
    KLA_ERR_INVALID_ARG = 1, /* null pointer where one is required, negative size, bad eps */
    KLA_ERR_UNSUPPORTED = 2, /* shape or dtype outside the supported set */
    KLA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the *_workspace() size */
    KLA_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
    KLA_ERR_TIMEOUT = 5      /* a bounded device-side wait expired (kla_check_device_error) */
} kla_status;

typedef enum { KLA_F32 = 0, KLA_BF16 = 1 } kla_dtype;

/* OR into a dtype argument: beta_t = eta_t as given (see the conventions above). */
#define KLA_BETA_DIRECT 0x100

/* Static string naming a status code (never NULL). */
const char *kla_status_string(int status);

/* One-line description of the last non-OK status returned on the calling thread. */
const char *kla_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int kla_version(void);

/*
 * kla_chunk_fwd -- chunkwise-parallel prefill.
 * "Kaczmarz Linear Attention", section 4, Propositions 3 and 4 (Eqs. 7-9), Algorithm 1
 * (right panel); the result equals the tokenwise recurrence above for every token.
 *
 *   q, k, v      in   [B,T,H,Dk|Dv] of `dtype`
 *   eta, g       in   [B,T,H] fp32: write gate (0..1 intended) and log-decay
 *   eps          in   stabiliser of Eq. (3), >= 0
 *   S0           in   [B,H,Dk,Dv] fp32 initial state, or NULL for a zero state
 *   o            out  [B,T,H,Dv] of `out_dtype`, or NULL to skip the readout
 *   S_T          out  [B,H,Dk,Dv] fp32 final state, or NULL.  May alias S0.
 *   S_chunks     out  [B,H,ceil(T/chunk),Dk,Dv] fp32 state at the start of every chunk, or
 *                     NULL.  Passing it to kla_chunk_bwd saves the backward's recompute.
 *   ws, ws_bytes      caller workspace (device memory, 32-byte aligned, owned by the caller,
 *                     contents need not be initialised), or NULL.  With at least
 *                     kla_chunk_fwd_workspace() bytes, bf16 inputs with Dk == Dv == 128 run the
 *                     split path: a chunk-parallel kernel stores every chunk's state-independent
 *                     operands there (about 80.5 KiB per chunk and head), then a sequential state
 *                     pass consumes them (segmented, for long sequences over few heads).  With
 *                     NULL or a smaller buffer the forward still runs, as one fused kernel per
 *                     head.  The workspace must not be shared with a concurrent call.
 *                     When the heads are few (at most half the SMs), the split path runs the
 *                     sequence as two slabs of chunks: the second slab's preparation runs on an
 *                     internal stream of the device while the first slab's state pass runs on
 *                     `stream`, which then waits for it before the second state pass (results
 *                     are bit-identical to one run; the call stays ordered on `stream`).
 * Returns KLA_OK or an error status; on error nothing is launched.
 */
size_t kla_chunk_fwd_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
/* Number of kernels one kla_chunk_fwd call launches for these shapes when given at least
 * kla_chunk_fwd_workspace() bytes of workspace (1 for shapes that take none); 0 for invalid
 * shapes. */
int kla_chunk_fwd_kernel_launches(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
kla_status kla_chunk_fwd(const void *q, const void *k, const void *v, const float *eta,
                         const float *g, float eps, const float *S0, void *o, float *S_T,
                         float *S_chunks, int B, int T, int H, int Dk, int Dv, int chunk,
                         int dtype, int out_dtype, void *ws, size_t ws_bytes, void *stream);

/*
 * kla_chunk_fwd_prep, kla_chunk_fwd_state -- the two stages of kla_chunk_fwd's split path, for
 * callers that schedule them separately (for example, preparing the next layer's chunks on
 * another stream, or timing each stage).  Same math as kla_chunk_fwd ("Kaczmarz Linear
 * Attention", section 4, Eqs. 7-9): _prep computes, for every chunk in parallel, everything that
 * does not depend on the incoming state (key norms and Kaczmarz coefficients, decays, the UT
 * transform inverse and W, T Diag(c) for U' = T Diag(c) V, the decayed keys, the masked scores)
 * and stores it in ws; _state then runs the sequential state pass from ws, reading q and v
 * (for U') itself.  Together they equal one kla_chunk_fwd call with that workspace, bit for bit.
 *   Arguments as for kla_chunk_fwd.  Only dtype == KLA_BF16 with Dk == Dv == 128 and T >= 1 is
 *   supported (KLA_ERR_UNSUPPORTED / KLA_ERR_INVALID_ARG otherwise).  ws (device, 32-byte
 *   aligned, at least kla_chunk_fwd_workspace() bytes, owned by the caller) is required
 *   (KLA_ERR_WORKSPACE otherwise); _state must get the same ws, q, v, g and sizes as the _prep
 *   call it follows, ordered after it (same stream, or an event), with ws untouched between.
 * Returns KLA_OK or an error status; on error nothing is launched.
 */
kla_status kla_chunk_fwd_prep(const void *q, const void *k, const void *v, const float *eta,
                              const float *g, float eps, int B, int T, int H, int Dk, int Dv,
                              int chunk, int dtype, void *ws, size_t ws_bytes, void *stream);
kla_status kla_chunk_fwd_state(const void *q, const void *v, const float *g, const float *S0,
                               void *o, float *S_T, float *S_chunks, int B, int T, int H, int Dk,
                               int Dv, int chunk, int dtype, int out_dtype, void *ws,
                               size_t ws_bytes, void *stream);
/*
 * kla_chunk_fwd_state_segments -- how the state pass of the split path runs for these shapes:
 * 1 = one run per head over all its chunks (as one or two slabs inside kla_chunk_fwd), n > 1 =
 * n parallel segments per head chained by a scan ("Kaczmarz Linear Attention", section 4: the
 * chunk-to-chunk state map S -> gamma_last S + Ktil^T (U' - W S) is affine in S, so a segment's
 * map is found from two runs, one from zero and one from the identity, and the segments' start
 * states follow by composing the maps in order).  0 for shapes the split path does not take.
 *
 * kla_chunk_fwd_state_stage -- one part of kla_chunk_fwd_state, for timing or scheduling them
 * apart.  stage 0 is the whole state pass (= kla_chunk_fwd_state).  With segments (above > 1):
 * 1 the transition pass (both runs of every segment, into ws), 2 the segment scan (start
 * states, and S_T, into ws), 3 the output pass (o and S_chunks from every segment's start
 * state); run 1, 2, 3 in order on one stream, with the same arguments, they equal stage 0 bit
 * for bit.  With one run per head stage 3 is the whole pass and 1, 2 launch nothing.
 *   Other arguments, requirements and ownership as for kla_chunk_fwd_state.
 * Returns KLA_OK, KLA_ERR_INVALID_ARG for a stage outside 0..3, or the errors of
 * kla_chunk_fwd_state; on error nothing is launched.
 */
int kla_chunk_fwd_state_segments(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
kla_status kla_chunk_fwd_state_stage(int stage, const void *q, const void *v, const float *g,
                                     const float *S0, void *o, float *S_T, float *S_chunks,
                                     int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                                     int out_dtype, void *ws, size_t ws_bytes, void *stream);

/*
 * kla_chunk_bwd -- gradients of the chunkwise forward.
 * The paper gives no backward; this one differentiates the forward above exactly (same
 * result as reverse-mode differentiation of the tokenwise recurrence).  Given the upstream
 * gradients dO (of o) and dS_T (of S_T, NULL = zero), it returns the gradients of every
 * input: dq, dk, dv (of `out_dtype`), deta, dg ([B,T,H] fp32) and dS0 ([B,H,Dk,Dv] fp32;
 * written even when S0 is NULL).  S_chunks may be the array kla_chunk_fwd wrote for the
 * same inputs, or NULL to recompute it inside the workspace.
 * At a key of exactly zero norm the write vanishes but dk does not: it is returned exactly,
 * dk_t = beta_t Gbar_t v_t with beta_t = eta_t / eps (eta_t in the direct mode; 0 when
 * eps == 0) and Gbar_t the gradient of the state after token t.
 * ws, ws_bytes: caller workspace (device, 32-byte aligned, owned by the caller, contents need
 * not be initialised) of at least kla_chunk_bwd_workspace_min() bytes (required; smaller is
 * KLA_ERR_WORKSPACE).  With at least kla_chunk_bwd_workspace() bytes, bf16 inputs with
 * Dk == Dv == 128 run on the tensor cores: the split forward's preparation and state pass are
 * recomputed into ws (about 290 KiB per chunk and head; S_chunks is then not read), a reverse
 * state pass carries the state gradient chunk by chunk (in parallel segments chained by a scan
 * for long sequences over few heads: kla_chunk_bwd_reverse_segments), and a chunk-parallel
 * kernel forms every gradient.  With less, and for every other shape, the CUDA-core backward runs.
 * The workspace must not be shared with a concurrent call.
 * Every output is fully overwritten.
 */
size_t kla_chunk_bwd_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                               int have_S_chunks);
/* Segments of the tensor-core backward's reverse state pass for these shapes: 1 for one run per
 * head; more when the sequences are long and the heads few (each segment's map of the state
 * gradient in parallel, a scan over segments newest first, then every segment's pass from its
 * true end gradient, as for the forward's segmented state pass); 0 for shapes without the
 * tensor-core backward. */
int kla_chunk_bwd_reverse_segments(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
/* With one reverse run per head (above == 1): how many of the newest chunks the reverse pass
 * takes first as a slab of its own, 0 for one run.  With a slab the gradient kernel of those
 * chunks runs on an internal stream of the device, on the SMs the reverse pass leaves free,
 * while the reverse pass goes on over the older chunks from the gradient it left (the call stays
 * ordered on `stream`).  0 also for shapes without the tensor-core backward. */
int kla_chunk_bwd_reverse_slab_chunks(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
size_t kla_chunk_bwd_workspace_min(int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                                   int have_S_chunks);
kla_status kla_chunk_bwd(const void *q, const void *k, const void *v, const float *eta,
                         const float *g, float eps, const float *S0, const void *dO,
                         const float *dS_T, const float *S_chunks, void *dq, void *dk, void *dv,
                         float *deta, float *dg, float *dS0, int B, int T, int H, int Dk,
                         int Dv, int chunk, int dtype, int out_dtype, void *ws, size_t ws_bytes,
                         void *stream);

/*
 * kla_chunk_fwd_train, kla_chunk_bwd_after_train -- a training step's forward and backward
 * sharing one workspace, so the backward does not recompute the forward.  Same math as
 * kla_chunk_fwd and kla_chunk_bwd ("Kaczmarz Linear Attention", section 4, Eqs. 7-9, and their
 * exact derivative), same results bit for bit.
 *   kla_chunk_fwd_train: arguments as kla_chunk_fwd without S_chunks; writes o and S_T (either
 *     may be NULL) and leaves in ws what the backward needs: for bf16 inputs with
 *     Dk == Dv == 128 and at least kla_chunk_bwd_workspace(..., have_S_chunks = 0) bytes, the
 *     split forward's per-chunk records and every chunk's T, S and U as bf16 tile images;
 *     otherwise (at least kla_chunk_bwd_workspace_min(..., 0) bytes) the chunk states.
 *   kla_chunk_bwd_after_train: arguments as kla_chunk_bwd without S0 and S_chunks; must get the
 *     same q, k, v, eta, g, eps, sizes, dtype, ws and ws_bytes as the kla_chunk_fwd_train call it
 *     follows (ordered after it: same stream, or an event), with ws untouched in between.
 * ws: device memory, 32-byte aligned, owned by the caller, contents need not be initialised;
 * too small is KLA_ERR_WORKSPACE.  Returns KLA_OK or an error status; on error nothing is
 * launched.
 */
kla_status kla_chunk_fwd_train(const void *q, const void *k, const void *v, const float *eta,
                               const float *g, float eps, const float *S0, void *o, float *S_T,
                               int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                               int out_dtype, void *ws, size_t ws_bytes, void *stream);
kla_status kla_chunk_bwd_after_train(const void *q, const void *k, const void *v, const float *eta,
                                     const float *g, float eps, const void *dO, const float *dS_T,
                                     void *dq, void *dk, void *dv, float *deta, float *dg,
                                     float *dS0, int B, int T, int H, int Dk, int Dv, int chunk,
                                     int dtype, int out_dtype, void *ws, size_t ws_bytes,
                                     void *stream);

/*
 * kla_decode_step -- one generated token: Algorithm 1 (left panel), update and readout (readout
 * without the 1/||q|| factor, as above), for every (b, h) at once.
 *
 *   q, k    in     [B,H,Dk] of `dtype`      v   in  [B,H,Dv] of `dtype`
 *   eta, g  in     [B,H] fp32               eps in  >= 0
 *   S       in/out [B,H,Dk,Dv] fp32, updated in place to S_t
 *   o       out    [B,H,Dv] of `out_dtype` (o_t = S_t^T q_t), or NULL
 * Each state element is read once and written once.
 */
kla_status kla_decode_step(const void *q, const void *k, const void *v, const float *eta,
                           const float *g, float eps, float *S, void *o, int B, int H, int Dk,
                           int Dv, int dtype, int out_dtype, void *stream);

/*
 * Diagonal (per-key-channel) gating -- "Kaczmarz Linear Attention", Appendix A.5 (the Kaczmarz
 * step does not depend on how the decayed state was produced) and Appendix B.5 (the chunk form
 * under a diagonal decay).  The decay of token t is Diag(alpha_t), alpha_t = exp(g_t) with one
 * log-decay per key channel:
 *     Sbar = Diag(alpha_t) S_{t-1};  e_t = v_t - Sbar^T k_t;  S_t = Sbar + beta_t k_t e_t^T;
 *     o_t = S_t^T q_t,  beta_t as for kla_chunk_fwd (Kaczmarz step, or KLA_BETA_DIRECT).
 * Arguments, conventions and error behaviour are those of the scalar-gated entry points above,
 * except that g (and dg) are [B, T, H, Dk] fp32 (decode: [B, H, Dk]).  The chunk entry points
 * run on CUDA cores in fp32 (16-token internal chunks, so every decay factor exp(G_i - G_j) is
 * formed directly, channel by channel, and stays <= 1 for g <= 0); the decode step is the
 * TMA-pipelined kernel of kla_decode_step with the per-channel decay folded in.
 *
 * kla_chunk_fwd_diag   -- prefill: o ([B,T,H,Dv] of out_dtype, or NULL) and S_T ([B,H,Dk,Dv]
 *                         fp32, or NULL; may alias S0) from S0 (NULL = zero state).  ws (device,
 *                         32-byte aligned, caller-owned, contents need not be initialised) of at
 *                         least kla_chunk_fwd_diag_workspace() bytes selects the split path: a
 *                         chunk-parallel kernel stores every chunk's state-independent operands
 *                         there, then a sequential state pass reads them.  bf16 with Dk = Dv =
 *                         128 runs both on the tensor cores over 64-token chunks (a 97 KiB
 *                         record per chunk and head, as two slabs or parallel segments like
 *                         kla_chunk_fwd); other shapes run on the CUDA cores over 16-token
 *                         chunks (about 34 KiB per chunk and head at Dk = Dv = 128).  With NULL
 *                         or less, one kernel per (head, 64 value columns) does both on the
 *                         CUDA cores (slower, no workspace).
 *                         The tensor-core preparation forms the chunk's pairwise decay factors
 *                         exp(G_i - G_j) per channel as exp(G_i - R) exp(R - G_j) around the
 *                         channel's mid-range R; a chunk where some channel's prefix G spans
 *                         160 or more takes them exactly, on the CUDA cores (slower).
 * kla_chunk_bwd_diag   -- gradients of <o, dO> + <S_T, dS_T> with respect to q, k, v, eta, g
 *                         (dg per channel, [B,T,H,Dk]) and S0; dS_T may be NULL.  ws: device,
 *                         32-byte aligned, caller-owned, at least kla_chunk_bwd_diag_workspace()
 *                         bytes (the state at every internal chunk start, fp32 accumulators
 *                         cleared by the call, and the split forward's records), else
 *                         KLA_ERR_WORKSPACE.  At a key
 *                         of zero norm dk is exact, as for kla_chunk_bwd.
 * kla_decode_step_diag -- one token for every (b, h); S [B,H,Dk,Dv] updated in place.
 * Returns KLA_OK or an error status; on error nothing is launched.
 */
size_t kla_chunk_fwd_diag_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
/* Kernels one kla_chunk_fwd_diag call launches for these shapes when given at least
 * kla_chunk_fwd_diag_workspace() bytes; 0 for invalid shapes. */
int kla_chunk_fwd_diag_kernel_launches(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
kla_status kla_chunk_fwd_diag(const void *q, const void *k, const void *v, const float *eta,
                              const float *g, float eps, const float *S0, void *o, float *S_T,
                              int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                              int out_dtype, void *ws, size_t ws_bytes, void *stream);
size_t kla_chunk_bwd_diag_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype);
kla_status kla_chunk_bwd_diag(const void *q, const void *k, const void *v, const float *eta,
                              const float *g, float eps, const float *S0, const void *dO,
                              const float *dS_T, void *dq, void *dk, void *dv, float *deta,
                              float *dg, float *dS0, int B, int T, int H, int Dk, int Dv,
                              int chunk, int dtype, int out_dtype, void *ws, size_t ws_bytes,
                              void *stream);
kla_status kla_decode_step_diag(const void *q, const void *k, const void *v, const float *eta,
                                const float *g, float eps, float *S, void *o, int B, int H,
                                int Dk, int Dv, int dtype, int out_dtype, void *stream);

/*
 * kla_gate_prologue -- the per-token inputs of the recurrence computed from the layer's token
 * vectors, for every head at once ("Kaczmarz Linear Attention", section 3.3: the write gate is a
 * sigmoid-activated linear projection of the input token; alpha_t = exp(g_t)):
 *     z_t = W x_t + bias,  eta_t[h] = sigmoid(z_t[h]),  g_t[h] = -softplus(z_t[H + h])
 * and, when q is given, qhat = q / ||q|| per (token, head) (Algorithm 1's readout divides by
 * ||q_t||; o is linear in q, so the recurrence run on qhat gives that readout; a zero query
 * gives qhat = 0).  The pages print no projection for g: the one here is a reading (a linear
 * projection through -softplus, so that g <= 0).
 *   x      in   [N, D] of `dtype` (N = B*T tokens; D % 8 == 0)
 *   W      in   [2H, D] of `dtype`: rows 0..H-1 project eta, rows H..2H-1 project g
 *   bias   in   [2H] fp32
 *   q      in   [N, H, Dk] of `dtype`, or NULL (no normalisation); Dk in {64, 128}
 *   eta, g out  [N, H] fp32
 *   q_hat  out  [N, H, Dk] of `dtype` (NULL exactly when q is NULL)
 * 1 <= H <= 64.  bf16 with D % 64 == 0 and H % 8 == 0 runs the projection on the tensor cores
 * (fp32 accumulation); other shapes and fp32 on CUDA cores.  Returns KLA_OK or an error status;
 * on error nothing is launched.
 *
 * kla_gate_prologue_bwd -- gradients of <eta, deta> + <g, dg> (+ <q_hat, dq_hat>) with respect
 * to x, W, bias (and q), from the prologue's own outputs eta and g for the same x, W, bias:
 *     dz = [deta * eta (1 - eta), dg * expm1(g)],  dx = dz W,  dW = dz^T x,  dbias = sum_t dz,
 *     dq = (dq_hat - q_hat (q_hat . dq_hat)) / ||q||   (zero where q is zero)
 * deta, dg [N, H], dq_hat [N, H, Dk] fp32 in; dx [N, D], dW [2H, D], dbias [2H], dq [N, H, Dk]
 * fp32 out (q, dq_hat and dq all given or all NULL).  ws: device, 32-byte aligned,
 * caller-owned, at least kla_gate_prologue_bwd_workspace() bytes (per-tile partial sums of dW
 * and dbias, added in a fixed order: the result is deterministic).
 */
kla_status kla_gate_prologue(const void *x, const void *W, const float *bias, const void *q, float *eta,
                             float *g, void *q_hat, int N, int D, int H, int Dk, int dtype, void *stream);
size_t kla_gate_prologue_bwd_workspace(int N, int D, int H);
kla_status kla_gate_prologue_bwd(const void *x, const void *W, const float *eta, const float *g,
                                 const void *q, const float *deta, const float *dg, const float *dq_hat,
                                 float *dx, float *dW, float *dbias, float *dq, int N, int D, int H, int Dk,
                                 int dtype, void *ws, size_t ws_bytes, void *stream);

/*
 * kla_check_device_error -- synchronises `stream`, then reads and clears the library's
 * device error word.  Returns KLA_ERR_TIMEOUT if a kernel gave up on a bounded internal
 * wait since the last check (its outputs are then invalid), KLA_ERR_CUDA if the stream
 * reports an error, KLA_OK otherwise.  Not part of the paper: a failure-detection hook.
 */
kla_status kla_check_device_error(void *stream);

/*
 * kla_debug_inject_wait_timeout -- failure injection for tests of the path above.  The next
 * kla_decode_step call (on any thread) launches its kernel so that every CTA's first bounded
 * wait is on a barrier that nothing completes; after about 20 ms that wait expires, the kernel
 * lets the loads it already issued land, stores nothing (S keeps its input values, o is not
 * written) and records the expiry, which kla_check_device_error then reports as
 * KLA_ERR_TIMEOUT.  No copy is cut short and nothing faults: the context stays usable and the
 * following calls run normally.  One-shot; has no effect until called.  Not part of the paper.
 */
void kla_debug_inject_wait_timeout(void);

/*
 * kla_chunk_bwd_noalloc -- kla_chunk_bwd for callers that cannot allocate device memory.
 * The paper has no counterpart; this entry point exists for deployment reasons only.
 *
 * kla_chunk_bwd needs a scratch workspace from the caller.  Some callers cannot allocate
 * one: code recorded into a CUDA graph that must not allocate, plugins whose host framework
 * owns all device memory, or latency-critical paths where cudaMalloc may block or
 * synchronise.  This variant takes no workspace argument and uses a scratch array of
 * KLA_NOALLOC_SCRATCH_BYTES compiled into libkla.so (every GPU that loads the library holds
 * it until the process exits).  It calls no cudaMalloc, cudaFree or allocating routine;
 * inputs and outputs are still the caller's, exactly as for kla_chunk_bwd, and the result is
 * the same.
 *   - Limit: a call is accepted when kla_chunk_bwd_workspace_min() for its sizes is at most
 *     KLA_NOALLOC_SCRATCH_BYTES (about 16K token-heads at Dk = Dv = 128 without S_chunks,
 *     about 32K with it); larger calls are rejected with KLA_ERR_WORKSPACE before anything is
 *     launched.  Which backward runs follows kla_chunk_bwd's rule for a workspace of
 *     KLA_NOALLOC_SCRATCH_BYTES: bf16 inputs with Dk == Dv == 128 run on the tensor cores when
 *     kla_chunk_bwd_workspace() also fits (about 6K token-heads), otherwise the CUDA-core
 *     backward runs (same results within the tolerance, about ten times slower).
 *   - The first call on each device looks up the scratch array's device address (with that
 *     device current) and caches it for the life of the process; make that first call before
 *     any stream capture begins.  The cached address does not survive cudaDeviceReset: do not
 *     call this entry point on a device after resetting it.
 *   - All calls on a device share the one array and the library clears what must start at
 *     zero on every call.  Calls that may overlap on the GPU (different streams, or host
 *     threads without ordering) race on the shared scratch: serialise them.
 */
#define KLA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
size_t kla_chunk_bwd_noalloc_scratch_bytes(void);
kla_status kla_chunk_bwd_noalloc(const void *q, const void *k, const void *v, const float *eta,
                                 const float *g, float eps, const float *S0, const void *dO,
                                 const float *dS_T, const float *S_chunks, void *dq, void *dk,
                                 void *dv, float *deta, float *dg, float *dS0, int B, int T, int H,
                                 int Dk, int Dv, int chunk, int dtype, int out_dtype, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KLA_H_ */
