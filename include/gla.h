/*
 * gla.h -- C ABI of libgla, the B200 (sm_100a) Simple Gated Linear Attention
 * mixer library.
 *
 * The mixer (page "AWS serve Laplace 3B di i14 con uno stato fisso di 29,5 MB",
 * section "GLA sostituisce i token conservati con uno stato ricorrente": every
 * layer replaces softmax attention with Simple GLA, which updates a
 * fixed-size matrix state per token) computes, per (batch, head), with a
 * scalar log-decay a_t <= 0 per token and head:
 *
 *     S_t = exp(a_t) * S_{t-1} + k_t^T v_t         S: dk x dv, fp32
 *     o_t = scale * q_t S_t                         scale: normally dk^-1/2
 *
 * Shapes follow page "Como i14 llevo Laplace 3B a AWS Trainium2", section
 * "Diseno esencial de Laplace 3B": H = 16 heads, dk = 96, dv = 192.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is DEVICE memory owned by the caller.  libgla never
 *     allocates, never frees and never synchronises (except the two status
 *     readers at the end of this file, which say so).
 *   - Every call is asynchronous on the caller's stream and returns a
 *     gla_status.  Argument errors are detected on the host before anything
 *     is launched; in that case nothing is written.
 *   - Layout is token-major: [B, T, H, d] with d innermost and contiguous.
 *     Base pointers must be 16-byte aligned (GLA_ERR_MISALIGNED otherwise).
 *   - No exception crosses this ABI.
 *   - Preconditions not checked on the device: a_t <= 0 and finite; inputs
 *     finite.
 *   - Device-side waits (on TMA / tensor-core completion barriers) are
 *     bounded.  A wait that runs out records GLA_ERR_TIMEOUT in a device status
 *     word, the kernel releases what it holds and returns; read the word with
 *     gla_get_device_status().
 */
#ifndef GLA_H
#define GLA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gla_status {
    GLA_OK = 0,
    GLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, workspace too small */
    GLA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. dk != 96)    */
    GLA_ERR_MISALIGNED = 3,    /* pointer or stride not 16-byte aligned        */
    GLA_ERR_CUDA = 4,          /* a CUDA call failed; see gla_last_cuda_error  */
    GLA_ERR_TIMEOUT = 5        /* a bounded device-side wait ran out           */
} gla_status;

typedef enum gla_dtype {
    GLA_BF16 = 0,              /* bf16 q/k/v/o/dO; fp32 state and decay        */
    GLA_F32 = 1                /* fp32 everywhere (forward only)               */
} gla_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* gla_status_string(gla_status s);

/* cudaError_t of the last failed CUDA call made by libgla on this host thread
 * (0 when none). */
int gla_last_cuda_error(void);

/* Number of kernel launches libgla has issued from this process (all
 * threads), for launch accounting by callers. */
unsigned long long gla_launch_count(void);

/* How this copy of the library was built: a bit mask of GLA_BUILD_* flags.
 * GLA_BUILD_DEBUG_BOUNDS marks the checking build (libgla_debug.so, compiled
 * with -DGLA_DEBUG_BOUNDS).  It has the same ABI and results as the normal
 * build and additionally, without ever trapping:
 *   - scans the inputs of every chunk, segment and decode call before its
 *     kernels run: a_t <= 0 and finite, q/k/v/dO and fp32 states finite;
 *   - checks the index of each direct global store in its kernels against
 *     the tensor it writes, and skips a store that would fall outside;
 * and records GLA_ERR_INVALID_ARG in the device status word on a violation
 * (read it with gla_get_device_status).  The scans cost one extra read of
 * the inputs per call. */
#define GLA_BUILD_DEBUG_BOUNDS 1
int gla_build_flags(void);

/* ---------------------------------------------------------------------------
 * Chunked prefill / training forward.
 *
 * The chunked form ("Como i14 ...", section "Adaptaciones para AWS
 * Trainium2", item 1: T = 2048 processed as 16 chunks of 128 tokens) is an
 * exact reorganisation of the recurrence above.  Chunk size is 128.
 *
 *   q, k    [B, T, H, dk]  dt       token stride ld_qkv elements (0 = packed:
 *   v       [B, T, H, dv]  dt       H*dk for q and k, H*dv for v); head stride
 *                                   dk (q, k) or dv (v); batch stride T*ld.
 *                                   ld_qkv lets q/k/v be views into one fused
 *                                   projection buffer (e.g. 9216 per token).
 *   a       [B, T, H]      fp32     log-decay, contiguous.
 *   s0      [B, H, dk, dv] fp32     initial state; NULL means zeros.
 *   o       [B, T, H, dv]  dt       output, contiguous.
 *   s_final [B, H, dk, dv] fp32     final state S_T; NULL to skip.
 *   ws      workspace of ws_bytes >= gla_chunk_workspace_bytes(B,T,H,dk,dv,0)
 *           (may be NULL when that size is 0).  Its contents on entry do not
 *           matter and are undefined on return.  (for_bwd: 0 forward, 1
 *           gla_chunk_bwd, 2 gla_chunk_bwd_saved.)
 *   scale   multiplies q once (normally dk^-1/2); must be > 0 and finite.
 *   dt      GLA_BF16 (tensor-core path: fp32 accumulation, fp32 state) or
 *           GLA_F32 (fp32 CUDA-core path, for small problems).
 * Supported: dk == 96, dv == 192, B, H >= 1, T >= 1 (any T; the last chunk may
 * be partial).  ld_qkv must be a multiple of 8 and >= the packed stride.
 * ------------------------------------------------------------------------ */
size_t gla_chunk_workspace_bytes(int B, int T, int H, int dk, int dv, int for_bwd);

gla_status gla_chunk_fwd(const void* q, const void* k, const void* v, const float* a,
                         const float* s0, void* o, float* s_final, void* ws, size_t ws_bytes,
                         int B, int T, int H, int dk, int dv, int64_t ld_qkv, float scale,
                         gla_dtype dt, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Training pair: a forward that also keeps what the backward needs, and the
 * backward that reads it instead of recomputing it.  The backward needs the
 * state entering every chunk (the states of the recurrence at the chunk
 * boundaries, "Como i14 ...", section "Adaptaciones para AWS Trainium2",
 * item 1); the forward computes them anyway, so it can write them out.
 *
 * gla_chunk_fwd_train: gla_chunk_fwd (same arguments and results) that also
 * writes the state entering each chunk c of every (b, h) into `saved`:
 *   saved   [B, H, NC, 2, dk, dv] bf16, NC = ceil(T / 128): plane 0 holds
 *           bf16(S), plane 1 bf16(S - plane 0), together within 2^-17 of the
 *           fp32 state; saved_bytes >= gla_chunk_saved_state_bytes(B,T,H,dk,dv).
 * gla_chunk_bwd_saved: gla_chunk_bwd given those states (and, when ds_final is
 * given, the forward's s_final, which the dS_T term of da needs) in place of
 * s0; it skips the backward's own state-recompute pass.  Its workspace is
 * gla_chunk_workspace_bytes(B,T,H,dk,dv, 2) (smaller than the plain
 * backward's: no state planes of its own).  Results equal gla_chunk_bwd's.
 * Both: dt must be GLA_BF16; other arguments, layouts and status codes as
 * gla_chunk_fwd / gla_chunk_bwd.
 * ------------------------------------------------------------------------ */
size_t gla_chunk_saved_state_bytes(int B, int T, int H, int dk, int dv);

gla_status gla_chunk_fwd_train(const void* q, const void* k, const void* v, const float* a,
                               const float* s0, void* o, float* s_final, void* saved, size_t saved_bytes,
                               void* ws, size_t ws_bytes, int B, int T, int H, int dk, int dv,
                               int64_t ld_qkv, float scale, gla_dtype dt, cudaStream_t stream);

gla_status gla_chunk_bwd_saved(const void* q, const void* k, const void* v, const float* a,
                               const void* saved, size_t saved_bytes, const float* s_final,
                               const void* dO, const float* ds_final, void* grad_q, void* grad_k,
                               void* grad_v, float* grad_a, float* grad_s0, void* ws, size_t ws_bytes,
                               int B, int T, int H, int dk, int dv, int64_t ld_qkv, float scale,
                               gla_dtype dt, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Chunked forward over a packed batch of sequences of different lengths
 * (prefill of several requests at once): gla_chunk_fwd for each sequence n,
 * whose tokens are rows cu_seqlens[n] .. cu_seqlens[n+1]-1 of q, k, v, a and
 * o, each sequence with its own initial and final state.  The chunk grid
 * restarts at every sequence; tokens of one sequence never enter another's
 * state or output.
 *   q, k        [total_T, H, 96], v [total_T, H, 192] bf16, token stride
 *               ld_qkv as in gla_chunk_fwd (0 = packed).
 *   a           [total_T, H] fp32.    o [total_T, H, 192] bf16.
 *   cu_seqlens  DEVICE pointer, [N+1] int32, non-decreasing, cu_seqlens[0] >= 0,
 *               cu_seqlens[N] <= total_T.  A sequence whose offsets fall
 *               outside 0 .. total_T is skipped and GLA_ERR_INVALID_ARG is
 *               recorded in the device status word (gla_get_device_status).
 *   s0, s_final [N, H, 96, 192] fp32 or NULL (zeros / not wanted).
 *   ws          workspace of ws_bytes >= gla_chunk_varlen_workspace_bytes(N,
 *               total_T, H, dk, dv), or NULL.  With it, sequences longer than a
 *               segment (about total_T H / (148 x 128) chunks, so that the
 *               segments of all sequences make about one wave of CTAs) are cut
 *               into segments that run in parallel (state-only pre-pass, fp32
 *               fold, output pass), so one long sequence no longer sets the
 *               time; a small kernel reads the lengths on the device and
 *               splits only when the longest sequence spans at least two
 *               segments.  Without it (or when the size is 0) each
 *               (sequence, head) is one sweep.  Contents on entry do not
 *               matter.  When cu_seqlens is invalid and a workspace is given,
 *               the outputs of the valid sequences are undefined as well.
 * Rows of o outside every sequence are not written.  dt must be GLA_BF16;
 * N <= 65535.
 * ------------------------------------------------------------------------ */
size_t gla_chunk_varlen_workspace_bytes(int N, int total_T, int H, int dk, int dv);

gla_status gla_chunk_fwd_varlen(const void* q, const void* k, const void* v, const float* a,
                                const int32_t* cu_seqlens, int N, const float* s0, void* o,
                                float* s_final, void* ws, size_t ws_bytes, int total_T, int H, int dk,
                                int dv, int64_t ld_qkv, float scale, gla_dtype dt, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * gla_chunk_fwd for callers that cannot allocate device memory.  (The pages
 * have no counterpart to this call; it exists for library users.)
 *
 * Some callers cannot obtain a workspace: a runtime that keeps all device
 * memory in its own pool and forbids side allocations, a plugin host that
 * does not let extensions call cudaMalloc, or a path that cannot afford the
 * device synchronisation that cudaMalloc/cudaFree imply.  This call takes
 * the arguments of gla_chunk_fwd without ws/ws_bytes and uses a fixed
 * scratch array inside libgla instead; it allocates nothing.
 *   - The array is GLA_NOALLOC_SCRATCH_BYTES per GPU that loads the library,
 *     held until the process exits, and shared by every call on that GPU.
 *   - Shapes whose workspace (gla_chunk_workspace_bytes) is larger are
 *     rejected with GLA_ERR_UNSUPPORTED before anything is launched; use
 *     gla_chunk_fwd with a workspace for those.
 *   - Calls that overlap on the GPU (e.g. on two streams at once) race on the
 *     shared array; order them.  The array's leftover contents never matter.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress) with that device current, and so does the first
 *     call after the device's current context has changed (cudaDeviceReset,
 *     another context); make those calls before any stream capture starts.
 * Everything else (layouts, validation, status codes) is as gla_chunk_fwd.
 * ------------------------------------------------------------------------ */
#define GLA_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

gla_status gla_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* a,
                                 const float* s0, void* o, float* s_final, int B, int T, int H,
                                 int dk, int dv, int64_t ld_qkv, float scale, gla_dtype dt,
                                 cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Chunked backward (the sequential chunk backward of "Como i14 ...", section
 * "Adaptaciones para AWS Trainium2", item 3).  Same inputs as the forward plus
 *   dO       [B, T, H, dv]  dt     upstream gradient of o, contiguous.
 *   ds_final [B, H, dk, dv] fp32   upstream gradient of S_T; NULL means zero.
 * Outputs (contiguous):
 *   grad_q, grad_k [B, T, H, dk] dt;  grad_v [B, T, H, dv] dt;
 *   grad_a [B, T, H] fp32;  grad_s0 [B, H, dk, dv] fp32 (NULL to skip).
 * grad_q is the gradient with respect to the unscaled q that was passed in.
 * ws_bytes >= gla_chunk_workspace_bytes(B,T,H,dk,dv,1).  dt must be GLA_BF16.
 * ------------------------------------------------------------------------ */
gla_status gla_chunk_bwd(const void* q, const void* k, const void* v, const float* a,
                         const float* s0, const void* dO, const float* ds_final,
                         void* grad_q, void* grad_k, void* grad_v, float* grad_a,
                         float* grad_s0, void* ws, size_t ws_bytes, int B, int T, int H, int dk,
                         int dv, int64_t ld_qkv, float scale, gla_dtype dt, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Sequence split across ranks (long documents, "Como i14 ...", section "Por
 * qué atención lineal importa": cost linear in T with a fixed-size state).
 * A sequence cut into R consecutive segments, one per rank, is exact in
 * three steps, because the state is linear in its inputs (section
 * "Adaptaciones para AWS Trainium2", item 1: chunking only regroups the
 * recurrence):
 *   1. each rank: gla_segment_state_fwd on its own tokens -> (L_r, G_r), and
 *      for the backward also gla_segment_state_bwd -> D_r;
 *   2. exchange (an all_gather of those B*H*(dk*dv + 1) floats per rank);
 *   3. each rank: gla_state_fold to get the state entering its segment
 *      (entries 0 .. r-1, in order, from S_0) and, for the backward, the
 *      state gradient at its end (entries r+1 .. R-1, right to left, from
 *      dS_T); then gla_chunk_fwd / gla_chunk_bwd on its tokens with those
 *      as s0 / ds_final.
 *
 * gla_segment_state_fwd: for every (b, h) of a segment of T tokens,
 *     s_seg = sum_t exp(A_{T-1} - A_t) k_t^T v_t   (the end state from zero)
 *     g_seg = A_{T-1} = sum_t a_t                  (natural log)
 *   k [B,T,H,dk], v [B,T,H,dv] bf16 with token stride ld_qkv as in
 *   gla_chunk_fwd; a [B,T,H] fp32; s_seg [B,H,dk,dv] fp32 (required);
 *   g_seg [B,H] fp32 (NULL to skip).
 * gla_segment_state_bwd: with zero state gradient at the segment's end,
 *     ds_seg = dL/dS entering the segment
 *            = sum_t scale exp(A_t) q_t^T dO_t     (A_t inclusive of a_t)
 *   q [B,T,H,dk] bf16 (token stride ld_qkv); dO [B,T,H,dv] bf16 contiguous;
 *   ds_seg [B,H,dk,dv] fp32 (required); g_seg as above.
 * Both: dt must be GLA_BF16; ws_bytes >= gla_segment_workspace_bytes(B,T,H,
 * dk,dv) (a scratch of per-sub-segment states; contents do not matter).
 * T == 0 gives zeros.
 *
 * gla_state_fold: out = x after x <- exp(g[j]) x + s[j] for j = 0 .. n-1
 * (j = n-1 .. 0 when reverse != 0), starting from x = s_in (zeros if NULL).
 *   s [n][units][dk][dv] fp32, g [n][units] fp32 (natural log), s_in and
 *   out [units][dk][dv] fp32; out may be s_in.  n == 0 copies s_in (or
 *   zeros) to out.  units = B*H.
 * All pointers are device memory, 16-byte aligned except g (4 bytes, so
 * that g may start at any entry of a gathered array); every call is
 * asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
size_t gla_segment_workspace_bytes(int B, int T, int H, int dk, int dv);

gla_status gla_segment_state_fwd(const void* k, const void* v, const float* a, float* s_seg,
                                 float* g_seg, void* ws, size_t ws_bytes, int B, int T, int H,
                                 int dk, int dv, int64_t ld_qkv, gla_dtype dt, cudaStream_t stream);

gla_status gla_segment_state_bwd(const void* q, const void* dO, const float* a, float* ds_seg,
                                 float* g_seg, void* ws, size_t ws_bytes, int B, int T, int H,
                                 int dk, int dv, int64_t ld_qkv, float scale, gla_dtype dt,
                                 cudaStream_t stream);

gla_status gla_state_fold(const float* s, const float* g, int n, int reverse, const float* s_in,
                          float* out, int units, int dk, int dv, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * One decode step for N sequences (the fixed per-sequence state of "AWS serve
 * Laplace 3B ...", section "Lo stato di Laplace 3B resta fisso durante
 * l'inferenza"; 1,280 concurrent sequences in "Como i14 ...", section
 * "Resultados de entrenamiento e inferencia").  For every (n, h):
 *     S <- exp(a[n,h]) * S + k[n,h]^T v[n,h]     (in place, fp32)
 *     o[n,h] = scale * q[n,h] S                   (the updated S)
 *   state    [n_slots, H, dk, dv] fp32, updated in place.
 *   slot_idx [N] int32: state slot of sequence n (NULL = identity).  Slots
 *            must be distinct within one call.  A slot outside
 *            [0, n_slots) is skipped (its state is not touched and o[n] is
 *            not written) and GLA_ERR_INVALID_ARG is recorded in the device
 *            status word (gla_get_device_status).
 *   n_slots  number of slots in state; >= N when slot_idx is NULL.
 *   q, k     [N, H, dk] bf16;  v [N, H, dv] bf16;  a [N, H] fp32 (contiguous).
 *   o        [N, H, dv] fp32.
 * Supported: dk == 96, dv == 192.
 * ------------------------------------------------------------------------ */
gla_status gla_decode_step(float* state, const int32_t* slot_idx, int n_slots, const void* q, const void* k,
                           const void* v, const float* a, float* o, int N, int H, int dk, int dv,
                           float scale, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Front end of each layer ("Como i14 ...", section "Diseno esencial de
 * Laplace 3B": the residual vector goes through LayerNorm, then a causal
 * depthwise Conv1d of width 4 with SiLU, a 4-gram summary before the mixer):
 *     xn[t]   = LayerNorm(x[t]) over D   (biased variance, eps inside the root,
 *                                          then * gamma + beta) if apply_ln,
 *               else x[t]
 *     y[t,c]  = SiLU( sum_{j<W} w[c,j] * xn[t-(W-1)+j, c] + bias[c] )
 * Positions before t = 0 come from conv_state_in (zeros when NULL).
 *   x, y            [B, T, D] bf16, contiguous.
 *   ln_gamma/beta   [D] fp32, NULL = 1 / 0.
 *   w               [D, W] fp32 (w[c, W-1] multiplies the current token).
 *   bias            [D] fp32 or NULL.
 *   conv_state_in   [B, W-1, D] fp32 or NULL: the last W-1 conv inputs (xn)
 *                   before t = 0, oldest first.
 *   conv_state_out  [B, W-1, D] fp32 or NULL: the last W-1 conv inputs of
 *                   this call, for the next call.  Must not alias
 *                   conv_state_in.
 * Supported: W == 4, D % 8 == 0, 8 <= D <= 4096.
 * ------------------------------------------------------------------------ */
gla_status conv1d_silu_causal(const void* x, int apply_ln, const float* ln_gamma,
                              const float* ln_beta, float ln_eps, const float* w,
                              const float* bias, const float* conv_state_in,
                              float* conv_state_out, void* y, int B, int T, int D, int W,
                              cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Backward of conv1d_silu_causal, for training the mixer block: given dy,
 * the gradient of a loss with respect to y, compute the gradients of x, of
 * the conv weights and bias, of the LayerNorm affine and of conv_state_in.
 * The forward is recomputed from x (nothing is saved between the calls);
 * conv_state_out carries no gradient back.  With u the conv output before
 * SiLU, s = sigmoid(u), xhat the normalised rows:
 *     du      = dy * s * (1 + u (1 - s))
 *     dxn[p]  = sum_j w[c,j] * du[p+W-1-j]            (rows p < 0: dconv_state_in)
 *     dx      = rstd * (g - mean(g) - xhat * mean(g * xhat)),  g = dxn * gamma
 *               (dx = dxn without LayerNorm)
 *     dw[c,j] = sum_{b,t} du[t,c] * xn[t-(W-1)+j, c]     dbias = sum du
 *     dln_gamma = sum dxn * xhat                           dln_beta = sum dxn
 *   x, dy, dx       [B, T, D] bf16.   dw [D, W] fp32 (required).
 *   dbias, dln_gamma, dln_beta [D] fp32, dconv_state_in [B, W-1, D] fp32:
 *                   each NULL = not wanted.  Every output is overwritten.
 *   ws              ws_bytes >= conv1d_silu_causal_bwd_workspace_bytes(B,T,D,W)
 *                   (per-CTA partial sums, added in a fixed order: results do
 *                   not depend on scheduling).
 * Other arguments as in conv1d_silu_causal.  Supported: W == 4, D % 8 == 0,
 * 8 <= D <= 4096, B <= 65535.
 * ------------------------------------------------------------------------ */
size_t conv1d_silu_causal_bwd_workspace_bytes(int B, int T, int D, int W);
gla_status conv1d_silu_causal_bwd(const void* x, int apply_ln, const float* ln_gamma,
                                  const float* ln_beta, float ln_eps, const float* w,
                                  const float* bias, const float* conv_state_in, const void* dy,
                                  void* dx, float* dw, float* dbias, float* dln_gamma,
                                  float* dln_beta, float* dconv_state_in, void* ws,
                                  size_t ws_bytes, int B, int T, int D, int W,
                                  cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Front end at decode time: conv1d_silu_causal at T = 1 for N sequences
 * whose conv histories live in a pool of slots, updated in place -- the way
 * gla_decode_step addresses the recurrent states (the serving wrapper links
 * the state to the serving memory pool: "AWS serve Laplace 3B ...", section
 * "Lo stato di Laplace 3B resta fisso durante l'inferenza").  For sequence n
 * with slot s = slot_idx[n] (n when NULL):
 *     xn       = LayerNorm(x[n]) as in conv1d_silu_causal if apply_ln, else x[n]
 *     y[n,c]   = SiLU( sum_{j<W-1} w[c,j] * h[s,j,c] + w[c,W-1] * xn[c] + bias[c] )
 *     h[s]    <- (h[s,1], ..., h[s,W-2], xn)        (in place)
 *   x, y        [N, D] bf16, contiguous.
 *   conv_state  [n_slots, W-1, D] fp32: h, the last W-1 conv inputs of each
 *               slot, oldest first (the layout of conv1d_silu_causal's
 *               conv_state_in / _out for one sequence), updated in place.
 *   slot_idx    [N] int32 or NULL (identity).  Slots must be distinct within
 *               one call.  A slot outside [0, n_slots) is skipped (nothing
 *               read or written for that sequence) and GLA_ERR_INVALID_ARG is
 *               recorded in the device status word.
 *   n_slots     number of slots in conv_state; >= N when slot_idx is NULL.
 *   ln_gamma/beta, w, bias as in conv1d_silu_causal.
 * Supported: W == 4, D % 8 == 0, 8 <= D <= 4096.
 * ------------------------------------------------------------------------ */
gla_status conv1d_silu_decode_step(const void* x, const int32_t* slot_idx, int n_slots, int apply_ln,
                                   const float* ln_gamma, const float* ln_beta, float ln_eps,
                                   const float* w, const float* bias, float* conv_state, void* y,
                                   int N, int D, int W, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Device status.  gla_get_device_status SYNCHRONISES the stream, copies the
 * device status word of the current device (0 or a gla_status recorded by a
 * kernel, e.g. GLA_ERR_TIMEOUT) into *device_status and clears it.
 * gla_set_wait_limit_ns sets the bound on every device-side wait of later
 * launches (default 2e9 ns; 0 restores the default).
 * gla_selftest_wait_timeout launches one kernel whose only wait is on a
 * barrier that nothing completes, so the bound runs out by design and the
 * kernel returns having recorded GLA_ERR_TIMEOUT; it lets callers check the
 * failure path without faulting or hanging the GPU.
 * ------------------------------------------------------------------------ */
gla_status gla_get_device_status(cudaStream_t stream, int* device_status);

/* ---------------------------------------------------------------------------
 * Kernel tracing.  While enabled, libgla brackets every kernel it launches
 * with two CUDA events recorded on the launch stream (events come from a
 * pool owned by libgla; no device memory is allocated).  gla_trace_enable(1)
 * clears earlier records; gla_trace_enable(0) stops recording.
 * gla_trace_summary SYNCHRONISES on the recorded events and reports, per
 * kernel name (at most max_entries, in first-launch order): the name (a
 * static string), the number of launches and their summed device time in
 * milliseconds.  It returns the number of entries written.
 * ------------------------------------------------------------------------ */
gla_status gla_trace_enable(int enable);
int gla_trace_summary(const char** names, unsigned long long* launches, double* total_ms,
                      int max_entries);
gla_status gla_set_wait_limit_ns(unsigned long long ns);
gla_status gla_selftest_wait_timeout(cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* GLA_H */
