/*
 * swimba.h -- C ABI of libswimba.so: the Swimba (Switch Mamba) layer on B200 (sm_100a).
 *
 * The layer (sources: "Swimba: Switch Mamba Model Scales State Space Models", technical summaries
 * §2 "Metodología / Arquitectura de Swimba" (es), "Methodologie / Kernmechanisme van Swimba" (nl),
 * "Méthodologie / Architecture de Swimba" (fr); and "Mamba y las SSMs: el retorno del estado
 * persistente", sections "SSMs", "Mamba" (Figura 2) and "Estado interno puramente lineal"):
 *
 *   route       logits_t = x_t W_r; idx_t = top-k (descending, ties to the lower index);
 *               gates_t  = softmax over the k selected logits.
 *   mixed_proj  per selected expert e: [dt_low | B^e | C^e] = x_t W_x^e, dt^e = dt_low W_dt^e + b_dt^e;
 *               mixed in parameter space with the gates: dt_mix = sum_j g_j dt^{e_j},
 *               B_mix = sum_j g_j B^{e_j}, C_mix = sum_j g_j C^{e_j}; delta = softplus(dt_mix).
 *   scan_fwd    ONE recurrence on the mixed parameters (no per-expert state):
 *               A_t = sum_j g_j A^{e_j};  h_t = exp(delta_t A_t) * h_{t-1} + delta_t B_mix,t x_t;
 *               y_t = C_mix,t . h_t + D_skip * x_t;  out_t = y_t * SiLU(z_t).
 *   step        the same for one token per sequence, state updated in place (decode).
 *
 * Conventions shared by every call
 *   - All tensors are dense, row-major, last index fastest. Shapes use B = batch, L = seqlen,
 *     D = d_inner, N = d_state, R = dt_rank, E = n_experts, k = top_k, T = B*L tokens.
 *   - Pointers are DEVICE pointers. The caller owns every buffer; the library never allocates,
 *     frees or synchronises (except swimba_get_device_status, which synchronises its stream).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy stream).
 *   - Argument errors are returned synchronously, before anything is launched. Errors found on
 *     the device (a bounded wait that gave up) are written to the status block at the start of
 *     the workspace and returned by swimba_get_device_status.
 *   - Requirements: 1 <= k <= E <= 16; 1 <= N <= 16; D % 8 == 0; 1 <= R <= 256;
 *     every tensor pointer (x, z, out, delta, B_mix, C_mix, h0, h_final, y_pre, the weight
 *     tables) and the workspace 16-byte aligned. Anything else returns SWIMBA_ERR_UNSUPPORTED /
 *     SWIMBA_ERR_ALIGN; there is no host-side fallback path.
 *   - One workspace must not be used by two calls that may run concurrently.
 */
#ifndef SWIMBA_H
#define SWIMBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SWIMBA_OK = 0,
  SWIMBA_ERR_INVALID_ARG = 1, /* null required pointer, non-positive size, k > E, ... */
  SWIMBA_ERR_UNSUPPORTED = 2, /* shape outside the supported envelope (see above) */
  SWIMBA_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  SWIMBA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than swimba_workspace_size() */
  SWIMBA_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  SWIMBA_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up (device status only) */
} swimba_status;

typedef enum { SWIMBA_F32 = 0, SWIMBA_BF16 = 1 } swimba_dtype;

/* Operation codes for swimba_workspace_size. */
enum {
  SWIMBA_OP_ROUTE = 0,
  SWIMBA_OP_PROJ = 1,
  SWIMBA_OP_SCAN = 2,
  SWIMBA_OP_STEP = 3,
  SWIMBA_OP_LAYER = 4,  /* large enough for every op of the layer */
  SWIMBA_OP_SUMMARY = 5, /* swimba_scan_summary */
  SWIMBA_OP_SEPARATE = 6, /* swimba_separate_scan */
  SWIMBA_OP_SCAN_BWD = 7,  /* swimba_scan_bwd */
  SWIMBA_OP_PROJ_BWD = 8,  /* swimba_proj_bwd */
  SWIMBA_OP_ROUTE_BWD = 9  /* swimba_route_bwd */
};

typedef struct {
  int64_t batch;     /* B */
  int64_t seqlen;    /* L (1 for swimba_step) */
  int32_t d_inner;   /* D */
  int32_t d_state;   /* N */
  int32_t dt_rank;   /* R */
  int32_t n_experts; /* E */
  int32_t top_k;     /* k */
  int32_t io_dtype;  /* swimba_dtype of x, z and out */
  int32_t w_dtype;   /* swimba_dtype of W_x and W_dt */
} swimba_dims;

typedef struct {
  const float *W_r;    /* [D, E]        router weights, fp32 */
  const void *W_x;     /* [E, D, R+2N]  per-expert x -> [dt_low | B | C], w_dtype */
  const void *W_dt;    /* [E, R, D]     per-expert dt_low -> dt, w_dtype */
  const float *b_dt;   /* [E, D]        per-expert dt bias, fp32 */
  const float *A;      /* [E, D, N]     per-expert diagonal transition, fp32, all < 0 */
  const float *D_skip; /* [D]           skip weights, fp32 */
} swimba_weights;

/* Bytes of device workspace `op` needs for `dims` (0 on invalid dims). The first 256 bytes are
 * the device status block: zero the whole workspace once after allocating it; the library keeps
 * the block consistent afterwards. */
size_t swimba_workspace_size(const swimba_dims *dims, int op);

/* Router (the pages' π_t): logits = x W_r accumulated in fp32; idx = the k largest in descending
 * order, equal logits to the lower expert index; gates = softmax of the k selected logits.
 * bf16 x with D a multiple of 64 and E in {4, 8, 12, 16} runs on the tensor cores (W_r split
 * exactly into three bf16 parts, fp32 accumulation); other shapes on the SIMT cores. A token whose
 * routing gave up after a bounded device-side wait (a device error, not expected in operation)
 * gets idx = -1 and gate 0; the later calls clamp such indices.
 *   x     [B, L, D] io_dtype          (in)
 *   W_r   [D, E] fp32                 (in)
 *   idx   [B, L, k] int32             (out)
 *   gates [B, L, k] fp32              (out; rows sum to 1, top-1 gives exactly 1) */
swimba_status swimba_route(const swimba_dims *dims, const void *x, const float *W_r, int32_t *idx,
                           float *gates, void *stream);

/* Per-expert SSM parameter streams mixed in parameter space (bf16 x/W on tcgen05 tensor cores with
 * fp32 accumulation when io_dtype = w_dtype = BF16; fp32 SIMT otherwise).
 *   x [B, L, D] io; idx, gates [B, L, k] from swimba_route; weights: W_x, W_dt, b_dt used.
 *   delta [B, L, D] fp32 (out) = softplus(dt_mix)
 *   B_mix [B, L, N] fp32 (out), C_mix [B, L, N] fp32 (out)
 *   ws: workspace of at least swimba_workspace_size(dims, SWIMBA_OP_PROJ) bytes. */
swimba_status swimba_mixed_proj(const swimba_dims *dims, const void *x, const int32_t *idx,
                                const float *gates, const swimba_weights *w, float *delta,
                                float *B_mix, float *C_mix, void *ws, size_t ws_bytes, void *stream);

/* The scan's contract on delta: it is the step size itself, delta = softplus(dt_mix), as
 * swimba_mixed_proj writes it (not the pre-softplus dt_mix), and every value must be finite and
 * >= 0. The fused discretise + scan + readout + skip + gate over the whole sequence.
 *   x, z [B, L, D] io; delta [B, L, D] fp32; B_mix, C_mix [B, L, N] fp32; idx, gates [B, L, k];
 *   weights: A, D_skip used.
 *   h0      [B, D, N] fp32 starting state, or NULL for zeros            (in)
 *   out     [B, L, D] io = y * SiLU(z)                                   (out)
 *   h_final [B, D, N] fp32 state after the last token, or NULL          (out; may alias h0)
 *   y_pre   [B, L, D] fp32 y before the gate, or NULL                   (out; diagnostics)
 *   ws: workspace of at least swimba_workspace_size(dims, SWIMBA_OP_SCAN) bytes (holds the
 *       per-segment carries when the sequence is split across CTAs). */
swimba_status swimba_scan_fwd(const swimba_dims *dims, const void *x, const void *z,
                              const float *delta, const float *B_mix, const float *C_mix,
                              const int32_t *idx, const float *gates, const swimba_weights *w,
                              const float *h0, void *out, float *h_final, float *y_pre, void *ws,
                              size_t ws_bytes, void *stream);

/* swimba_scan_fwd with the zero-order-hold injection of "Mamba y las SSMs: el retorno del estado
 * persistente", section "Mamba" (B-bar = A^-1 (exp(delta A) - I) B) in place of the Euler form
 * delta B x: with the diagonal mixed transition A_t the state update is
 *   h_t = exp(delta_t A_t) * h_{t-1} + (exp(delta_t A_t) - 1) / A_t * B_mix,t x_t.
 * Arguments, workspace and outputs as swimba_scan_fwd. Each state element costs one more
 * special-function operation (a reciprocal) than the Euler scan. */
swimba_status swimba_scan_fwd_zoh(const swimba_dims *dims, const void *x, const void *z,
                                  const float *delta, const float *B_mix, const float *C_mix,
                                  const int32_t *idx, const float *gates, const swimba_weights *w,
                                  const float *h0, void *out, float *h_final, float *y_pre, void *ws,
                                  size_t ws_bytes, void *stream);

/* Backward pass of swimba_scan_fwd (Euler injection): the exact gradients of the scan's outputs
 * with respect to its inputs, given g_out = dL/dout. The pages train Swimba-14B ("Swimba: Switch
 * Mamba Model Scales State Space Models", Dutch summary, "Resultaten") but give no training
 * details; this is reverse-mode differentiation of the forward above:
 *   dy_t = g_out,t SiLU(z_t);  dz_t = g_out,t y_t SiLU'(z_t)
 *   lambda_t = C_mix,t dy_t + exp(delta_{t+1} A_{t+1}) lambda_{t+1}      (per channel and state)
 *   dx_t = D dy_t + delta_t sum_n lambda_t B_mix,t;  dB_t = sum_d lambda_t delta_t x_t;
 *   dC_t = sum_d dy_t h_t;  ddelta_t = sum_n lambda_t (A_t a_t h_{t-1} + B_mix,t x_t);
 *   dA^e += g_j lambda_t delta_t a_t h_{t-1} (e = idx_j);  dgates_j = sum_{d,n} of that times A^e;
 *   dD = sum_t dy_t x_t;  dh0 = exp(delta_0 A_0) lambda_0.
 * The forward states are recomputed (checkpoints every 16 tokens, kept in ws), not read from the
 * forward call.
 *   Inputs as swimba_scan_fwd (x, z, g_out in io_dtype; delta, B_mix, C_mix, gates, A, D_skip, h0
 *   fp32); g_out [B, L, D] required.
 *   Outputs, fp32, all required except dh0: dx, dz, ddelta [B, L, D]; dB, dC [B, L, N];
 *   dgates [B, L, k]; dA [E, D, N] (w's A table shape); dD [D]; dh0 [B, D, N] or NULL.
 *   The sums over channels, tokens and sequences are taken in a fixed order (deterministic).
 *   ws: at least swimba_workspace_size(dims, SWIMBA_OP_SCAN_BWD) bytes (checkpoints, partial
 *   sums and a per-block scratch of the sub-block states: about B L D N / 4 + B L (2N + k) D / 16
 *   + 256 B D bytes). No pointer may alias another. */
swimba_status swimba_scan_bwd(const swimba_dims *dims, const void *x, const void *z,
                              const float *delta, const float *B_mix, const float *C_mix,
                              const int32_t *idx, const float *gates, const swimba_weights *w,
                              const float *h0, const void *g_out, float *dx, float *dz,
                              float *ddelta, float *dB, float *dC, float *dgates, float *dA,
                              float *dD, float *dh0, void *ws, size_t ws_bytes, void *stream);

/* Backward pass of swimba_mixed_proj: given dL/ddelta (g_delta, e.g. swimba_scan_bwd's ddelta) and
 * dL/dB_mix, dL/dC_mix, the gradients of the mixed projection's inputs and weights ("Swimba: Switch
 * Mamba Model Scales State Space Models", §2 "Generación de Parámetros" / "Mezcla en el Espacio de
 * Parámetros": v_j = x W_x^{e_j} = [dt_low | B | C], dt_j = dt_low W_dt^{e_j} + b_dt^{e_j},
 * delta = softplus(sum_j g_j dt_j), B_mix = sum_j g_j B_j, C_mix = sum_j g_j C_j; the pages give no
 * training details, this is the exact reverse-mode gradient). softplus' derivative is taken from
 * delta itself: sigma(dt_mix) = 1 - exp(-delta).
 *   x [B, L, D] bf16; idx, gates [B, L, k] (the router's); w: W_x, W_dt (bf16), b_dt (fp32);
 *   delta [B, L, D] fp32 (the forward's output); g_delta [B, L, D], g_B, g_C [B, L, N] fp32.
 *   Outputs fp32: dx [B, L, D] (overwritten, or added to when dx_accumulate != 0);
 *   dgates [B, L, k] (this step's part of dL/dgates); dW_x [E, D, R+2N]; dW_dt [E, R, D];
 *   db_dt [E, D] (every expert's, zeros for an expert no token chose).
 * Products run on the tensor cores with bf16 operands (x, dL/d(dt_mix), and the per-token rows
 * built from them are rounded to bf16 once) and fp32 accumulation. Needs io_dtype = w_dtype =
 * bf16, R % 8 == 0, N % 4 == 0 (SWIMBA_ERR_UNSUPPORTED otherwise). The call reads the number of
 * (token, slot) pairs per expert back to the host once, so it synchronises `stream` and cannot be
 * captured in a CUDA graph. ws: swimba_workspace_size(dims, SWIMBA_OP_PROJ_BWD) bytes. */
swimba_status swimba_proj_bwd(const swimba_dims *dims, const void *x, const int32_t *idx,
                              const float *gates, const swimba_weights *w, const float *delta,
                              const float *g_delta, const float *g_B, const float *g_C, float *dx,
                              int32_t dx_accumulate, float *dgates, float *dW_x, float *dW_dt,
                              float *db_dt, void *ws, size_t ws_bytes, void *stream);

/* Backward pass of swimba_route: the gates are the softmax of the k selected logits of x W_r (the
 * selection itself is piecewise constant and carries no gradient). With G = g_gates_a (+ g_gates_b
 * when not NULL, e.g. the scan's and the projection's parts of dL/dgates):
 *   dL/dlogit_{idx_j} = gates_j (G_j - sum_i gates_i G_i);  dx += dlogits W_r^T;  dW_r = x^T dlogits.
 *   x [B, L, D] io_dtype; W_r [D, E] fp32; idx, gates, g_gates_* [B, L, k] fp32.
 *   dx [B, L, D] fp32 (overwritten, or added to when dx_accumulate != 0); dW_r [D, E] fp32.
 *   ws: swimba_workspace_size(dims, SWIMBA_OP_ROUTE_BWD) bytes. */
swimba_status swimba_route_bwd(const swimba_dims *dims, const void *x, const float *W_r,
                               const int32_t *idx, const float *gates, const float *g_gates_a,
                               const float *g_gates_b, float *dx, int32_t dx_accumulate,
                               float *dW_r, void *ws, size_t ws_bytes, void *stream);

/* swimba_scan_fwd without a caller workspace, for callers that cannot allocate device memory: a
 * plugin inside a framework that owns all device memory and gives it no allocator, or a
 * latency-critical loop that must not call cudaMalloc (which can synchronise the device). The pages
 * have no counterpart of this; it is a deployment convenience.
 *   Arguments as swimba_scan_fwd, minus ws / ws_bytes. The scratch is a fixed 8 MiB array inside the
 *   library (every GPU that loads the library holds it until the process exits). Shapes whose
 *   scratch would exceed it return SWIMBA_ERR_WORKSPACE (swimba_last_error_string says how much was
 *   needed); nothing is allocated or freed.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress, once per
 *   device, with that device current); make that first call before any stream capture.
 *   Every call shares the one array and overwrites what the last call left there; calls that may
 *   overlap on the GPU (other streams, other threads) race and must not be issued. The status
 *   block at the start of the array is cleared at every call; a bounded device-side wait that gave
 *   up during the call is recorded there and read by swimba_scan_fwd_noalloc_status. */
swimba_status swimba_scan_fwd_noalloc(const swimba_dims *dims, const void *x, const void *z,
                                      const float *delta, const float *B_mix, const float *C_mix,
                                      const int32_t *idx, const float *gates, const swimba_weights *w,
                                      const float *h0, void *out, float *h_final, float *y_pre,
                                      void *stream);

/* Device status of the last swimba_scan_fwd_noalloc call on the current device: synchronises
 * `stream`, returns SWIMBA_OK or SWIMBA_ERR_TIMEOUT (a bounded wait that gave up; out, h_final and
 * y_pre are then incomplete) from the fixed array's status block, and clears it. */
swimba_status swimba_scan_fwd_noalloc_status(void *stream);

/* Device address of that status block on the current device (NULL if the lookup failed): the
 * 256-byte block swimba_get_device_status and swimba_check_wait_timeout accept as `ws`. */
void *swimba_scan_fwd_noalloc_status_block(void);

/* ---- Splitting a long sequence into pieces ---------------------------------------------------
 * ("Mamba y las SSMs: el retorno del estado persistente", "Estado interno puramente lineal": the
 * state is linear, so the recurrence can be cut and recombined.) Over a piece of tokens the state
 * after the piece is exp(sum_t delta_t A_t) * h_in + h_zero, h_zero being the end state when the
 * piece starts from zero. A sequence cut into P consecutive pieces (e.g. one per GPU) is scanned
 * by: swimba_scan_summary on every piece, an exchange of the summaries, swimba_scan_chain for the
 * start states, then swimba_scan_fwd on every piece from its start state (h0).
 *
 * Summary of the pieces given as the B sequences of `dims` (each its own piece):
 *   x [B, L, D] io; delta [B, L, D] fp32; B_mix [B, L, N] fp32; idx, gates [B, L, k]; weights: A.
 *   h_zero    [B, D, N] fp32 (out) end state of the recurrence started from zero
 *   log_decay [B, D, N] fp32 (out) sum over the piece's tokens of delta_t A_t (natural log)
 *   ws: at least swimba_workspace_size(dims, SWIMBA_OP_SUMMARY) bytes. */
swimba_status swimba_scan_summary(const swimba_dims *dims, const void *x, const float *delta,
                                  const float *B_mix, const int32_t *idx, const float *gates,
                                  const swimba_weights *w, float *h_zero, float *log_decay, void *ws,
                                  size_t ws_bytes, void *stream);

/* Start states of `parts` consecutive pieces from their summaries (dims: batch, d_inner and
 * d_state are used):
 *   h_zero, log_decay [parts, B, D, N] fp32 (in), piece 0 first
 *   h0      [B, D, N] fp32 state before piece 0, or NULL for zeros   (in)
 *   h_start [parts + 1, B, D, N] fp32 (out): h_start[0] = h0, h_start[p+1] =
 *           exp(log_decay[p]) * h_start[p] + h_zero[p]; h_start[parts] is the state after the
 *           whole sequence. */
swimba_status swimba_scan_chain(const swimba_dims *dims, int32_t parts, const float *h_zero,
                                const float *log_decay, const float *h0, float *h_start, void *stream);

/* ---- The MoE of separate SSMs (the design Swimba is set against) ----------------------------
 * ("Swimba: Switch Mamba Model Scales State Space Models", Spanish summary §2 "Distinción de
 * Diseños", Dutch "Methodologie", French "Distinction des deux designs MoE-SSM"; Teorema 2.) Every
 * expert keeps its own state trajectory h^(e) [B, D, N] and its own recurrence; at token t the k
 * active experts advance their states with their own unmixed streams and transition,
 *   h^(e_j) = exp(delta^j A^{e_j}) * h^(e_j) + delta^j B^j x_t   (delta^j = softplus(dt^j)),
 * the other experts' states stay as they are, and y_t = sum_j g_j C^j . h^(e_j) + D_skip * x_t,
 * out_t = y_t * SiLU(z_t). Built as the measured comparison for Teorema 2; the recurrence work
 * grows with k (Swimba's does not).
 *
 * Per-slot streams (SIMT, one CTA per token; weights W_x, W_dt, b_dt):
 *   delta_j [B, L, k, D] fp32 (out) = softplus(x W_x^{e_j}[:, :R] W_dt^{e_j} + b_dt^{e_j})
 *   B_j, C_j [B, L, k, N] fp32 (out) = the slot's B and C columns of x W_x^{e_j}, unmixed */
swimba_status swimba_separate_proj(const swimba_dims *dims, const void *x, const int32_t *idx,
                                   const float *gates, const swimba_weights *w, float *delta_j,
                                   float *B_j, float *C_j, void *stream);

/* The separate-SSM scan over whole sequences.
 *   x, z [B, L, D] io; delta_j [B, L, k, D]; B_j, C_j [B, L, k, N]; idx, gates [B, L, k];
 *   weights: A, D_skip used.
 *   h0      [E, B, D, N] fp32 every expert's start state, or NULL for zeros   (in)
 *   out     [B, L, D] io                                                         (out)
 *   h_final [E, B, D, N] fp32 every expert's state after the last token, or NULL (out)
 *   y_pre   [B, L, D] fp32 or NULL                                              (out)
 *   ws: at least swimba_workspace_size(dims, SWIMBA_OP_SEPARATE) bytes (the status block).
 * bf16 io with N = 16, k <= 2, E <= 8 and D % 16 == 0 keeps every expert's A rows and state in
 * tensor memory; other shapes run a per-channel SIMT kernel. */
swimba_status swimba_separate_scan(const swimba_dims *dims, const void *x, const void *z,
                                   const float *delta_j, const float *B_j, const float *C_j,
                                   const int32_t *idx, const float *gates, const swimba_weights *w,
                                   const float *h0, void *out, float *h_final, float *y_pre, void *ws,
                                   size_t ws_bytes, void *stream);

/* ---- Swimba on the Mamba-2 state-space-dual form ---------------------------------------------
 * ("Swimba: Switch Mamba Model Scales State Space Models", Spanish summary §2 "Arquitectura de
 * Swimba": built on Mamba-2 and its state space duality; expert-specific streams B^(e), C^(e),
 * X^(e); the transition A shared by the experts and over time; Dutch summary §2 "Architectuur
 * Implementatie": the SSD computation and chunked processing carry over.) Heads of P channels,
 * one negative scalar A_h per head, one step delta_t[h] per token, the active expert's streams
 * X_t [H, P] and B_t [N], gate g_t and the gate-mixed readout C_mix,t [N]:
 *   S_t[h] = exp(delta_t[h] A_h) S_{t-1}[h] + delta_t[h] g_t X_t[h] (outer) B_t
 *   y_t[h] = S_t[h] C_mix,t + D_skip[h] g_t X_t[h]
 * evaluated in chunks of 128 tokens on the tensor cores (the decay-masked C B^T products, the
 * carried state's readout and the state update are bf16 MMAs with fp32 accumulation; the state is
 * carried in fp32). Supported: head_dim 64, d_state 128, top_k 1 (the pages' model routes each
 * token to one expert); anything else returns SWIMBA_ERR_UNSUPPORTED. */
typedef struct {
  int64_t batch;    /* B */
  int64_t seqlen;   /* L */
  int32_t n_heads;  /* H */
  int32_t head_dim; /* P */
  int32_t d_state;  /* N */
  int32_t top_k;    /* k (active experts per token) */
} swimba_ssd_dims;

/*   X       [B, L, k, H, P] bf16: the active expert's input stream X^(e_t)_t       (in)
 *   B_j     [B, L, k, N] bf16: its state-input stream B^(e_t)_t                   (in)
 *   C_mix   [B, L, N] bf16: the gate-mixed readout stream                         (in)
 *   gates   [B, L, k] fp32; delta [B, L, H] fp32 (> 0); A [H] fp32 (< 0); D_skip [H] fp32
 *   S0      [B, H, P, N] fp32 start state, or NULL for zeros                       (in)
 *   y       [B, L, H, P] fp32                                                      (out)
 *   S_final [B, H, P, N] fp32 state after the last token, or NULL                  (out)
 *   ws: at least 256 bytes (the status block). One CTA per (sequence, head). */
swimba_status swimba_ssd_scan(const swimba_ssd_dims *dims, const void *X, const void *B_j,
                              const void *C_mix, const float *gates, const float *delta,
                              const float *A, const float *D_skip, const float *S0, float *y,
                              float *S_final, void *ws, size_t ws_bytes, void *stream);

/* One decode step (dims->seqlen must be 1): the scan for a single token per sequence, continuing
 * from and overwriting the cached state h [B, D, N] fp32. Other arguments as swimba_scan_fwd. */
swimba_status swimba_step(const swimba_dims *dims, const void *x, const void *z, const float *delta,
                          const float *B_mix, const float *C_mix, const int32_t *idx,
                          const float *gates, const swimba_weights *w, float *h, void *out,
                          void *stream);

/* ---- The surrounding block -------------------------------------------------------------------
 * ("Mamba y las SSMs: el retorno del estado persistente", section "Mamba", Figura 3: a linear
 * projection makes the two branches, a convolution and SiLU act on the SSM branch, the gated SSM,
 * a linear output projection; section "Estado interno puramente lineal": output projection and
 * residual connection. "Swimba: Switch Mamba Model Scales State Space Models", Dutch summary §2
 * "Architectuur Implementatie": the base block's in-projection becomes the module that makes the
 * expert-specific parameters, the rest of the block is unchanged.)
 *
 *   [x_pre | z] = u W_in;  x = SiLU(c),  c[t,d] = conv_b[d] + sum_{i<W} conv_w[d,i] p[t+i,d],
 *   p = [conv_state_in ; x_pre] along time (the W-1 inputs before the first token, oldest first);
 *   the Swimba layer on (x, z) gives out_layer = y * SiLU(z);  o = out_layer W_out + u.
 *
 * The in- and out-projections are dense GEMMs run by the library's own kernel (swimba_block_gemm
 * below: tcgen05 tensor cores for bf16, fp32 accumulation; a SIMT kernel for fp32). The
 * in-projection is one GEMM whose output columns are split between x_pre and z; the
 * out-projection adds the residual u in its epilogue. With bf16 activations x_pre, z, x, the
 * layer output and o are each rounded to bf16 once. Nothing allocates: every block call can be
 * captured in a CUDA graph. */

/* The block's projection GEMM on its own: C = A B (+ R), with the output columns [0, split)
 * written to C0 and [split, N) to C1 (the in-projection's [x_pre | z] split; split = N writes
 * everything to C0).
 *   dtype  SWIMBA_BF16: tcgen05 tensor cores, fp32 accumulation in tensor memory, bf16 out;
 *          SWIMBA_F32: fp32 SIMT kernel. A, B, R, C0, C1 all of that type.
 *   A      [M, K] row-major, row stride lda >= K                                   (in)
 *   B      [K, N] row-major, row stride ldb >= N                                   (in)
 *   R      [M, N] row stride ldr >= N, or NULL: added to the product (a residual)  (in)
 *   C0     [M, split] row stride ldc0 >= split; C1 [M, N - split] row stride ldc1  (out)
 *   C0 or C1 may be R itself (each element is read and written by one thread); no other overlap.
 * bf16 needs N, split and every row stride a multiple of 8 elements and 16-byte aligned
 * pointers (SWIMBA_ERR_UNSUPPORTED / SWIMBA_ERR_ALIGN otherwise). M = 0 or N = 0 is a no-op;
 * K must be at least 1. ws: at least 256 bytes (the status block; a tensor-core wait that
 * runs out leaves SWIMBA_ERR_TIMEOUT there). */
swimba_status swimba_block_gemm(int32_t dtype, int32_t M, int32_t N, int32_t K, const void *A,
                                int32_t lda, const void *B, int32_t ldb, void *C0, int32_t ldc0,
                                void *C1, int32_t ldc1, int32_t split, const void *R, int32_t ldr,
                                void *ws, size_t ws_bytes, void *stream);

typedef struct {
  swimba_dims layer; /* B, L, D, N, R, E, k and dtypes of the Swimba layer inside the block */
  int32_t d_model;   /* width of the block's input u and output o; a multiple of 8 */
  int32_t d_conv;    /* taps W of the causal convolution, 1 .. 8 */
} swimba_block_dims;

typedef struct {
  const void *W_in;     /* [d_model, 2D] io_dtype: columns [0, D) make x_pre, [D, 2D) make z */
  const float *conv_w;  /* [D, d_conv] taps; tap d_conv-1 weighs the current token */
  const float *conv_b;  /* [D] */
  const void *W_out;    /* [D, d_model] io_dtype */
  swimba_weights layer; /* the layer's weights (W_r, W_x, W_dt, b_dt, A, D_skip) */
} swimba_block_weights;

/* Causal depthwise convolution + SiLU over whole sequences (the block's second step).
 *   x_pre [B, L, D] io (in); conv_w [D, W] fp32; conv_b [D] fp32;
 *   conv_state_in  [B, W-1, D] io, the inputs before each sequence's first token, or NULL (zeros);
 *   x [B, L, D] io (out) = SiLU(c);
 *   conv_state_out [B, W-1, D] io (out) = the last W-1 rows of [conv_state_in ; x_pre], or NULL.
 *   conv_state_out must not be the same buffer as conv_state_in (W > 1). Both state pointers are
 *   ignored when W = 1. Requirements of the layer dims apply (D % 8 == 0, 16-byte alignment). */
swimba_status swimba_conv1d_fwd(const swimba_dims *dims, int32_t d_conv, const void *x_pre,
                                const float *conv_w, const float *conv_b, const void *conv_state_in,
                                void *x, void *conv_state_out, void *stream);

/* One decode token per sequence (dims->seqlen must be 1): x = SiLU(conv) from conv_state
 * [B, W-1, D] io and x_pre [B, 1, D]; conv_state is shifted by one token in place. */
swimba_status swimba_conv1d_step(const swimba_dims *dims, int32_t d_conv, const void *x_pre,
                                 const float *conv_w, const float *conv_b, void *conv_state,
                                 void *x, void *stream);

/* Bytes of device workspace a block call needs (0 on invalid dims). Its first 256 bytes are the
 * status block read by swimba_get_device_status; zero the workspace once after allocating it. */
size_t swimba_block_workspace_size(const swimba_block_dims *bd);

/* The whole block over whole sequences.
 *   u [B, L, d_model] io (in); h0 [B, D, N] fp32 or NULL (zeros); conv_state_in [B, W-1, D] io or
 *   NULL (zeros); out [B, L, d_model] io (out; may be u itself); h_final [B, D, N] fp32 or NULL
 *   (may alias h0); conv_state_out [B, W-1, D] io or NULL (not the same buffer as conv_state_in).
 *   Requires io_dtype == w_dtype and d_model % 8 == 0 (else SWIMBA_ERR_UNSUPPORTED). */
swimba_status swimba_block_fwd(const swimba_block_dims *bd, const void *u,
                               const swimba_block_weights *w, const float *h0,
                               const void *conv_state_in, void *out, float *h_final,
                               void *conv_state_out, void *ws, size_t ws_bytes, void *stream);

/* One decode step of the block (bd->layer.seqlen must be 1) from the cached SSM state h
 * [B, D, N] fp32 and conv state [B, W-1, D] io, both updated in place. */
swimba_status swimba_block_step(const swimba_block_dims *bd, const void *u,
                                const swimba_block_weights *w, float *h, void *conv_state,
                                void *out, void *ws, size_t ws_bytes, void *stream);

/* Synchronises `stream`, returns the device status recorded in the workspace's status block
 * (SWIMBA_OK or SWIMBA_ERR_TIMEOUT) and clears it. */
swimba_status swimba_get_device_status(void *ws, void *stream);

/* Runs the library's bounded-wait error path on the device, on purpose: one warp waits on an
 * mbarrier that nothing completes; after `limit_ns` nanoseconds (1e3 .. 1e9) it gives up and
 * records SWIMBA_ERR_TIMEOUT in the status block at the start of `ws`, as a stalled pipeline
 * stage of the other kernels would, then the kernel exits normally. Lets a caller check that a
 * stalled wait ends with a status (read it with swimba_get_device_status) rather than a hang, and
 * that the context stays usable. ws: at least 256 bytes of device memory (the status block).
 * The pages have no counterpart of this call; it exists to test failure reporting. */
swimba_status swimba_check_wait_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns, void *stream);

/* Static description of a status code. */
const char *swimba_status_string(swimba_status s);

/* Name and description of the last CUDA error this thread's calls turned into SWIMBA_ERR_CUDA. */
const char *swimba_last_error_string(void);

/* Number of kernels this library has launched in this process (all devices, all streams). */
uint64_t swimba_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* SWIMBA_H */
