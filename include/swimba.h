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
  SWIMBA_OP_LAYER = 4 /* large enough for every op of the layer */
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

/* The fused discretise + scan + readout + skip + gate over the whole sequence.
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
 *   overlap on the GPU (other streams, other threads) race and must not be issued. Device-side
 *   status of this variant is cleared at every call and is not reported. */
swimba_status swimba_scan_fwd_noalloc(const swimba_dims *dims, const void *x, const void *z,
                                      const float *delta, const float *B_mix, const float *C_mix,
                                      const int32_t *idx, const float *gates, const swimba_weights *w,
                                      const float *h0, void *out, float *h_final, float *y_pre,
                                      void *stream);

/* One decode step (dims->seqlen must be 1): the scan for a single token per sequence, continuing
 * from and overwriting the cached state h [B, D, N] fp32. Other arguments as swimba_scan_fwd. */
swimba_status swimba_step(const swimba_dims *dims, const void *x, const void *z, const float *delta,
                          const float *B_mix, const float *C_mix, const int32_t *idx,
                          const float *gates, const swimba_weights *w, float *h, void *out,
                          void *stream);

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
