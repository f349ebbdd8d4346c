// C ABI of libswimba: argument validation, workspace layout and kernel dispatch. The layer's
// steps run in the kernels of route.cu, proj_simt.cu, proj_tc.cu and scan.cu.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "proj.cuh"
#include "scan.cuh"
#include "sm100.cuh"

namespace swimba {
cudaError_t run_route(const void* x, bool io_bf16, const float* W_r, int32_t* idx, float* gates, int64_t T, int D,
                      int E, int k, cudaStream_t s);
cudaError_t run_proj_simt(const ProjParams& p, bool io_bf16, bool w_bf16, cudaStream_t s);
bool proj_tc_supported(const ProjParams& p, bool io_bf16, bool w_bf16);
size_t proj_tc_workspace(int64_t T, int E, int k, int R, int D);
cudaError_t run_proj_tc(const ProjParams& p, void* ws, cudaStream_t s);
cudaError_t run_separate_proj(const ProjParams& p, bool io_bf16, bool w_bf16, float* dj, float* bj, float* cj,
                              cudaStream_t s);
cudaError_t separate_scan_entry(const void* x, const void* z, const float* dj, const float* bj, const float* cj,
                                const int32_t* idx, const float* gates, const float* A, const float* D_skip,
                                const float* h0, void* out, float* h_final, float* y_pre, void* status, int64_t L,
                                int B, int D, int N, int E, int k, bool io_bf16, cudaStream_t s);
size_t proj_bwd_workspace(int64_t T, int D, int R, int N, int E, int k);
cudaError_t run_proj_bwd(const void* x, const float* delta, const float* g_delta, const float* gB, const float* gC,
                         const int32_t* idx, const float* gates, const void* W_x, const void* W_dt, const void* b_dt,
                         bool b_bf16, float* dx, int accumulate, float* dgates, float* dW_x, float* dW_dt, float* db,
                         int64_t T, int D, int R, int N, int E, int k, void* ws, void* status, cudaStream_t s);
size_t route_bwd_workspace(int64_t T, int D, int E);
cudaError_t run_route_bwd(const void* x, bool io_bf16, const float* W_r, const int32_t* idx, const float* gates,
                          const float* gg_a, const float* gg_b, void* ws, float* dx, int accumulate, float* dW_r,
                          int64_t T, int D, int E, int k, cudaStream_t s);
bool ssd_supported(int P, int N, int k);
cudaError_t run_ssd(const void* X, const void* Bm, const void* Cmix, const float* gates, const float* delta,
                    const float* A, const float* D_skip, const float* S0, float* y, float* S_final, void* status,
                    int64_t L, int B, int H, cudaStream_t s);
}  // namespace swimba

namespace swimba {
static std::atomic<uint64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace swimba

using namespace swimba;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

swimba_status check_dims(const swimba_dims* d) {
  if (d == nullptr) return SWIMBA_ERR_INVALID_ARG;
  if (d->batch <= 0 || d->seqlen <= 0 || d->d_inner <= 0 || d->d_state <= 0 || d->dt_rank <= 0 ||
      d->n_experts <= 0 || d->top_k <= 0)
    return SWIMBA_ERR_INVALID_ARG;
  if (d->top_k > d->n_experts) return SWIMBA_ERR_INVALID_ARG;
  if ((d->io_dtype != SWIMBA_F32 && d->io_dtype != SWIMBA_BF16) ||
      (d->w_dtype != SWIMBA_F32 && d->w_dtype != SWIMBA_BF16))
    return SWIMBA_ERR_INVALID_ARG;
  if (d->n_experts > 16 || d->d_state > 16 || d->dt_rank > 256 || (d->d_inner % 8) != 0)
    return SWIMBA_ERR_UNSUPPORTED;
  if (d->batch > (1 << 30) || d->seqlen > (int64_t(1) << 40) || d->batch * d->seqlen > (int64_t(1) << 31))
    return SWIMBA_ERR_UNSUPPORTED;
  if ((int64_t)d->batch * d->seqlen * d->d_inner > (int64_t(1) << 40)) return SWIMBA_ERR_UNSUPPORTED;
  return SWIMBA_OK;
}

thread_local char g_last_error[256] = "no error";

swimba_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SWIMBA_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return SWIMBA_ERR_CUDA;
}

// Shape-only projection parameters (pointers unset), used to pick the path and size workspaces.
ProjParams proj_shape(const swimba_dims* d) {
  ProjParams p{};
  p.T = d->batch * d->seqlen;
  p.D = d->d_inner;
  p.N = d->d_state;
  p.R = d->dt_rank;
  p.E = d->n_experts;
  p.k = d->top_k;
  return p;
}

bool use_tc(const swimba_dims* d) {
  return proj_tc_supported(proj_shape(d), d->io_dtype == SWIMBA_BF16, d->w_dtype == SWIMBA_BF16);
}

size_t proj_workspace(const swimba_dims* d) {
  return use_tc(d) ? proj_tc_workspace(d->batch * d->seqlen, d->n_experts, d->top_k, d->dt_rank, d->d_inner) : kStatusBytes;
}

ScanPlan scan_plan(const swimba_dims* d) {
  return scan_fast_plan(d->batch, d->seqlen, d->d_inner, d->d_state, d->n_experts, d->top_k,
                        d->io_dtype == SWIMBA_BF16);
}

size_t scan_workspace(const swimba_dims* d) {
  const ScanPlan pl = scan_plan(d);
  return kStatusBytes + (pl.fast ? pl.ws_bytes : 0);
}

size_t summary_workspace(const swimba_dims* d) {
  const ScanPlan pl = scan_plan(d);
  return kStatusBytes + (pl.fast ? scan_fast_summary_ws(pl, d->batch, d->d_inner) : 0);
}

}  // namespace

namespace swimba {
// Shared with block.cu (the surrounding block's entry points).
swimba_status api_check_dims(const swimba_dims* d) { return check_dims(d); }
swimba_status api_cuda_status(cudaError_t e) { return cuda_status(e); }
void api_set_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

// One warp waits on an mbarrier that nothing arrives on (its phase 0 never completes) until
// limit_ns have passed, then records SWIMBA_ERR_TIMEOUT like the pipelines' bounded waits do.
__global__ void wait_timeout_kernel(void* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncwarp();
  const uint64_t t0 = sm100::globaltimer_ns();
  while (!sm100::mbar_try_wait(&bar, 0)) {
    if (sm100::globaltimer_ns() - t0 > limit_ns) {
      if (threadIdx.x == 0) record_device_error(status, SWIMBA_ERR_TIMEOUT, 90, 0, 0);
      break;
    }
  }
}
}  // namespace swimba

extern "C" {

size_t swimba_workspace_size(const swimba_dims* dims, int op) {
  if (check_dims(dims) != SWIMBA_OK) return 0;
  switch (op) {
    case SWIMBA_OP_ROUTE:
    case SWIMBA_OP_STEP:
      return kStatusBytes;
    case SWIMBA_OP_SCAN:
      return scan_workspace(dims);
    case SWIMBA_OP_PROJ:
      return proj_workspace(dims);
    case SWIMBA_OP_LAYER:
      return std::max(proj_workspace(dims), scan_workspace(dims));
    case SWIMBA_OP_SUMMARY:
      return summary_workspace(dims);
    case SWIMBA_OP_SEPARATE:
      return kStatusBytes;
    case SWIMBA_OP_PROJ_BWD:
      return kStatusBytes + proj_bwd_workspace(dims->batch * dims->seqlen, dims->d_inner, dims->dt_rank,
                                               dims->d_state, dims->n_experts, dims->top_k);
    case SWIMBA_OP_ROUTE_BWD:
      return kStatusBytes + route_bwd_workspace(dims->batch * dims->seqlen, dims->d_inner, dims->n_experts);
    case SWIMBA_OP_SCAN_BWD:
      return kStatusBytes + scan_bwd_workspace(dims->batch, dims->seqlen, dims->d_inner, dims->d_state,
                                               dims->n_experts, dims->top_k);
    default:
      return 0;
  }
}

swimba_status swimba_route(const swimba_dims* dims, const void* x, const float* W_r, int32_t* idx, float* gates,
                           void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !W_r || !idx || !gates) return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W_r)) return SWIMBA_ERR_ALIGN;
  const int64_t T = dims->batch * dims->seqlen;
  return cuda_status(run_route(x, dims->io_dtype == SWIMBA_BF16, W_r, idx, gates, T, dims->d_inner, dims->n_experts,
                               dims->top_k, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_mixed_proj(const swimba_dims* dims, const void* x, const int32_t* idx, const float* gates,
                                const swimba_weights* w, float* delta, float* B_mix, float* C_mix, void* ws,
                                size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !idx || !gates || !w || !w->W_x || !w->W_dt || !w->b_dt || !delta || !B_mix || !C_mix)
    return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(delta) || !aligned16(w->W_x) || !aligned16(w->W_dt)) return SWIMBA_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < swimba_workspace_size(dims, SWIMBA_OP_PROJ)) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  ProjParams p{x,     idx,   gates, w->W_x,       w->W_dt,        w->b_dt,         delta,
               B_mix, C_mix, dims->batch * dims->seqlen, dims->d_inner, dims->d_state, dims->dt_rank,
               dims->n_experts, dims->top_k};
  if (use_tc(dims)) {
    if (!aligned16(w->b_dt) || !aligned16(B_mix) || !aligned16(C_mix)) return SWIMBA_ERR_ALIGN;
    return cuda_status(run_proj_tc(p, ws, static_cast<cudaStream_t>(stream)));
  }
  return cuda_status(run_proj_simt(p, dims->io_dtype == SWIMBA_BF16, dims->w_dtype == SWIMBA_BF16,
                                   static_cast<cudaStream_t>(stream)));
}

static swimba_status scan_common(const swimba_dims* dims, const void* x, const void* z, const float* delta,
                                 const float* B_mix, const float* C_mix, const int32_t* idx, const float* gates,
                                 const swimba_weights* w, const float* h0, void* out, float* h_final, float* y_pre,
                                 bool step, void* ws, void* stream, bool zoh = false) {
  if (!x || !z || !delta || !B_mix || !C_mix || !idx || !gates || !w || !w->A || !w->D_skip || !out)
    return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(z) || !aligned16(out) || !aligned16(delta)) return SWIMBA_ERR_ALIGN;
  if (dims->d_state == 16 && (!aligned16(B_mix) || !aligned16(C_mix))) return SWIMBA_ERR_ALIGN;
  if ((h0 && !aligned16(h0)) || (h_final && !aligned16(h_final)) || (y_pre && !aligned16(y_pre)))
    return SWIMBA_ERR_ALIGN;
  if (!aligned16(w->A) || !aligned16(w->D_skip)) return SWIMBA_ERR_ALIGN;
  ScanParams p{x,   z,       delta, B_mix,          C_mix,          idx,           gates,
               w->A, w->D_skip, h0,  out,            h_final,        y_pre,         dims->seqlen,
               (int)dims->batch, dims->d_inner, dims->d_state, dims->n_experts, dims->top_k};
  p.zoh = zoh ? 1 : 0;
  if (!step) {
    const ScanPlan pl = scan_plan(dims);
    if (pl.fast) {
      uint8_t* seg_ws = reinterpret_cast<uint8_t*>(ws) + kStatusBytes;
      return cuda_status(run_scan_fast(p, pl, seg_ws, ws, static_cast<cudaStream_t>(stream)));
    }
  }
  return cuda_status(run_scan(p, dims->io_dtype == SWIMBA_BF16, step, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_scan_fwd(const swimba_dims* dims, const void* x, const void* z, const float* delta,
                              const float* B_mix, const float* C_mix, const int32_t* idx, const float* gates,
                              const swimba_weights* w, const float* h0, void* out, float* h_final, float* y_pre,
                              void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (ws == nullptr || ws_bytes < swimba_workspace_size(dims, SWIMBA_OP_SCAN)) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  return scan_common(dims, x, z, delta, B_mix, C_mix, idx, gates, w, h0, out, h_final, y_pre, false, ws, stream);
}

swimba_status swimba_scan_fwd_zoh(const swimba_dims* dims, const void* x, const void* z, const float* delta,
                                  const float* B_mix, const float* C_mix, const int32_t* idx, const float* gates,
                                  const swimba_weights* w, const float* h0, void* out, float* h_final, float* y_pre,
                                  void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (ws == nullptr || ws_bytes < swimba_workspace_size(dims, SWIMBA_OP_SCAN)) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  return scan_common(dims, x, z, delta, B_mix, C_mix, idx, gates, w, h0, out, h_final, y_pre, false, ws, stream,
                     true);
}

swimba_status swimba_scan_bwd(const swimba_dims* dims, const void* x, const void* z, const float* delta,
                              const float* B_mix, const float* C_mix, const int32_t* idx, const float* gates,
                              const swimba_weights* w, const float* h0, const void* g_out, float* dx, float* dz,
                              float* ddelta, float* dB, float* dC, float* dgates, float* dA, float* dD, float* dh0,
                              void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !z || !delta || !B_mix || !C_mix || !idx || !gates || !w || !w->A || !w->D_skip || !g_out || !dx || !dz ||
      !ddelta || !dB || !dC || !dgates || !dA || !dD)
    return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(w->A) || !aligned16(w->D_skip) || !aligned16(ws) || !aligned16(x) || !aligned16(z) ||
      !aligned16(delta) || !aligned16(B_mix) || !aligned16(C_mix) || !aligned16(g_out) || !aligned16(dx) ||
      !aligned16(dz) || !aligned16(ddelta) || (h0 && !aligned16(h0)) || (dh0 && !aligned16(dh0)))
    return SWIMBA_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < swimba_workspace_size(dims, SWIMBA_OP_SCAN_BWD)) return SWIMBA_ERR_WORKSPACE;
  ScanBwdParams p{};
  p.x = x;
  p.z = z;
  p.delta = delta;
  p.B_mix = B_mix;
  p.C_mix = C_mix;
  p.idx = idx;
  p.gates = gates;
  p.A = w->A;
  p.D_skip = w->D_skip;
  p.h0 = h0;
  p.g_out = g_out;
  p.dx = dx;
  p.dz = dz;
  p.ddelta = ddelta;
  p.dB = dB;
  p.dC = dC;
  p.dgates = dgates;
  p.dA = dA;
  p.dD = dD;
  p.dh0 = dh0;
  p.L = dims->seqlen;
  p.B = (int)dims->batch;
  p.D = dims->d_inner;
  p.N = dims->d_state;
  p.E = dims->n_experts;
  p.k = dims->top_k;
  p.status = ws;
  return cuda_status(run_scan_bwd(p, dims->io_dtype == SWIMBA_BF16, static_cast<uint8_t*>(ws) + kStatusBytes,
                                  static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_proj_bwd(const swimba_dims* dims, const void* x, const int32_t* idx, const float* gates,
                              const swimba_weights* w, const float* delta, const float* g_delta, const float* g_B,
                              const float* g_C, float* dx, int32_t dx_accumulate, float* dgates, float* dW_x,
                              float* dW_dt, float* db_dt, void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !idx || !gates || !w || !w->W_x || !w->W_dt || !w->b_dt || !delta || !g_delta || !g_B || !g_C || !dx ||
      !dgates || !dW_x || !dW_dt || !db_dt)
    return SWIMBA_ERR_INVALID_ARG;
  const int64_t T = dims->batch * dims->seqlen;
  if (dims->io_dtype != SWIMBA_BF16 || dims->w_dtype != SWIMBA_BF16 || dims->dt_rank % 8 != 0 ||
      dims->d_state % 4 != 0 || T * dims->top_k >= (int64_t(1) << 31))
    return SWIMBA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(delta) || !aligned16(g_delta) || !aligned16(dx) || !aligned16(dW_x) ||
      !aligned16(dW_dt) || !aligned16(db_dt) || !aligned16(w->W_x) || !aligned16(w->W_dt) ||
      !aligned16(w->b_dt) || !aligned16(ws))
    return SWIMBA_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < swimba_workspace_size(dims, SWIMBA_OP_PROJ_BWD)) return SWIMBA_ERR_WORKSPACE;
  return cuda_status(run_proj_bwd(x, delta, g_delta, g_B, g_C, idx, gates, w->W_x, w->W_dt, w->b_dt, false, dx,
                                  dx_accumulate ? 1 : 0, dgates, dW_x, dW_dt, db_dt, T, dims->d_inner, dims->dt_rank,
                                  dims->d_state, dims->n_experts, dims->top_k, static_cast<uint8_t*>(ws) + kStatusBytes,
                                  ws, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_route_bwd(const swimba_dims* dims, const void* x, const float* W_r, const int32_t* idx,
                               const float* gates, const float* g_gates_a, const float* g_gates_b, float* dx,
                               int32_t dx_accumulate, float* dW_r, void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !W_r || !idx || !gates || !g_gates_a || !dx || !dW_r) return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < swimba_workspace_size(dims, SWIMBA_OP_ROUTE_BWD)) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(dx) || !aligned16(W_r)) return SWIMBA_ERR_ALIGN;
  return cuda_status(run_route_bwd(x, dims->io_dtype == SWIMBA_BF16, W_r, idx, gates, g_gates_a, g_gates_b,
                                   static_cast<uint8_t*>(ws) + kStatusBytes, dx, dx_accumulate ? 1 : 0, dW_r,
                                   dims->batch * dims->seqlen, dims->d_inner, dims->n_experts, dims->top_k,
                                   static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_scan_fwd_noalloc(const swimba_dims* dims, const void* x, const void* z, const float* delta,
                                      const float* B_mix, const float* C_mix, const int32_t* idx, const float* gates,
                                      const swimba_weights* w, const float* h0, void* out, float* h_final,
                                      float* y_pre, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  const size_t need = scan_workspace(dims);
  if (need > kScanNoAllocScratchBytes) {
    snprintf(g_last_error, sizeof(g_last_error), "swimba_scan_fwd_noalloc: needs %zu bytes of scratch, the fixed "
             "array holds %zu", need, kScanNoAllocScratchBytes);
    return SWIMBA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (cuda_status(scan_noalloc_scratch(&scratch)) != SWIMBA_OK) return SWIMBA_ERR_CUDA;
  // the status block must start at zero; the segment carries are written before they are read
  if (cuda_status(cudaMemsetAsync(scratch, 0, kStatusBytes, static_cast<cudaStream_t>(stream))) != SWIMBA_OK)
    return SWIMBA_ERR_CUDA;
  return scan_common(dims, x, z, delta, B_mix, C_mix, idx, gates, w, h0, out, h_final, y_pre, false, scratch, stream);
}

swimba_status swimba_scan_fwd_noalloc_status(void* stream) {
  void* scratch = nullptr;
  if (cuda_status(scan_noalloc_scratch(&scratch)) != SWIMBA_OK) return SWIMBA_ERR_CUDA;
  return swimba_get_device_status(scratch, stream);
}

void* swimba_scan_fwd_noalloc_status_block(void) {
  void* scratch = nullptr;
  return scan_noalloc_scratch(&scratch) == cudaSuccess ? scratch : nullptr;
}

swimba_status swimba_scan_summary(const swimba_dims* dims, const void* x, const float* delta, const float* B_mix,
                                  const int32_t* idx, const float* gates, const swimba_weights* w, float* h_zero,
                                  float* log_decay, void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !delta || !B_mix || !idx || !gates || !w || !w->A || !h_zero || !log_decay) return SWIMBA_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < swimba_workspace_size(dims, SWIMBA_OP_SUMMARY)) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws) || !aligned16(x) || !aligned16(delta) || !aligned16(w->A) || !aligned16(h_zero) ||
      !aligned16(log_decay))
    return SWIMBA_ERR_ALIGN;
  if (dims->d_state == 16 && !aligned16(B_mix)) return SWIMBA_ERR_ALIGN;
  ScanParams p{x,       nullptr,  delta,   B_mix,  nullptr, idx,          gates,           w->A,
               nullptr, nullptr,  nullptr, nullptr, nullptr, dims->seqlen, (int)dims->batch, dims->d_inner,
               dims->d_state, dims->n_experts, dims->top_k};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ScanPlan pl = scan_plan(dims);
  if (pl.fast) {
    uint8_t* seg_ws = reinterpret_cast<uint8_t*>(ws) + kStatusBytes;
    return cuda_status(run_scan_summary_fast(p, pl, seg_ws, ws, h_zero, log_decay, s));
  }
  return cuda_status(run_scan_summary(p, dims->io_dtype == SWIMBA_BF16, h_zero, log_decay, s));
}

swimba_status swimba_scan_chain(const swimba_dims* dims, int32_t parts, const float* h_zero, const float* log_decay,
                                const float* h0, float* h_start, void* stream) {
  if (dims == nullptr || dims->batch <= 0 || dims->d_inner <= 0 || dims->d_state <= 0 || parts <= 0)
    return SWIMBA_ERR_INVALID_ARG;
  if (!h_zero || !log_decay || !h_start) return SWIMBA_ERR_INVALID_ARG;
  const int64_t bdn = dims->batch * (int64_t)dims->d_inner * dims->d_state;
  if (bdn > (int64_t(1) << 40) || parts > (1 << 20)) return SWIMBA_ERR_UNSUPPORTED;
  return cuda_status(run_scan_chain(bdn, parts, h_zero, log_decay, h0, h_start, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_separate_proj(const swimba_dims* dims, const void* x, const int32_t* idx, const float* gates,
                                   const swimba_weights* w, float* delta_j, float* B_j, float* C_j, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !idx || !gates || !w || !w->W_x || !w->W_dt || !w->b_dt || !delta_j || !B_j || !C_j)
    return SWIMBA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(delta_j) || !aligned16(w->W_x) || !aligned16(w->W_dt)) return SWIMBA_ERR_ALIGN;
  ProjParams p{x,       idx,     gates, w->W_x, w->W_dt, w->b_dt, nullptr, nullptr, nullptr, dims->batch * dims->seqlen,
               dims->d_inner, dims->d_state, dims->dt_rank, dims->n_experts, dims->top_k};
  return cuda_status(run_separate_proj(p, dims->io_dtype == SWIMBA_BF16, dims->w_dtype == SWIMBA_BF16, delta_j, B_j,
                                       C_j, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_separate_scan(const swimba_dims* dims, const void* x, const void* z, const float* delta_j,
                                   const float* B_j, const float* C_j, const int32_t* idx, const float* gates,
                                   const swimba_weights* w, const float* h0, void* out, float* h_final, float* y_pre,
                                   void* ws, size_t ws_bytes, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (!x || !z || !delta_j || !B_j || !C_j || !idx || !gates || !w || !w->A || !w->D_skip || !out)
    return SWIMBA_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < kStatusBytes) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws) || !aligned16(x) || !aligned16(z) || !aligned16(out) || !aligned16(delta_j) ||
      !aligned16(B_j) || !aligned16(C_j) || !aligned16(w->A) || !aligned16(w->D_skip))
    return SWIMBA_ERR_ALIGN;
  if ((h0 && !aligned16(h0)) || (h_final && !aligned16(h_final)) || (y_pre && !aligned16(y_pre)))
    return SWIMBA_ERR_ALIGN;
  return cuda_status(separate_scan_entry(x, z, delta_j, B_j, C_j, idx, gates, w->A, w->D_skip, h0, out, h_final,
                                         y_pre, ws, dims->seqlen, (int)dims->batch, dims->d_inner, dims->d_state,
                                         dims->n_experts, dims->top_k, dims->io_dtype == SWIMBA_BF16,
                                         static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_ssd_scan(const swimba_ssd_dims* d, const void* X, const void* B_j, const void* C_mix,
                              const float* gates, const float* delta, const float* A, const float* D_skip,
                              const float* S0, float* y, float* S_final, void* ws, size_t ws_bytes, void* stream) {
  if (d == nullptr || d->batch <= 0 || d->seqlen <= 0 || d->n_heads <= 0 || d->head_dim <= 0 || d->d_state <= 0 ||
      d->top_k <= 0)
    return SWIMBA_ERR_INVALID_ARG;
  if (!X || !B_j || !C_mix || !gates || !delta || !A || !D_skip || !y) return SWIMBA_ERR_INVALID_ARG;
  if (!ssd_supported(d->head_dim, d->d_state, d->top_k) || d->batch * d->n_heads > (int64_t(1) << 30) ||
      d->batch * d->seqlen > (int64_t(1) << 31))
    return SWIMBA_ERR_UNSUPPORTED;
  if (ws == nullptr || ws_bytes < kStatusBytes) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws) || !aligned16(X) || !aligned16(B_j) || !aligned16(C_mix) || !aligned16(y) ||
      (S0 && !aligned16(S0)) || (S_final && !aligned16(S_final)))
    return SWIMBA_ERR_ALIGN;
  return cuda_status(run_ssd(X, B_j, C_mix, gates, delta, A, D_skip, S0, y, S_final, ws, d->seqlen, (int)d->batch,
                             d->n_heads, static_cast<cudaStream_t>(stream)));
}

swimba_status swimba_step(const swimba_dims* dims, const void* x, const void* z, const float* delta,
                          const float* B_mix, const float* C_mix, const int32_t* idx, const float* gates,
                          const swimba_weights* w, float* h, void* out, void* stream) {
  swimba_status st = check_dims(dims);
  if (st != SWIMBA_OK) return st;
  if (dims->seqlen != 1 || h == nullptr) return SWIMBA_ERR_INVALID_ARG;
  return scan_common(dims, x, z, delta, B_mix, C_mix, idx, gates, w, h, out, h, nullptr, true, nullptr, stream);
}

swimba_status swimba_check_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream) {
  if (ws == nullptr || ws_bytes < kStatusBytes) return SWIMBA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SWIMBA_ERR_ALIGN;
  if (limit_ns < 1000 || limit_ns > 1000000000ull) return SWIMBA_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ws, limit_ns);
  note_launch();
  return cuda_status(cudaGetLastError());
}

swimba_status swimba_get_device_status(void* ws, void* stream) {
  if (ws == nullptr) return SWIMBA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SWIMBA_ERR_CUDA;
  DeviceStatus host{};
  if (cudaMemcpy(&host, ws, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess) return SWIMBA_ERR_CUDA;
  if (host.code != 0) {
    if (cudaMemset(ws, 0, sizeof(DeviceStatus)) != cudaSuccess) return SWIMBA_ERR_CUDA;
    return static_cast<swimba_status>(host.code);
  }
  return SWIMBA_OK;
}

const char* swimba_last_error_string(void) { return g_last_error; }

uint64_t swimba_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* swimba_status_string(swimba_status s) {
  switch (s) {
    case SWIMBA_OK: return "ok";
    case SWIMBA_ERR_INVALID_ARG: return "invalid argument";
    case SWIMBA_ERR_UNSUPPORTED: return "unsupported shape";
    case SWIMBA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SWIMBA_ERR_WORKSPACE: return "workspace missing or too small";
    case SWIMBA_ERR_CUDA: return "CUDA runtime error";
    case SWIMBA_ERR_TIMEOUT: return "bounded device wait gave up";
  }
  return "unknown status";
}

}  // extern "C"
