// Parameters of the scan and decode-step kernels.
#pragma once

#include "common.cuh"

namespace swimba {

struct ScanParams {
  const void* x;         // [B, L, D] io
  const void* z;         // [B, L, D] io
  const float* delta;    // [B, L, D]  softplus(dt_mix)
  const float* B_mix;    // [B, L, N]
  const float* C_mix;    // [B, L, N]
  const int32_t* idx;    // [B, L, k]
  const float* gates;    // [B, L, k]
  const float* A;        // [E, D, N]
  const float* D_skip;   // [D]
  const float* h0;       // [B, D, N] or null
  void* out;             // [B, L, D] io
  float* h_final;        // [B, D, N] or null
  float* y_pre;          // [B, L, D] or null
  int64_t L;
  int B, D, N, E, k;
  int zoh = 0;           // 1: zero-order-hold injection instead of Euler's
};

cudaError_t run_scan(const ScanParams& p, bool io_bf16, bool step, cudaStream_t s);

// Fast path plan: whether it applies, how many sequence segments, their length (a multiple of the
// 16-token chunk) and the workspace the segment carries need.
struct ScanPlan {
  bool fast;
  int S;
  int64_t Lseg;
  size_t ws_bytes;
};
ScanPlan scan_fast_plan(int64_t B, int64_t L, int D, int N, int E, int k, bool io_bf16);
cudaError_t run_scan_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, cudaStream_t s);
// The recurrence alone over whole sequences from h0 (bf16 x, N = 16, k <= 2: the fast-path shapes),
// writing the state at the start of every 16-token chunk into ckpt [B, nck, D, 16].
cudaError_t run_scan_fast_ckpt(const ScanParams& sp, float* ckpt, int nck, void* status, cudaStream_t s);

// Summary of a whole sequence (the hand-off of one piece of a longer one): h_zero [B, D, N] = the
// end state from zero, log_decay [B, D, N] = Σ_t Δ_t A_t. The fast path stages per-segment
// aggregates in scan_fast_summary_ws bytes of workspace; the generic path needs none.
size_t scan_fast_summary_ws(const ScanPlan& pl, int64_t B, int D);
cudaError_t run_scan_summary_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, float* h_zero,
                                  float* log_decay, cudaStream_t s);
cudaError_t run_scan_summary(const ScanParams& p, bool io_bf16, float* h_zero, float* log_decay, cudaStream_t s);

// Start states of P consecutive pieces from their summaries: h_start[0] = h0 (or zeros),
// h_start[p+1] = exp(log_decay[p]) h_start[p] + h_zero[p]; arrays [P(+1), B, D, N].
cudaError_t run_scan_chain(int64_t BDN, int P, const float* h_zero, const float* log_decay, const float* h0,
                           float* h_start, cudaStream_t s);

// Fixed device scratch used by swimba_scan_fwd_noalloc (status block + segment carries).
constexpr size_t kScanNoAllocScratchBytes = size_t(8) << 20;
cudaError_t scan_noalloc_scratch(void** addr);

// Backward pass of the scan (Euler injection): inputs as ScanParams plus the incoming gradient of
// out; gradients in fp32. ckpt, part, part_A, part_D and nck are set by run_scan_bwd inside `ws`.
struct ScanBwdParams {
  const void* x;         // [B, L, D] io
  const void* z;         // [B, L, D] io
  const float* delta;    // [B, L, D]
  const float* B_mix;    // [B, L, N]
  const float* C_mix;    // [B, L, N]
  const int32_t* idx;    // [B, L, k]
  const float* gates;    // [B, L, k]
  const float* A;        // [E, D, N]
  const float* D_skip;   // [D]
  const float* h0;       // [B, D, N] or null
  const void* g_out;     // [B, L, D] io: dL/dout
  float* dx;             // [B, L, D]
  float* dz;             // [B, L, D]
  float* ddelta;         // [B, L, D]
  float* dB;             // [B, L, N]
  float* dC;             // [B, L, N]
  float* dgates;         // [B, L, k]
  float* dA;             // [E, D, N]
  float* dD;             // [D]
  float* dh0;            // [B, D, N] or null
  float* ckpt;           // [B, nck, D, N]: the state at the start of every 16-token chunk
  float* part;           // [tiles, B, L, 2N + k]: per channel tile, dB | dC | dgates
  float* part_A;         // [B, E, D, N]
  float* part_D;         // [B, D]
  float* sub;            // [tiles * B, 4, 2, 128] float4: the packed kernel's sub-block states
  void* status;          // the workspace's device status block (bounded waits that gave up)
  int64_t L;
  int B, D, N, E, k;
  int nck;
};

size_t scan_bwd_workspace(int64_t B, int64_t L, int D, int N, int E, int k);
cudaError_t run_scan_bwd(ScanBwdParams p, bool io_bf16, void* ws, cudaStream_t s);

}  // namespace swimba
