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

// Fixed device scratch used by swimba_scan_fwd_noalloc (status block + segment carries).
constexpr size_t kScanNoAllocScratchBytes = size_t(8) << 20;
cudaError_t scan_noalloc_scratch(void** addr);

}  // namespace swimba
