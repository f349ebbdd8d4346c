// Router pieces shared by the SIMT kernels (route.cu) and the tensor-core kernel (route_tc.cu).
#pragma once
#include "common.cuh"

namespace swimba {

struct RouteParams {
  const void* x;
  const float* W_r;
  int32_t* idx;
  float* gates;
  int64_t T;
  int D, E, k;
};

// top-k of one token's logits l[0..E): repeatedly take the largest remaining logit; a strict
// comparison in ascending expert order keeps the lower index on ties. gates = softmax of the
// selected logits (exp relative to the largest, so the first gate's weight is exactly 1).
template <int EP>
__device__ __forceinline__ void select_topk(const float (&l)[EP], int E, int k, int32_t* idx, float* gates) {
  unsigned taken = 0u;
  float wsel[16];
  float top = 0.f, sum = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    wsel[j] = 0.f;
    if (j < k) {
      int bi = -1;
      float best = 0.f;
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        const bool ok = (e < E) && !((taken >> e) & 1u);
        if (ok && (bi < 0 || l[e] > best)) {
          best = l[e];
          bi = e;
        }
      }
      taken |= 1u << bi;
      if (j == 0) top = best;
      wsel[j] = expf(best - top);
      sum += wsel[j];
      idx[j] = bi;
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (j < k) gates[j] = wsel[j] / sum;
}

// Up to this many tokens the router runs one CTA per 2-4 tokens (route_small_kernel): enough CTAs
// to fill the GPU when T is small, where the tile-streaming kernels would leave most SMs idle.
constexpr int64_t kSmallT = 2048;

// Tensor-core router (route_tc.cu): bf16 x, D a multiple of 64, E <= 16.
bool route_tc_supported(bool io_bf16, int D, int E, int k);
cudaError_t run_route_tc(const RouteParams& p, cudaStream_t s);

}  // namespace swimba
