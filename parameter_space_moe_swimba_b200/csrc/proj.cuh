// Parameters shared by the two mixed-projection paths (SIMT and tcgen05).
#pragma once

#include "common.cuh"

namespace swimba {

struct ProjParams {
  const void* x;        // [T, D] io
  const int32_t* idx;   // [T, k]
  const float* gates;   // [T, k]
  const void* W_x;      // [E, D, R+2N] w
  const void* W_dt;     // [E, R, D] w
  const float* b_dt;    // [E, D]
  float* delta;         // [T, D]  softplus(dt_mix)
  float* B_mix;         // [T, N]
  float* C_mix;         // [T, N]
  int64_t T;
  int D, N, R, E, k;
};

// softplus(v) = log(1 + e^v); for v > 20 the correction log1p(e^-v) is below 2e-9 relative.
__device__ __forceinline__ float softplus_f32(float v) { return v > 20.f ? v : log1pf(expf(v)); }

}  // namespace swimba
