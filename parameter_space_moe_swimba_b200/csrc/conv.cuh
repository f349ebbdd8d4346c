// Causal depthwise convolution + SiLU of the Swimba block (kernels in conv.cu).
#pragma once

#include "common.cuh"

namespace swimba {

constexpr int kMaxConvWidth = 8;

struct ConvParams {
  int64_t Bsz, L;        // sequences, tokens per sequence (1 for the decode step)
  int D, W;              // channels (D % 8 == 0), taps (1 .. kMaxConvWidth)
  const void* x_pre;     // [B, L, D] io
  const float* conv_w;   // [D, W]
  const float* conv_b;   // [D]
  const void* state_in;  // [B, W-1, D] io or null (zeros); unused by the step
  void* x;               // [B, L, D] io = SiLU(conv)
  void* state_out;       // [B, W-1, D] io or null; the step's in/out state
};

// step = false: the whole sequence (state_in -> state_out); step = true: one token per sequence,
// state_out read and shifted in place.
cudaError_t run_conv1d(const ConvParams& p, bool io_bf16, bool step, cudaStream_t s);

}  // namespace swimba
