// Router of the Swimba layer: logits = x W_r (fp32 accumulation), top-k, softmax of the selected.
//
// Source: "Swimba: Switch Mamba Model Scales State Space Models", §2 "Arquitectura de Swimba"
// (es) / "Kernmechanisme van Swimba" (nl): a router gives each token mixing weights π_t over the
// active experts (top-1 or top-k).
//
// Layout: one warp routes TOK consecutive tokens. Lanes stride over the channel dimension in
// 16-byte chunks of x (8 bf16 or 4 fp32), so every x load is a coalesced 128-bit load and x is
// read from HBM exactly once. The TOK x E partial sums of every lane are combined with a
// butterfly of warp shuffles; then lane tt selects the experts of token t0+tt.
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

template <typename IO, int EP, int TOK>
__global__ void __launch_bounds__(128) route_kernel(RouteParams p) {
  constexpr int V = Vec16<IO>::n;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t t0 = warp * TOK;
  if (t0 >= p.T) return;
  const int E = p.E;
  const int nchunks = p.D / V;
  const IO* x = reinterpret_cast<const IO*>(p.x);

  float acc[TOK][EP];
#pragma unroll
  for (int tt = 0; tt < TOK; ++tt)
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[tt][e] = 0.f;

  for (int c = lane; c < nchunks; c += 32) {
    float xf[TOK][V];
#pragma unroll
    for (int tt = 0; tt < TOK; ++tt) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t0 + tt < p.T) v = __ldg(reinterpret_cast<const uint4*>(x + (t0 + tt) * p.D) + c);
      Vec16<IO>::unpack(v, xf[tt]);
    }
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int d = c * V + i;
      float w[EP];
      if (E == EP) {
#pragma unroll
        for (int e4 = 0; e4 < EP / 4; ++e4) {
          const float4 q = __ldg(reinterpret_cast<const float4*>(p.W_r + (size_t)d * EP) + e4);
          w[4 * e4 + 0] = q.x; w[4 * e4 + 1] = q.y; w[4 * e4 + 2] = q.z; w[4 * e4 + 3] = q.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < EP; ++e) w[e] = (e < E) ? __ldg(p.W_r + (size_t)d * E + e) : 0.f;
      }
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt)
#pragma unroll
        for (int e = 0; e < EP; ++e) acc[tt][e] = fmaf(xf[tt][i], w[e], acc[tt][e]);
    }
  }

#pragma unroll
  for (int tt = 0; tt < TOK; ++tt)
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      float v = acc[tt][e];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      acc[tt][e] = v;
    }

#pragma unroll
  for (int tt = 0; tt < TOK; ++tt) {
    const int64_t t = t0 + tt;
    if (lane != tt || t >= p.T) continue;
    // top-k: repeatedly take the largest remaining logit; a strict comparison in ascending
    // expert order keeps the lower index on ties.
    unsigned taken = 0u;
    float wsel[16];
    float top = 0.f, sum = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      wsel[j] = 0.f;
      if (j < p.k) {
        int bi = -1;
        float best = 0.f;
#pragma unroll
        for (int e = 0; e < EP; ++e) {
          const bool ok = (e < E) && !((taken >> e) & 1u);
          if (ok && (bi < 0 || acc[tt][e] > best)) {
            best = acc[tt][e];
            bi = e;
          }
        }
        taken |= 1u << bi;
        if (j == 0) top = best;
        wsel[j] = expf(best - top);
        sum += wsel[j];
        p.idx[t * p.k + j] = bi;
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < p.k) p.gates[t * p.k + j] = wsel[j] / sum;
  }
}

template <typename IO, int EP, int TOK>
static cudaError_t launch_route(const RouteParams& p, cudaStream_t s) {
  const int64_t warps = (p.T + TOK - 1) / TOK;
  const int64_t blocks = (warps + 3) / 4;
  route_kernel<IO, EP, TOK><<<(unsigned)blocks, 128, 0, s>>>(p);
  note_launch();
  return cudaGetLastError();
}

template <typename IO>
static cudaError_t route_dispatch(const RouteParams& p, cudaStream_t s) {
  if (p.E <= 4) return launch_route<IO, 4, 8>(p, s);
  if (p.E <= 8) return launch_route<IO, 8, 8>(p, s);
  return launch_route<IO, 16, 4>(p, s);
}

cudaError_t run_route(const void* x, bool io_bf16, const float* W_r, int32_t* idx, float* gates, int64_t T,
                      int D, int E, int k, cudaStream_t s) {
  RouteParams p{x, W_r, idx, gates, T, D, E, k};
  return io_bf16 ? route_dispatch<__nv_bfloat16>(p, s) : route_dispatch<float>(p, s);
}

}  // namespace swimba
