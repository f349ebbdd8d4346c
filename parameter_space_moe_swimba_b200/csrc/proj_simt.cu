// Mixed expert projection, fp32 SIMT path (fp32 activations or weights, and small token counts).
//
// Source: "Swimba: Switch Mamba Model Scales State Space Models", §2 "Generación de Parámetros" /
// "Mezcla en el Espacio de Parámetros" (es), "Kernmechanisme van Swimba" (nl): each expert has its
// own linear projections producing token-dependent parameter streams; the streams of the active
// experts are combined with the router weights before the single recurrence.
//
// One CTA per token. Stage 1: v_j = x_t W_x^{e_j} ([dt_low | B | C]) with threads over the output
// columns (coalesced along the row of W_x). Stage 2 and the combine: threads over channels d,
// dt_mix[d] = sum_j g_j (dt_low_j . W_dt^{e_j}[:, d] + b_dt^{e_j}[d]), then delta = softplus.
#include "common.cuh"
#include "proj.cuh"

namespace swimba {

template <typename IO, typename WT>
__global__ void __launch_bounds__(256) proj_simt_kernel(ProjParams p) {
  extern __shared__ float sm[];
  const int64_t t = blockIdx.x;
  const int D = p.D, N = p.N, R = p.R, k = p.k;
  const int W = R + 2 * N;
  float* xs = sm;      // [D]
  float* vs = sm + D;  // [k][W]
  const IO* x = reinterpret_cast<const IO*>(p.x) + t * D;
  const WT* Wx = reinterpret_cast<const WT*>(p.W_x);
  const WT* Wdt = reinterpret_cast<const WT*>(p.W_dt);
  for (int d = threadIdx.x; d < D; d += blockDim.x) xs[d] = to_f32(x[d]);
  __syncthreads();
  for (int j = 0; j < k; ++j) {
    const int e = min(max(p.idx[t * k + j], 0), p.E - 1);  // indices outside [0, E) are clamped
    const WT* We = Wx + (size_t)e * D * W;
    for (int o = threadIdx.x; o < W; o += blockDim.x) {
      float s = 0.f;
      for (int d = 0; d < D; ++d) s = fmaf(xs[d], to_f32(We[(size_t)d * W + o]), s);
      vs[j * W + o] = s;
    }
  }
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float dt = 0.f;
    for (int j = 0; j < k; ++j) {
      const int e = min(max(p.idx[t * k + j], 0), p.E - 1);
      const float g = p.gates[t * k + j];
      const WT* We = Wdt + (size_t)e * R * D + d;
      float s = p.b_dt[(size_t)e * D + d];
      for (int r = 0; r < R; ++r) s = fmaf(vs[j * W + r], to_f32(We[(size_t)r * D]), s);
      dt = fmaf(g, s, dt);
    }
    p.delta[t * D + d] = softplus_f32(dt);
  }
  for (int n = threadIdx.x; n < N; n += blockDim.x) {
    float b = 0.f, c = 0.f;
    for (int j = 0; j < k; ++j) {
      const float g = p.gates[t * k + j];
      b = fmaf(g, vs[j * W + R + n], b);
      c = fmaf(g, vs[j * W + R + N + n], c);
    }
    p.B_mix[t * N + n] = b;
    p.C_mix[t * N + n] = c;
  }
}

template <typename IO, typename WT>
static cudaError_t launch_simt(const ProjParams& p, cudaStream_t s) {
  const size_t smem = sizeof(float) * ((size_t)p.D + (size_t)p.k * (p.R + 2 * p.N));
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(proj_simt_kernel<IO, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  proj_simt_kernel<IO, WT><<<(unsigned)p.T, 256, smem, s>>>(p);
  note_launch();
  return cudaGetLastError();
}

cudaError_t run_proj_simt(const ProjParams& p, bool io_bf16, bool w_bf16, cudaStream_t s) {
  if (io_bf16 && w_bf16) return launch_simt<__nv_bfloat16, __nv_bfloat16>(p, s);
  if (io_bf16) return launch_simt<__nv_bfloat16, float>(p, s);
  if (w_bf16) return launch_simt<float, __nv_bfloat16>(p, s);
  return launch_simt<float, float>(p, s);
}

}  // namespace swimba
