// Router of the Swimba layer: logits = x W_r (fp32 accumulation), top-k, softmax of the selected.
//
// Source: "Swimba: Switch Mamba Model Scales State Space Models", §2 "Arquitectura de Swimba"
// (es) / "Kernmechanisme van Swimba" (nl): a router gives each token mixing weights π_t over the
// active experts (top-1 or top-k).
//
// Layout (global-memory variant, used when W_r does not fit in shared memory): one warp routes TOK
// consecutive tokens. Lanes stride over the channel dimension in
// 16-byte chunks of x (8 bf16 or 4 fp32), so every x load is a coalesced 128-bit load and x is
// read from HBM exactly once. The TOK x E partial sums of every lane are combined with a
// butterfly of warp shuffles; then lane tt selects the experts of token t0+tt.
#include <algorithm>

#include "route.cuh"

namespace swimba {

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
  for (int tt = 0; tt < TOK; ++tt)
    if (lane == tt && t0 + tt < p.T) select_topk<EP>(acc[tt], E, p.k, p.idx + (t0 + tt) * p.k, p.gates + (t0 + tt) * p.k);
}

template <typename IO, int EP, int TOK>
__global__ void __launch_bounds__(512, 1) route_smem_kernel(RouteParams p) {
  extern __shared__ float2 Wp[];  // [EP/2][V][C]
  constexpr int V = Vec16<IO>::n;
  const int C = p.D / V;
  const int E = p.E;
  for (int q = threadIdx.x; q < (EP / 2) * p.D; q += blockDim.x) {
    const int ep = q / p.D, d = q - ep * p.D;
    const int e0 = 2 * ep, e1 = 2 * ep + 1;
    const float w0 = e0 < E ? p.W_r[(size_t)d * E + e0] : 0.f;
    const float w1 = e1 < E ? p.W_r[(size_t)d * E + e1] : 0.f;
    Wp[((size_t)ep * V + (d % V)) * C + d / V] = make_float2(w0, w1);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const IO* x = reinterpret_cast<const IO*>(p.x);
  for (int64_t grp = (int64_t)blockIdx.x * nwarps + (threadIdx.x >> 5); grp * TOK < p.T; grp += (int64_t)gridDim.x * nwarps) {
    const int64_t t0 = grp * TOK;
    float2 acc[TOK][EP / 2];
#pragma unroll
    for (int tt = 0; tt < TOK; ++tt)
#pragma unroll
      for (int e = 0; e < EP / 2; ++e) acc[tt][e] = make_float2(0.f, 0.f);
    // x chunks of the next iteration are loaded while the current one is accumulated
    uint4 xn[TOK];
#pragma unroll
    for (int tt = 0; tt < TOK; ++tt) {
      xn[tt] = make_uint4(0, 0, 0, 0);
      if (lane < C && t0 + tt < p.T) xn[tt] = __ldcs(reinterpret_cast<const uint4*>(x + (t0 + tt) * p.D) + lane);
    }
    for (int c = lane; c < C; c += 32) {
      uint4 xv[TOK];
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt) {
        xv[tt] = xn[tt];
        xn[tt] = make_uint4(0, 0, 0, 0);
        if (c + 32 < C && t0 + tt < p.T) xn[tt] = __ldcs(reinterpret_cast<const uint4*>(x + (t0 + tt) * p.D) + c + 32);
      }
      float xf[TOK][V];
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt) Vec16<IO>::unpack(xv[tt], xf[tt]);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        float2 w[EP / 2];
#pragma unroll
        for (int e = 0; e < EP / 2; ++e) w[e] = Wp[((size_t)e * V + i) * C + c];
#pragma unroll
        for (int tt = 0; tt < TOK; ++tt) {
          const float2 xx = make_float2(xf[tt][i], xf[tt][i]);
#pragma unroll
          for (int e = 0; e < EP / 2; ++e) acc[tt][e] = __ffma2_rn(xx, w[e], acc[tt][e]);
        }
      }
    }
    float a[TOK][EP];
#pragma unroll
    for (int tt = 0; tt < TOK; ++tt)
#pragma unroll
      for (int e = 0; e < EP / 2; ++e) {
        a[tt][2 * e] = acc[tt][e].x;
        a[tt][2 * e + 1] = acc[tt][e].y;
      }
#pragma unroll
    for (int tt = 0; tt < TOK; ++tt)
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        float v = a[tt][e];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        a[tt][e] = v;
      }
#pragma unroll
    for (int tt = 0; tt < TOK; ++tt)
      if (lane == tt && t0 + tt < p.T) select_topk<EP>(a[tt], E, p.k, p.idx + (t0 + tt) * p.k, p.gates + (t0 + tt) * p.k);
  }
}

// Few tokens (decode steps, short prompts): one CTA of 512 threads per TB tokens (TB = 4, 2 for
// E > 8), so every SM works even when T is a few hundred while each W_r row read from L2 serves TB
// tokens. The threads split the channels in 16-byte chunks of x (one chunk each at D = 4096
// bf16); for each chunk a thread loads the TB tokens' x, then the chunk's W_r rows in groups (all
// loads of a group issued before its multiply-adds), and accumulates the E partial logits of every
// token; per token a shuffle butterfly and a shared-memory pass over the warps reduce them (in the
// same order for every TB, so the logits do not depend on it), and one thread per token selects and
// normalises its experts.
constexpr int kSmallThreads = 512;  // one 16-byte chunk of x per thread at D = 4096 (bf16)

template <typename IO, int EP, int TB>
__global__ void __launch_bounds__(kSmallThreads, 1) route_small_kernel(RouteParams p) {
  constexpr int V = Vec16<IO>::n;
  constexpr int kWarps = kSmallThreads / 32;
  constexpr int VG = 32 / EP < V ? 32 / EP : V;  // W_r rows per load group: at most 32 registers
  __shared__ float part[kWarps][TB][EP];
  __shared__ float logit[TB][EP];
  const int64_t t0 = (int64_t)blockIdx.x * TB;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_trigger();
  pdl_wait();  // x may come from the kernel before
  float acc[TB][EP];
#pragma unroll
  for (int tb = 0; tb < TB; ++tb)
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[tb][e] = 0.f;
  const bool vec = (p.E & 3) == 0;  // W_r rows of 16-byte multiples: float4 loads
  for (int c = threadIdx.x; c < p.D / V; c += kSmallThreads) {
    float xf[TB][V];
#pragma unroll
    for (int tb = 0; tb < TB; ++tb) {
      const int64_t t = t0 + tb < p.T ? t0 + tb : p.T - 1;  // past the end: a repeat, not stored
      Vec16<IO>::unpack(__ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.x) + t * p.D) + c),
                        xf[tb]);
    }
    if (vec) {
#pragma unroll
      for (int v0 = 0; v0 < V; v0 += VG) {
        float4 w4[VG][EP / 4];
#pragma unroll
        for (int v = 0; v < VG; ++v)
#pragma unroll
          for (int q = 0; q < EP / 4; ++q)
            w4[v][q] = 4 * q < p.E
                           ? __ldg(reinterpret_cast<const float4*>(p.W_r + (size_t)(c * V + v0 + v) * p.E) + q)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int tb = 0; tb < TB; ++tb)
#pragma unroll
          for (int v = 0; v < VG; ++v)
#pragma unroll
            for (int q = 0; q < EP / 4; ++q) {
              acc[tb][4 * q] = fmaf(xf[tb][v0 + v], w4[v][q].x, acc[tb][4 * q]);
              acc[tb][4 * q + 1] = fmaf(xf[tb][v0 + v], w4[v][q].y, acc[tb][4 * q + 1]);
              acc[tb][4 * q + 2] = fmaf(xf[tb][v0 + v], w4[v][q].z, acc[tb][4 * q + 2]);
              acc[tb][4 * q + 3] = fmaf(xf[tb][v0 + v], w4[v][q].w, acc[tb][4 * q + 3]);
            }
      }
    } else {
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const float* w = p.W_r + (size_t)(c * V + v) * p.E;
#pragma unroll
        for (int e = 0; e < EP; ++e)
          if (e < p.E) {
            const float we = __ldg(w + e);
#pragma unroll
            for (int tb = 0; tb < TB; ++tb) acc[tb][e] = fmaf(xf[tb][v], we, acc[tb][e]);
          }
      }
    }
  }
#pragma unroll
  for (int tb = 0; tb < TB; ++tb)
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      float a = acc[tb][e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) part[warp][tb][e] = a;
    }
  __syncthreads();
  if (threadIdx.x < TB * EP) {
    const int tb = threadIdx.x / EP, e = threadIdx.x % EP;
    float a = 0.f;
    for (int w = 0; w < kWarps; ++w) a += part[w][tb][e];
    logit[tb][e] = a;
  }
  __syncthreads();
  if (threadIdx.x < TB && t0 + threadIdx.x < p.T) {
    const int tb = threadIdx.x;
    float l[EP];
#pragma unroll
    for (int e = 0; e < EP; ++e) l[e] = logit[tb][e];
    const int64_t t = t0 + tb;
    select_topk<EP>(l, p.E, p.k, p.idx + t * p.k, p.gates + t * p.k);
  }
}

template <typename IO, int EP, int TOK>
static cudaError_t launch_route(const RouteParams& p, cudaStream_t s) {
  constexpr int V = Vec16<IO>::n;
  const size_t smem = sizeof(float2) * (EP / 2) * (size_t)p.D;
  (void)V;
  if (p.T <= kSmallT) {
    constexpr int TB = EP <= 8 ? 4 : 2;
    const cudaError_t e =
        launch_pdl(route_small_kernel<IO, EP, TB>, dim3((unsigned)((p.T + TB - 1) / TB)), dim3(kSmallThreads), 0, s, p);
    if (e != cudaSuccess) return e;
  } else if (smem <= 160 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(route_smem_kernel<IO, EP, TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t groups = (p.T + TOK - 1) / TOK;
    const int64_t blocks = std::min<int64_t>(sms, (groups + 15) / 16);
    route_smem_kernel<IO, EP, TOK><<<(unsigned)blocks, 512, smem, s>>>(p);
  } else {
    const int64_t warps = (p.T + TOK - 1) / TOK;
    const int64_t blocks = (warps + 3) / 4;
    route_kernel<IO, EP, TOK><<<(unsigned)blocks, 128, 0, s>>>(p);
  }
  note_launch();
  return cudaGetLastError();
}

template <typename IO>
static cudaError_t route_dispatch(const RouteParams& p, cudaStream_t s) {
  if (p.E <= 4) return launch_route<IO, 4, 4>(p, s);
  if (p.E <= 8) return launch_route<IO, 8, 4>(p, s);
  return launch_route<IO, 16, 2>(p, s);
}

cudaError_t run_route(const void* x, bool io_bf16, const float* W_r, int32_t* idx, float* gates, int64_t T,
                      int D, int E, int k, cudaStream_t s) {
  RouteParams p{x, W_r, idx, gates, T, D, E, k};
  if (T > kSmallT && route_tc_supported(io_bf16, D, E, k)) return run_route_tc(p, s);
  return io_bf16 ? route_dispatch<__nv_bfloat16>(p, s) : route_dispatch<float>(p, s);
}

}  // namespace swimba
