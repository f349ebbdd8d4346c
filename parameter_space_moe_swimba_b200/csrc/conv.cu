// Causal depthwise convolution over time followed by SiLU: the step between the block's
// in-projection and the Swimba layer ("Mamba y las SSMs: el retorno del estado persistente",
// section "Mamba", Figura 3: the convolution and the nonlinearity on the SSM branch of the block).
//
//   p = [conv_state_in ; x_pre] along time (state: the W-1 inputs before the first token, zeros
//   when absent);  c[t, d] = b[d] + sum_{i<W} w[d, i] p[t + i, d];  x = SiLU(c);
//   conv_state_out = the last W-1 rows of p.
//
// The kernel is bound by HBM (it reads x_pre and writes x once, 2 io bytes per channel-token), so
// it is built for coalesced accesses and many warps in flight: a thread owns 8 bytes of channels
// (4 bf16 or 2 fp32) and a run of kConvRun consecutive tokens of one sequence, keeps the last W-1
// inputs of its channels in registers, and keeps the next kConvUnroll rows in flight while it
// computes the current kConvUnroll (packed fp32x2 arithmetic, MUFU exp2 and reciprocal for the
// SiLU). A warp covers 256 contiguous bytes of a token row. The kernel interleaves a stream from
// HBM with 2 MUFU operations per element; with 16-byte chunks per thread the register footprint
// left too few warps per SM to overlap the two. The W-1 rows before a run are read
// again by the run's thread (L2 hits: the neighbouring run's CTA reads them at about the same time).
#include "conv.cuh"

namespace swimba {
namespace {

constexpr int kConvThreads = 128;
constexpr int kConvRun = 32;    // tokens per thread
constexpr int kConvUnroll = 2;  // rows in flight per thread (the next batch, while this one computes)

__device__ __forceinline__ uint2 ld_stream(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// A thread owns one 8-byte chunk of channels (4 bf16 or 2 fp32), computed as fp32x2 pairs.
template <typename IO>
struct Chunk {
  static constexpr int n = 8 / sizeof(IO);  // channels
  static constexpr int pairs = n / 2;
};

__device__ __forceinline__ void unpack2(const uint2& u, float2 (&f)[2], __nv_bfloat16*) {
  f[0] = make_float2(bf16lo(u.x), bf16hi(u.x));
  f[1] = make_float2(bf16lo(u.y), bf16hi(u.y));
}
__device__ __forceinline__ void unpack2(const uint2& u, float2 (&f)[1], float*) {
  f[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
}
__device__ __forceinline__ uint2 pack2(const float2 (&f)[2], __nv_bfloat16*) {
  const __nv_bfloat162 a = __float22bfloat162_rn(f[0]), b = __float22bfloat162_rn(f[1]);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}
__device__ __forceinline__ uint2 pack2(const float2 (&f)[1], float*) {
  return make_uint2(__float_as_uint(f[0].x), __float_as_uint(f[0].y));
}

// One output row of the thread's channels from the window (W-1 older inputs) and the current input:
// c = b + sum_i w_i p_i, then SiLU(c) = c / (1 + 2^{-c log2 e}) (MUFU exp2 and reciprocal).
template <typename IO, int W>
__device__ __forceinline__ uint2 conv_row(const float2 (&w)[W][Chunk<IO>::pairs], const float2 (&bias)[Chunk<IO>::pairs],
                                          const float2 (&win)[W > 1 ? W - 1 : 1][Chunk<IO>::pairs],
                                          const float2 (&cur)[Chunk<IO>::pairs]) {
  constexpr int P = Chunk<IO>::pairs;
  const float2 kNegLog2e = make_float2(-kLog2e, -kLog2e), kOne = make_float2(1.f, 1.f);
  float2 o[P];
#pragma unroll
  for (int q = 0; q < P; ++q) {
    float2 c = bias[q];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) c = __ffma2_rn(w[i][q], win[i][q], c);
    c = __ffma2_rn(w[W - 1][q], cur[q], c);
    const float2 a = __fmul2_rn(c, kNegLog2e);
    const float2 d = __fadd2_rn(make_float2(ex2_approx(a.x), ex2_approx(a.y)), kOne);
    float2 r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(d.x));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(d.y));
    o[q] = __fmul2_rn(c, r);
  }
  return pack2(o, static_cast<IO*>(nullptr));
}

template <typename IO, int W>
__global__ void __launch_bounds__(kConvThreads, 8) conv1d_fwd_kernel(const ConvParams p) {
  constexpr int V = Chunk<IO>::n;
  constexpr int P = Chunk<IO>::pairs;
  constexpr int WH = W > 1 ? W - 1 : 1;
  const int groups = p.D / V;
  const int gblocks = (groups + kConvThreads - 1) / kConvThreads;
  const int64_t unit = blockIdx.x / gblocks;  // (sequence, run)
  const int grp = (int)(blockIdx.x - unit * gblocks) * kConvThreads + threadIdx.x;
  if (grp >= groups) return;
  const int64_t runs = (p.L + kConvRun - 1) / kConvRun;
  const int64_t b = unit / runs;
  const int64_t t0 = (unit - b * runs) * kConvRun;
  const int nt = (int)(p.L - t0 < kConvRun ? p.L - t0 : (int64_t)kConvRun);
  const int c0 = grp * V;
  IO* const tag = nullptr;

  const IO* xp = static_cast<const IO*>(p.x_pre) + (size_t)b * p.L * p.D + c0;
  IO* xo = static_cast<IO*>(p.x) + (size_t)b * p.L * p.D + c0;
  const IO* st_in = p.state_in ? static_cast<const IO*>(p.state_in) + (size_t)b * WH * p.D + c0 : nullptr;

  // rows t0 + tb .. t0 + tb + kConvUnroll - 1 into r (rows past the run are not read)
  auto load_batch = [&](uint2 (&r)[kConvUnroll], int tb) {
#pragma unroll
    for (int u = 0; u < kConvUnroll; ++u)
      if (tb + u < nt) r[u] = ld_stream(xp + (t0 + tb + u) * p.D);
  };
  uint2 ra[kConvUnroll], rb[kConvUnroll];
  load_batch(ra, 0);  // requested before anything else

  // window: inputs of tokens t0 - W + 1 .. t0 - 1 (oldest first)
  float2 win[WH][P];
#pragma unroll
  for (int i = 0; i < W - 1; ++i) {
    const int64_t r = t0 - (W - 1) + i;
    if (r >= 0) {
      unpack2(ld_stream(xp + r * p.D), win[i], tag);
    } else if (st_in != nullptr) {
      unpack2(ld_stream(st_in + (W - 1 + r) * p.D), win[i], tag);
    } else {
#pragma unroll
      for (int q = 0; q < P; ++q) win[i][q] = make_float2(0.f, 0.f);
    }
  }
  float2 w[W][P], bias[P];
#pragma unroll
  for (int q = 0; q < P; ++q) {
    bias[q] = make_float2(__ldg(p.conv_b + c0 + 2 * q), __ldg(p.conv_b + c0 + 2 * q + 1));
#pragma unroll
    for (int i = 0; i < W; ++i)
      w[i][q] = make_float2(__ldg(p.conv_w + (size_t)(c0 + 2 * q) * W + i), __ldg(p.conv_w + (size_t)(c0 + 2 * q + 1) * W + i));
  }

  auto compute_batch = [&](const uint2 (&r)[kConvUnroll], int tb) {
#pragma unroll
    for (int u = 0; u < kConvUnroll; ++u) {
      if (tb + u < nt) {
        float2 cur[P];
        unpack2(r[u], cur, tag);
        *reinterpret_cast<uint2*>(xo + (t0 + tb + u) * p.D) = conv_row<IO, W>(w, bias, win, cur);
#pragma unroll
        for (int i = 0; i + 1 < W - 1; ++i)
#pragma unroll
          for (int q = 0; q < P; ++q) win[i][q] = win[i + 1][q];
        if (W > 1) {
#pragma unroll
          for (int q = 0; q < P; ++q) win[WH - 1][q] = cur[q];
        }
      }
    }
  };

  // each batch is computed while the next one's rows are in flight
#pragma unroll 1
  for (int tb = 0; tb < nt; tb += 2 * kConvUnroll) {
    load_batch(rb, tb + kConvUnroll);
    compute_batch(ra, tb);
    load_batch(ra, tb + 2 * kConvUnroll);
    compute_batch(rb, tb + kConvUnroll);
  }

  if (p.state_out != nullptr && t0 + nt == p.L) {
    IO* so = static_cast<IO*>(p.state_out) + (size_t)b * WH * p.D + c0;
#pragma unroll
    for (int i = 0; i < W - 1; ++i) *reinterpret_cast<uint2*>(so + (size_t)i * p.D) = pack2(win[i], tag);
  }
}

// Decode: one token per sequence, the state [B, W-1, D] read and shifted in place. One thread per
// (sequence, 16 bytes of channels); it reads every element it overwrites, so in-place is safe.
template <typename IO, int W>
__global__ void __launch_bounds__(kConvThreads) conv1d_step_kernel(const ConvParams p) {
  constexpr int V = Chunk<IO>::n;
  constexpr int P = Chunk<IO>::pairs;
  constexpr int WH = W > 1 ? W - 1 : 1;
  const int groups = p.D / V;
  const int64_t gid = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
  if (gid >= p.Bsz * groups) return;
  const int64_t b = gid / groups;
  const int c0 = (int)(gid - b * groups) * V;
  IO* const tag = nullptr;
  float2 w[W][P], bias[P];
#pragma unroll
  for (int q = 0; q < P; ++q) {
    bias[q] = make_float2(__ldg(p.conv_b + c0 + 2 * q), __ldg(p.conv_b + c0 + 2 * q + 1));
#pragma unroll
    for (int i = 0; i < W; ++i)
      w[i][q] = make_float2(__ldg(p.conv_w + (size_t)(c0 + 2 * q) * W + i), __ldg(p.conv_w + (size_t)(c0 + 2 * q + 1) * W + i));
  }
  IO* st = static_cast<IO*>(p.state_out) + (size_t)b * WH * p.D + c0;
  float2 win[WH][P], cur[P];
#pragma unroll
  for (int i = 0; i < W - 1; ++i) unpack2(*reinterpret_cast<const uint2*>(st + (size_t)i * p.D), win[i], tag);
  unpack2(*reinterpret_cast<const uint2*>(static_cast<const IO*>(p.x_pre) + (size_t)b * p.D + c0), cur, tag);
  *reinterpret_cast<uint2*>(static_cast<IO*>(p.x) + (size_t)b * p.D + c0) = conv_row<IO, W>(w, bias, win, cur);
  if (W > 1) {
#pragma unroll
    for (int i = 0; i + 1 < W - 1; ++i) *reinterpret_cast<uint2*>(st + (size_t)i * p.D) = pack2(win[i + 1], tag);
    *reinterpret_cast<uint2*>(st + (size_t)(WH - 1) * p.D) = pack2(cur, tag);
  }
}

template <typename IO, int W>
cudaError_t launch_conv(const ConvParams& p, bool step, cudaStream_t s) {
  constexpr int V = Chunk<IO>::n;
  const int groups = p.D / V;
  if (step) {
    const int64_t blocks = (p.Bsz * groups + kConvThreads - 1) / kConvThreads;
    conv1d_step_kernel<IO, W><<<(unsigned)blocks, kConvThreads, 0, s>>>(p);
  } else {
    const int64_t gblocks = (groups + kConvThreads - 1) / kConvThreads;
    const int64_t runs = (p.L + kConvRun - 1) / kConvRun;
    conv1d_fwd_kernel<IO, W><<<(unsigned)(p.Bsz * runs * gblocks), kConvThreads, 0, s>>>(p);
  }
  note_launch();
  return cudaGetLastError();
}

template <typename IO>
cudaError_t dispatch_width(const ConvParams& p, bool step, cudaStream_t s) {
  switch (p.W) {
    case 1: return launch_conv<IO, 1>(p, step, s);
    case 2: return launch_conv<IO, 2>(p, step, s);
    case 3: return launch_conv<IO, 3>(p, step, s);
    case 4: return launch_conv<IO, 4>(p, step, s);
    case 5: return launch_conv<IO, 5>(p, step, s);
    case 6: return launch_conv<IO, 6>(p, step, s);
    case 7: return launch_conv<IO, 7>(p, step, s);
    case 8: return launch_conv<IO, 8>(p, step, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t run_conv1d(const ConvParams& p, bool io_bf16, bool step, cudaStream_t s) {
  if (p.Bsz <= 0 || p.L <= 0) return cudaSuccess;
  return io_bf16 ? dispatch_width<__nv_bfloat16>(p, step, s) : dispatch_width<float>(p, step, s);
}

}  // namespace swimba
