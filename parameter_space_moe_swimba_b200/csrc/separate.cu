// The "MoE of separate SSMs" that the Swimba pages set against Swimba: every expert keeps its own
// state trajectory and runs its own recurrent update; only the outputs are mixed. It is built here
// as the measured side of Teorema 2 (the recurrence cost of Swimba's single mixed recurrence does
// not grow with the experts, the separate design's does).
//
// Sources: "Swimba: Switch Mamba Model Scales State Space Models", Spanish summary §2 "Distinción de
// Diseños", Dutch "Methodologie", French "Distinction des deux designs MoE-SSM" (one state
// trajectory and one recurrent update per expert; compute and memory grow with the experts); §3
// "Contribuciones", Teorema 2.
//
// Definition (the pages give no equations; the plainest reading): expert e has its own state
// h^(e) [B, D, N]. At token t the k active experts e_j advance their own states with their own,
// unmixed streams and their own transition,
//     Δ^j = softplus(dt^j);  h^(e_j) = exp(Δ^j A^{e_j}) h^(e_j) + Δ^j B^j x_t,
// the other experts' states stay as they are, and
//     y_t = Σ_j g_j C^j · h^(e_j) + D_skip x_t;  out_t = y_t SiLU(z_t).
//
// Kernels:
//  * separate_proj_kernel: the per-slot streams Δ^j, B^j, C^j (SIMT, one CTA per token; the
//    expert projections as in the mixed path, but nothing is mixed).
//  * separate_scan_fast: bf16 x/z/out, N = 16, k <= 2, E <= 8, D % 16 == 0. The lane layout of the
//    fast Swimba scan (a warp = 16 channels of one sequence; a lane = 2 channels x 4 states, packed
//    f32x2) with every expert's A rows AND every expert's state in the warp's tensor-memory window
//    (A at columns 8e, h^(e) at columns 8E + 8e): per token and slot one tcgen05.ld of the expert's
//    A rows, one of its state, the update, one tcgen05.st of the state back.
//  * separate_scan_generic: any other shape, one thread per (sequence, channel), every expert's
//    state of the channel in local memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "proj.cuh"
#include "scan.cuh"
#include "sm100.cuh"

namespace swimba {

using namespace sm100;

// ---- per-slot projection -------------------------------------------------------------------------
template <typename IO, typename WT>
__global__ void __launch_bounds__(256) separate_proj_kernel(ProjParams p, float* delta_j, float* B_j, float* C_j) {
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
  for (int j = 0; j < k; ++j) {
    const int e = min(max(p.idx[t * k + j], 0), p.E - 1);
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      const WT* We = Wdt + (size_t)e * R * D + d;
      float s = p.b_dt[(size_t)e * D + d];
      for (int r = 0; r < R; ++r) s = fmaf(vs[j * W + r], to_f32(We[(size_t)r * D]), s);
      delta_j[(t * k + j) * D + d] = softplus_f32(s);
    }
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
      B_j[(t * k + j) * N + n] = vs[j * W + R + n];
      C_j[(t * k + j) * N + n] = vs[j * W + R + N + n];
    }
  }
}

struct SeparateParams {
  const void* x;         // [B, L, D] io
  const void* z;         // [B, L, D] io
  const float* delta_j;  // [B, L, k, D]
  const float* B_j;      // [B, L, k, N]
  const float* C_j;      // [B, L, k, N]
  const int32_t* idx;    // [B, L, k]
  const float* gates;    // [B, L, k]
  const float* A;        // [E, D, N]
  const float* D_skip;   // [D]
  const float* h0;       // [E, B, D, N] or null
  void* out;             // [B, L, D] io
  float* h_final;        // [E, B, D, N] or null
  float* y_pre;          // [B, L, D] or null
  void* status;
  int64_t L;
  int B, D, N, E, k;
  int units, tmem_cols;
};

// ---- generic scan: one thread per (sequence, channel) ---------------------------------------------
template <typename IO>
__global__ void __launch_bounds__(128) separate_scan_generic(SeparateParams p) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over (b, d)
  if (i >= (int64_t)p.B * p.D) return;
  const int d = (int)(i % p.D);
  const int b = (int)(i / p.D);
  float h[16][16];  // [expert][state]
  for (int e = 0; e < p.E; ++e)
    for (int n = 0; n < p.N; ++n)
      h[e][n] = p.h0 != nullptr ? p.h0[(((size_t)e * p.B + b) * p.D + d) * p.N + n] : 0.f;
  const IO* x = reinterpret_cast<const IO*>(p.x);
  const IO* z = reinterpret_cast<const IO*>(p.z);
  IO* out = reinterpret_cast<IO*>(p.out);
  for (int64_t t = 0; t < p.L; ++t) {
    const size_t tok = (size_t)b * p.L + t;
    const float xv = to_f32(x[tok * p.D + d]);
    float y = p.D_skip[d] * xv;
    for (int j = 0; j < p.k; ++j) {
      const int e = min(max(p.idx[tok * p.k + j], 0), p.E - 1);
      const float dl = p.delta_j[(tok * p.k + j) * p.D + d];
      const float* Bv = p.B_j + (tok * p.k + j) * p.N;
      const float* Cv = p.C_j + (tok * p.k + j) * p.N;
      float yj = 0.f;
      for (int n = 0; n < p.N; ++n) {
        const float a = ex2_approx(dl * p.A[((size_t)e * p.D + d) * p.N + n] * kLog2e);
        h[e][n] = fmaf(a, h[e][n], dl * Bv[n] * xv);
        yj = fmaf(Cv[n], h[e][n], yj);
      }
      y = fmaf(p.gates[tok * p.k + j], yj, y);
    }
    if (p.y_pre != nullptr) p.y_pre[tok * p.D + d] = y;
    const float zv = to_f32(z[tok * p.D + d]);
    from_f32(out[tok * p.D + d], y * zv / (1.f + __expf(-zv)));
  }
  if (p.h_final != nullptr)
    for (int e = 0; e < p.E; ++e)
      for (int n = 0; n < p.N; ++n) p.h_final[(((size_t)e * p.B + b) * p.D + d) * p.N + n] = h[e][n];
}

// ---- fast scan: every expert's A rows and state in tensor memory -----------------------------------
namespace {

constexpr int LC = 16;         // tokens per chunk
constexpr int kStages = 2;
constexpr int kCPW = 16;       // channels per warp
constexpr int kMaxWarps = 16;
constexpr int kPRow = 4 * kCPW + 4;

template <int K>
struct SepStage {
  static constexpr int X = 0;                         // bf16 [LC][16]
  static constexpr int Z = X + LC * kCPW * 2;         // bf16 [LC][16]
  static constexpr int DL = Z + LC * kCPW * 2;        // f32  [K][LC][16]
  static constexpr int B = DL + K * LC * kCPW * 4;    // f32  [LC][K][16]
  static constexpr int C = B + K * LC * 16 * 4;       // f32  [LC][K][16]
  static constexpr int META = C + K * LC * 16 * 4;    // int4 [LC]
  static constexpr int BYTES = META + LC * 16;
  static_assert(DL % 128 == 0 && B % 128 == 0 && C % 128 == 0 && META % 128 == 0 && BYTES % 128 == 0,
                "TMA destinations must be 128-byte aligned");
};

struct SepEpi {
  static constexpr int P = 0;                         // f32 [LC][kPRow]
  static constexpr int O = P + LC * kPRow * 4;        // bf16 [2][LC][16]
  static constexpr int BYTES = O + 2 * LC * kCPW * 2;
};

template <int K>
constexpr int sep_warp_bytes() { return kStages * SepStage<K>::BYTES + SepEpi::BYTES; }

// TMEM columns of one warp: E x 8 for the A rows, E x 8 for the states, in 32-column granules.
__host__ __device__ constexpr int sep_cols_per_warp(int E) { return ((E * 16 + 31) / 32) * 32; }

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float2 v) {
  const __nv_bfloat162 b = __float22bfloat162_rn(v);
  return *reinterpret_cast<const uint32_t*>(&b);
}

}  // namespace

template <int K>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
    separate_scan_fast(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                       const __grid_constant__ CUtensorMap tm_dl, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_o,
                       const SeparateParams p) {
  using St = SepStage<K>;
  constexpr int WB = sep_warp_bytes<K>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  uint8_t* ring = smem + (size_t)warp * WB;
  uint8_t* epi = ring + kStages * St::BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nwarps * WB);
  uint64_t* full = bars + warp * kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + nwarps * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + nwarps * kStages) + 1;
  float* psm = reinterpret_cast<float*>(epi + SepEpi::P);

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    if (warp == 0) *abort_flag = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) +
                         (uint32_t)(warp >> 2) * (uint32_t)sep_cols_per_warp(p.E);
  const uint32_t hoff = (uint32_t)(8 * p.E);  // state columns after the A columns

  const int cp = lane >> 2, q = lane & 3;
  const int rt = lane >> 1, rc = (lane & 1) * 8;
  const int ntiles = p.D / kCPW;
  const uint32_t emax = (uint32_t)(p.E - 1);
  uint32_t phase_bits = 0;
  int ochunk = 0;
  constexpr uint32_t tx_bytes = 2 * LC * kCPW * 2 + K * LC * kCPW * 4 + 2 * K * LC * 16 * 4;
  const int u_begin = (int)((int64_t)p.units * blockIdx.x / gridDim.x);
  const int u_end = (int)((int64_t)p.units * (blockIdx.x + 1) / gridDim.x);

  for (int u = u_begin + warp; u < u_end; u += nwarps) {
    const int tile = u % ntiles;
    const int b = u / ntiles;
    const int dA = tile * kCPW + 2 * cp;
    const int nchunks = (int)((p.L + LC - 1) / LC);

    // every expert's transition rows (x log2 e) and start state into this warp's TMEM window
    for (int e = 0; e < p.E; ++e) {
      const float4 a0 = __ldg(reinterpret_cast<const float4*>(p.A + ((size_t)e * p.D + dA) * 16 + 4 * q));
      const float4 a1 = __ldg(reinterpret_cast<const float4*>(p.A + ((size_t)e * p.D + dA + 1) * 16 + 4 * q));
      const uint32_t r[8] = {__float_as_uint(a0.x * kLog2e), __float_as_uint(a1.x * kLog2e),
                             __float_as_uint(a0.y * kLog2e), __float_as_uint(a1.y * kLog2e),
                             __float_as_uint(a0.z * kLog2e), __float_as_uint(a1.z * kLog2e),
                             __float_as_uint(a0.w * kLog2e), __float_as_uint(a1.w * kLog2e)};
      tmem_st8(tbase + (uint32_t)(e * 8), r);
      float4 u0 = make_float4(0.f, 0.f, 0.f, 0.f), u1 = u0;
      if (p.h0 != nullptr) {
        const float* hs = p.h0 + (((size_t)e * p.B + b) * p.D + dA) * 16;
        u0 = *reinterpret_cast<const float4*>(hs + 4 * q);
        u1 = *reinterpret_cast<const float4*>(hs + 16 + 4 * q);
      }
      const uint32_t hr[8] = {__float_as_uint(u0.x), __float_as_uint(u1.x), __float_as_uint(u0.y),
                              __float_as_uint(u1.y), __float_as_uint(u0.z), __float_as_uint(u1.z),
                              __float_as_uint(u0.w), __float_as_uint(u1.w)};
      tmem_st8(tbase + hoff + (uint32_t)(e * 8), hr);
    }
    tmem_wait_st();
    float2 dsk[4];
    {
      const float4 d0 = __ldg(reinterpret_cast<const float4*>(p.D_skip + tile * kCPW + rc));
      const float4 d1 = __ldg(reinterpret_cast<const float4*>(p.D_skip + tile * kCPW + rc + 4));
      dsk[0] = make_float2(d0.x, d0.y);
      dsk[1] = make_float2(d0.z, d0.w);
      dsk[2] = make_float2(d1.x, d1.y);
      dsk[3] = make_float2(d1.z, d1.w);
    }

    auto load_meta = [&](int c) -> int4 {
      int4 m = make_int4(0, 0, 0, 0);
      const int64_t t = (int64_t)c * LC + lane;
      if (lane < LC && c < nchunks && t < p.L) {
        const size_t tok = (size_t)b * p.L + t;
        m.x = (int)(min((uint32_t)__ldg(p.idx + tok * K), emax) * 8u);
        m.z = __float_as_int(__ldg(p.gates + tok * K));
        if (K == 2) {
          m.y = (int)(min((uint32_t)__ldg(p.idx + tok * K + 1), emax) * 8u);
          m.w = __float_as_int(__ldg(p.gates + tok * K + 1));
        }
      }
      return m;
    };
    auto issue = [&](int c, int4 m) {
      uint8_t* st = ring + (c % kStages) * St::BYTES;
      if (lane < LC) reinterpret_cast<int4*>(st + St::META)[lane] = m;
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_smem();
        uint64_t* bar = &full[c % kStages];
        mbar_arrive_expect_tx(bar, tx_bytes);
        const int t0 = c * LC;
        tma_load_3d(st + St::X, &tm_x, bar, tile * kCPW, t0, b);
        tma_load_3d(st + St::Z, &tm_z, bar, tile * kCPW, t0, b);
        for (int j = 0; j < K; ++j)
          tma_load_3d(st + St::DL + j * LC * kCPW * 4, &tm_dl, bar, j * p.D + tile * kCPW, t0, b);
        tma_load_3d(st + St::B, &tm_b, bar, 0, t0, b);
        tma_load_3d(st + St::C, &tm_c, bar, 0, t0, b);
      }
    };

    int4 meta_next = load_meta(0);
    const int pre = nchunks < kStages ? nchunks : kStages;
    for (int c = 0; c < pre; ++c) {
      const int4 m = meta_next;
      meta_next = load_meta(c + 1);
      issue(c, m);
    }
    bool ok = true;
    int issued = pre, failed_chunk = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int sidx = c % kStages;
      if (!mbar_wait(&full[sidx], (phase_bits >> sidx) & 1u, abort_flag)) {
        ok = false;
        failed_chunk = c;
        break;
      }
      phase_bits ^= 1u << sidx;
      const uint8_t* st = ring + sidx * St::BYTES;
      const int4* meta = reinterpret_cast<const int4*>(st + St::META);
      const uint32_t* xs2 = reinterpret_cast<const uint32_t*>(st + St::X);
      const int64_t t0 = (int64_t)c * LC;
#pragma unroll 1
      for (int t = 0; t < LC; ++t) {
        const int4 m = meta[t];
        const uint32_t xw = xs2[t * (kCPW / 2) + cp];
        const float2 xv = make_float2(bf16lo(xw), bf16hi(xw));
        float2 y = f2(0.f);
#pragma unroll
        for (int j = 0; j < K; ++j) {
          const uint32_t col = (uint32_t)(j == 0 ? m.x : m.y);
          uint32_t ar[8], hr[8];
          tmem_ld8_nowait(tbase + col, ar);
          tmem_ld8_nowait(tbase + hoff + col, hr);
          const float2 dl = reinterpret_cast<const float2*>(st + St::DL + j * LC * kCPW * 4)[t * (kCPW / 2) + cp];
          const float4 bq = reinterpret_cast<const float4*>(st + St::B)[(t * K + j) * 4 + q];
          const float4 cq = reinterpret_cast<const float4*>(st + St::C)[(t * K + j) * 4 + q];
          const float2 dx = __fmul2_rn(dl, xv);
          tmem_wait_ld();
          const float bs[4] = {bq.x, bq.y, bq.z, bq.w};
          const float cs[4] = {cq.x, cq.y, cq.z, cq.w};
          float2 yj = f2(0.f);
          uint32_t hn[8];
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const float2 arg = __fmul2_rn(dl, make_float2(__uint_as_float(ar[2 * s]), __uint_as_float(ar[2 * s + 1])));
            const float2 a = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
            float2 h = make_float2(__uint_as_float(hr[2 * s]), __uint_as_float(hr[2 * s + 1]));
            h = __ffma2_rn(a, h, __fmul2_rn(dx, f2(bs[s])));
            yj = __ffma2_rn(f2(cs[s]), h, yj);
            hn[2 * s] = __float_as_uint(h.x);
            hn[2 * s + 1] = __float_as_uint(h.y);
          }
          tmem_st8(tbase + hoff + col, hn);
          if (j + 1 < K && m.x == m.y) tmem_wait_st();  // a repeated expert reads the state just written
          y = __ffma2_rn(f2(__int_as_float(j == 0 ? m.z : m.w)), yj, y);
        }
        // the next token may advance the same expert: its state must be back in TMEM first
        tmem_wait_st();
        *reinterpret_cast<float2*>(psm + t * kPRow + cp * 8 + q * 2) = y;
      }
      // readout pass: lane = (token rt, channels rc..rc+7)
      __syncwarp();
      float2 yv[4];
      {
        // channel pair i of this lane's 8 channels: (c0, c1) partials of the four state quarters
        const float4* pr = reinterpret_cast<const float4*>(psm + rt * kPRow + (rc / 2) * 8);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 a = pr[2 * i], b = pr[2 * i + 1];
          yv[i] = __fadd2_rn(__fadd2_rn(make_float2(a.x, a.y), make_float2(a.z, a.w)),
                             __fadd2_rn(make_float2(b.x, b.y), make_float2(b.z, b.w)));
        }
      }
      const uint4 xq = *reinterpret_cast<const uint4*>(st + St::X + (rt * kCPW + rc) * 2);
      const uint4 zq = *reinterpret_cast<const uint4*>(st + St::Z + (rt * kCPW + rc) * 2);
      const uint32_t xw4[4] = {xq.x, xq.y, xq.z, xq.w}, zw4[4] = {zq.x, zq.y, zq.z, zq.w};
      uint32_t packed[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 xf = make_float2(bf16lo(xw4[i]), bf16hi(xw4[i]));
        const float2 zf = make_float2(bf16lo(zw4[i]), bf16hi(zw4[i]));
        yv[i] = __ffma2_rn(dsk[i], xf, yv[i]);
        const float2 hz = __fmul2_rn(zf, f2(0.5f));
        const float2 th = make_float2(tanh_approx(hz.x), tanh_approx(hz.y));
        packed[i] = pack_bf16x2(__fmul2_rn(yv[i], __ffma2_rn(hz, th, hz)));
      }
      if (p.y_pre != nullptr && t0 + rt < p.L) {
        float4* yp = reinterpret_cast<float4*>(p.y_pre + ((size_t)b * p.L + t0 + rt) * p.D + tile * kCPW + rc);
        yp[0] = make_float4(yv[0].x, yv[0].y, yv[1].x, yv[1].y);
        yp[1] = make_float4(yv[2].x, yv[2].y, yv[3].x, yv[3].y);
      }
      uint8_t* obuf = epi + SepEpi::O + (ochunk & 1) * (LC * kCPW * 2);
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      *reinterpret_cast<uint4*>(obuf + (rt * kCPW + rc) * 2) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(&tm_o, obuf, tile * kCPW, (int)t0, b);
        bulk_commit();
      }
      ++ochunk;
      __syncwarp();
      if (c + kStages < nchunks) {
        const int4 mm = meta_next;
        meta_next = load_meta(c + kStages + 1);
        issue(c + kStages, mm);
        ++issued;
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 41, blockIdx.x, u);
      for (int c = failed_chunk; c < issued; ++c) {
        const int sidx = c % kStages;
        const uint64_t w0 = globaltimer_ns();
        while (!mbar_try_wait(&full[sidx], (phase_bits >> sidx) & 1u) && globaltimer_ns() - w0 < kWaitLimitNs) {
        }
        phase_bits ^= 1u << sidx;
      }
      break;
    }
    if (p.h_final != nullptr) {
      for (int e = 0; e < p.E; ++e) {
        uint32_t hr[8];
        tmem_ld8_nowait(tbase + hoff + (uint32_t)(e * 8), hr);
        tmem_wait_ld();
        float* ho = p.h_final + (((size_t)e * p.B + b) * p.D + dA) * 16;
        *reinterpret_cast<float4*>(ho + 4 * q) = make_float4(__uint_as_float(hr[0]), __uint_as_float(hr[2]),
                                                             __uint_as_float(hr[4]), __uint_as_float(hr[6]));
        *reinterpret_cast<float4*>(ho + 16 + 4 * q) = make_float4(__uint_as_float(hr[1]), __uint_as_float(hr[3]),
                                                                  __uint_as_float(hr[5]), __uint_as_float(hr[7]));
      }
    }
    __syncwarp();
  }
  if (lane == 0) bulk_wait<0>();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, (uint32_t)p.tmem_cols);
  }
}

// ---- host ------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 sep_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

bool sep_map3(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int64_t inner, int64_t L,
              int64_t B, int box_inner) {
  auto fn = sep_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t str[2] = {(cuuint64_t)(inner * esize), (cuuint64_t)(inner * L * esize)};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)LC, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int K>
cudaError_t launch_separate_fast(SeparateParams p, cudaStream_t s) {
  CUtensorMap tx, tz, td, tb, tc, to;
  if (!sep_map3(&tx, p.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.D, p.L, p.B, kCPW) ||
      !sep_map3(&tz, p.z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.D, p.L, p.B, kCPW) ||
      !sep_map3(&td, p.delta_j, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (int64_t)K * p.D, p.L, p.B, kCPW) ||
      !sep_map3(&tb, p.B_j, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, K * 16, p.L, p.B, K * 16) ||
      !sep_map3(&tc, p.C_j, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, K * 16, p.L, p.B, K * 16) ||
      !sep_map3(&to, p.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.D, p.L, p.B, kCPW))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int WB = sep_warp_bytes<K>();
  const int win = sep_cols_per_warp(p.E);
  int smem_optin = 0;
  cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int wsmem = std::max(1, (smem_optin - 256) / (WB + kStages * 8));
  const int wmax = std::max(1, std::min({kMaxWarps, wsmem, 4 * (512 / win)}));
  p.units = p.B * (p.D / kCPW);
  int ctas = std::max(1, std::min(sms, p.units));
  const int warps = std::min(wmax, (p.units + ctas - 1) / ctas);
  const int need = ((warps + 3) / 4) * win;
  p.tmem_cols = 32;
  while (p.tmem_cols < need) p.tmem_cols *= 2;
  const size_t smem = 128 + (size_t)warps * (WB + kStages * 8) + 16;
  auto kern = separate_scan_fast<K>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<ctas, warps * 32, smem, s>>>(tx, tz, td, tb, tc, to, p);
  note_launch();
  return cudaGetLastError();
}

template <typename IO, typename WT>
cudaError_t launch_separate_proj(const ProjParams& p, float* dj, float* bj, float* cj, cudaStream_t s) {
  const size_t smem = sizeof(float) * ((size_t)p.D + (size_t)p.k * (p.R + 2 * p.N));
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(separate_proj_kernel<IO, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  separate_proj_kernel<IO, WT><<<(unsigned)p.T, 256, smem, s>>>(p, dj, bj, cj);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool separate_fast_supported(bool io_bf16, int N, int k, int E, int D) {
  return io_bf16 && N == 16 && (k == 1 || k == 2) && E >= 1 && E <= 8 && D % kCPW == 0;
}

cudaError_t run_separate_proj(const ProjParams& p, bool io_bf16, bool w_bf16, float* dj, float* bj, float* cj,
                              cudaStream_t s) {
  if (io_bf16 && w_bf16) return launch_separate_proj<__nv_bfloat16, __nv_bfloat16>(p, dj, bj, cj, s);
  if (io_bf16) return launch_separate_proj<__nv_bfloat16, float>(p, dj, bj, cj, s);
  if (w_bf16) return launch_separate_proj<float, __nv_bfloat16>(p, dj, bj, cj, s);
  return launch_separate_proj<float, float>(p, dj, bj, cj, s);
}

cudaError_t run_separate_scan(const SeparateParams& p, bool io_bf16, cudaStream_t s) {
  if (separate_fast_supported(io_bf16, p.N, p.k, p.E, p.D))
    return p.k == 1 ? launch_separate_fast<1>(p, s) : launch_separate_fast<2>(p, s);
  const int64_t n = (int64_t)p.B * p.D;
  const unsigned grid = (unsigned)((n + 127) / 128);
  if (io_bf16)
    separate_scan_generic<__nv_bfloat16><<<grid, 128, 0, s>>>(p);
  else
    separate_scan_generic<float><<<grid, 128, 0, s>>>(p);
  note_launch();
  return cudaGetLastError();
}

// Argument marshalling for the C ABI (api.cu owns validation).
cudaError_t separate_scan_entry(const void* x, const void* z, const float* dj, const float* bj, const float* cj,
                                const int32_t* idx, const float* gates, const float* A, const float* D_skip,
                                const float* h0, void* out, float* h_final, float* y_pre, void* status, int64_t L,
                                int B, int D, int N, int E, int k, bool io_bf16, cudaStream_t s) {
  SeparateParams p{x, z, dj, bj, cj, idx, gates, A, D_skip, h0, out, h_final, y_pre, status, L, B, D, N, E, k, 0, 0};
  return run_separate_scan(p, io_bf16, s);
}

}  // namespace swimba
