// Backward pass of the selective scan (the layer's single recurrence, Euler injection).
//
// Source of the forward it differentiates: "Swimba: Switch Mamba Model Scales State Space Models",
// §2 "Arquitectura de Swimba" (one recurrence over the gate-mixed parameters) and "Mamba y las SSMs:
// el retorno del estado persistente", "Mamba" (ā = exp(Δ A)); the pages train Swimba-14B (Dutch
// summary, "Resultaten") without giving training details, so this is the exact gradient of the
// forward, reverse mode:
//   dy_t = G_t SiLU(z_t),  dz_t = G_t y_t SiLU'(z_t)
//   λ_t = C_t dy_t + a_{t+1} λ_{t+1}                        (per channel d and state n, reverse in t)
//   dC_t[n] = Σ_d dy_t h_t,  dB_t[n] = Σ_d λ_t Δ_t x_t,  dx_t = D dy_t + Δ_t Σ_n λ_t B_t
//   dΔ_t = Σ_n λ_t (A_t a_t h_{t-1} + B_t x_t)
//   dA_t = λ_t Δ_t a_t h_{t-1} -> dA^e += g_j dA_t,  dg_j = Σ_{d,n} dA_t A^{e_j};   dD = Σ_t dy_t x_t
//   dh0 = a_0 λ_0.
//
// Three kernels:
//   ckpt    the forward recurrence, writing the state at the start of every chunk of 16 tokens;
//   bwd     a CTA owns 64 channels of one sequence (thread = channel x quarter of the 16 states,
//           the A rows of every expert for its channels in shared memory); it walks the chunks
//           from the last: recomputes the chunk's 16 states per thread into registers from its
//           checkpoint (writing dz on the way), then runs the adjoint back through the chunk. The
//           per-token sums over channels (dB, dC, dgates) are reduced inside the warp by shuffles,
//           across the CTA's warps in shared memory, and written as one partial per channel tile;
//           dA accumulates per thread in shared memory, dD in a register;
//   reduce  sums the partials over channel tiles (dB, dC, dgates) and sequences (dA, dD) in a fixed
//           order, so the result does not depend on scheduling.
// Shapes: N <= 16, any k <= E <= 16, io fp32 or bf16.
#include "common.cuh"
#include "scan.cuh"

namespace swimba {

namespace {

constexpr int kBwdCh = 64;    // channels per CTA
constexpr int kBwdLc = 16;    // tokens per checkpoint chunk
constexpr int kBwdWarps = 8;  // 256 threads

__device__ __forceinline__ float sigmoid_f(float v) { return 1.f / (1.f + ex2_approx(-v * kLog2e)); }

// The A rows of every expert for the CTA's channels: As[e][c][16], zero beyond N.
__device__ __forceinline__ void load_a_rows(float* As, const float* A, int E, int D, int N, int d0, int nc) {
  for (int i = threadIdx.x; i < E * kBwdCh * 16; i += blockDim.x) {
    const int e = i / (kBwdCh * 16), r = i % (kBwdCh * 16), c = r / 16, n = r % 16;
    As[i] = (c < nc && n < N) ? A[((size_t)e * D + d0 + c) * N + n] : 0.f;
  }
}

}  // namespace

template <typename IO>
__global__ void __launch_bounds__(256) scan_bwd_ckpt_kernel(ScanBwdParams p) {
  extern __shared__ float As[];
  const int tid = threadIdx.x, c = tid >> 2, q = tid & 3;
  const int tiles = (p.D + kBwdCh - 1) / kBwdCh;
  const int tile = blockIdx.x % tiles, b = blockIdx.x / tiles;
  const int d0 = tile * kBwdCh, nc = min(kBwdCh, p.D - d0);
  load_a_rows(As, p.A, p.E, p.D, p.N, d0, nc);
  __syncthreads();
  if (c >= nc) return;  // no barrier below
  const int d = d0 + c;
  float h[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int n = 4 * q + s;
    h[s] = (p.h0 != nullptr && n < p.N) ? p.h0[((size_t)b * p.D + d) * p.N + n] : 0.f;
  }
  for (int64_t t = 0; t < p.L; ++t) {
    if (t % kBwdLc == 0) {
      float* ck = p.ckpt + (((size_t)b * p.nck + t / kBwdLc) * p.D + d) * p.N;
#pragma unroll
      for (int s = 0; s < 4; ++s)
        if (4 * q + s < p.N) ck[4 * q + s] = h[s];
    }
    const size_t bt = (size_t)b * p.L + t;
    const float dl = p.delta[bt * p.D + d];
    const float xv = to_f32(reinterpret_cast<const IO*>(p.x)[bt * p.D + d]);
    float at[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < p.k; ++j) {
      const int e = min(max(p.idx[bt * p.k + j], 0), p.E - 1);
      const float g = p.gates[bt * p.k + j];
      const float4 a4 = reinterpret_cast<const float4*>(As)[(e * kBwdCh + c) * 4 + q];
      at[0] = fmaf(g, a4.x, at[0]);
      at[1] = fmaf(g, a4.y, at[1]);
      at[2] = fmaf(g, a4.z, at[2]);
      at[3] = fmaf(g, a4.w, at[3]);
    }
    const float c0 = dl * kLog2e, dx = dl * xv;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int n = 4 * q + s;
      const float bn = n < p.N ? p.B_mix[bt * p.N + n] : 0.f;
      h[s] = fmaf(ex2_approx(c0 * at[s]), h[s], dx * bn);
    }
  }
}

template <typename IO>
__global__ void __launch_bounds__(256, 2) scan_bwd_kernel(ScanBwdParams p) {
  extern __shared__ float smem[];
  float* As = smem;                                  // [E][64][16]
  float* dAacc = As + p.E * kBwdCh * 16;             // [E][256 threads][4]
  float* red = dAacc + p.E * 256 * 4;                // [8 warps][16 tokens][rw]
  const int rw = 2 * p.N + p.k;                      // per token: dB[N], dC[N], dgates[k]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, c = tid >> 2, q = tid & 3;
  const int tiles = (p.D + kBwdCh - 1) / kBwdCh;
  const int tile = blockIdx.x % tiles, b = blockIdx.x / tiles;
  const int d0 = tile * kBwdCh, nc = min(kBwdCh, p.D - d0);
  const bool valid = c < nc;  // whole warps (8 channels; nc % 8 == 0)
  const int d = d0 + (valid ? c : 0);
  load_a_rows(As, p.A, p.E, p.D, p.N, d0, nc);
  for (int i = tid; i < p.E * 256 * 4; i += 256) dAacc[i] = 0.f;
  __syncthreads();
  const float dsk = p.D_skip[d];
  float carry[4] = {0.f, 0.f, 0.f, 0.f};
  float dD = 0.f;
  const IO* xg = reinterpret_cast<const IO*>(p.x);
  const IO* zg = reinterpret_cast<const IO*>(p.z);
  const IO* gg = reinterpret_cast<const IO*>(p.g_out);

  for (int ck = p.nck - 1; ck >= 0; --ck) {
    const int64_t t0 = (int64_t)ck * kBwdLc;
    const int nt = (int)(p.L - t0 < kBwdLc ? p.L - t0 : kBwdLc);
    float hs[4];
    {
      const float* src = p.ckpt + (((size_t)b * p.nck + ck) * p.D + d) * p.N;
#pragma unroll
      for (int s = 0; s < 4; ++s) hs[s] = (valid && 4 * q + s < p.N) ? src[4 * q + s] : 0.f;
    }
    // ---- recompute the chunk's states (H[i] = h after token t0 + i) and dy; write dz ----
    float H[kBwdLc][4];
    float DY[kBwdLc];
    {
      float h[4] = {hs[0], hs[1], hs[2], hs[3]};
#pragma unroll
      for (int i = 0; i < kBwdLc; ++i) {
        if (i < nt) {
          const size_t bt = (size_t)b * p.L + t0 + i;
          const float dl = valid ? p.delta[bt * p.D + d] : 0.f;
          const float xv = valid ? to_f32(xg[bt * p.D + d]) : 0.f;
          const float zv = valid ? to_f32(zg[bt * p.D + d]) : 0.f;
          const float go = valid ? to_f32(gg[bt * p.D + d]) : 0.f;
          float at[4] = {0.f, 0.f, 0.f, 0.f};
          for (int j = 0; j < p.k; ++j) {
            const int e = min(max(p.idx[bt * p.k + j], 0), p.E - 1);
            const float g = p.gates[bt * p.k + j];
            const float4 a4 = reinterpret_cast<const float4*>(As)[(e * kBwdCh + c) * 4 + q];
            at[0] = fmaf(g, a4.x, at[0]);
            at[1] = fmaf(g, a4.y, at[1]);
            at[2] = fmaf(g, a4.z, at[2]);
            at[3] = fmaf(g, a4.w, at[3]);
          }
          const float c0 = dl * kLog2e, dxv = dl * xv;
          float y = 0.f;
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const int n = 4 * q + s;
            const float bn = n < p.N ? p.B_mix[bt * p.N + n] : 0.f;
            const float cn = n < p.N ? p.C_mix[bt * p.N + n] : 0.f;
            h[s] = fmaf(ex2_approx(c0 * at[s]), h[s], dxv * bn);
            H[i][s] = h[s];
            y = fmaf(cn, h[s], y);
          }
          y += __shfl_xor_sync(0xffffffffu, y, 1);
          y += __shfl_xor_sync(0xffffffffu, y, 2);
          y = fmaf(dsk, xv, y);
          const float sg = sigmoid_f(zv);
          DY[i] = go * zv * sg;
          if (valid && q == 0) p.dz[bt * p.D + d] = go * y * sg * fmaf(zv, 1.f - sg, 1.f);
        }
      }
    }
    // ---- the adjoint back through the chunk ----
#pragma unroll
    for (int i = kBwdLc - 1; i >= 0; --i) {
      if (i < nt) {
        const size_t bt = (size_t)b * p.L + t0 + i;
        const float dl = valid ? p.delta[bt * p.D + d] : 0.f;
        const float xv = valid ? to_f32(xg[bt * p.D + d]) : 0.f;
        float at[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < p.k; ++j) {
          const int e = min(max(p.idx[bt * p.k + j], 0), p.E - 1);
          const float g = p.gates[bt * p.k + j];
          const float4 a4 = reinterpret_cast<const float4*>(As)[(e * kBwdCh + c) * 4 + q];
          at[0] = fmaf(g, a4.x, at[0]);
          at[1] = fmaf(g, a4.y, at[1]);
          at[2] = fmaf(g, a4.z, at[2]);
          at[3] = fmaf(g, a4.w, at[3]);
        }
        const float c0 = dl * kLog2e;
        float lam[4], dA[4], vB[4], vC[4];
        float sum_b = 0.f, sum_d = 0.f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int n = 4 * q + s;
          const float bn = n < p.N ? p.B_mix[bt * p.N + n] : 0.f;
          const float cn = n < p.N ? p.C_mix[bt * p.N + n] : 0.f;
          const float a = ex2_approx(c0 * at[s]);
          const float hp = i > 0 ? H[i > 0 ? i - 1 : 0][s] : hs[s];
          lam[s] = fmaf(cn, DY[i], carry[s]);
          const float ahp = a * hp;
          dA[s] = lam[s] * dl * ahp;
          sum_b = fmaf(lam[s], bn, sum_b);
          sum_d = fmaf(lam[s], at[s] * ahp, sum_d);
          vB[s] = lam[s] * dl * xv;
          vC[s] = DY[i] * H[i][s];
          carry[s] = a * lam[s];
        }
        sum_b += __shfl_xor_sync(0xffffffffu, sum_b, 1);
        sum_b += __shfl_xor_sync(0xffffffffu, sum_b, 2);
        sum_d += __shfl_xor_sync(0xffffffffu, sum_d, 1);
        sum_d += __shfl_xor_sync(0xffffffffu, sum_d, 2);
        if (valid && q == 0) {
          p.dx[bt * p.D + d] = fmaf(dsk, DY[i], dl * sum_b);
          p.ddelta[bt * p.D + d] = fmaf(sum_b, xv, sum_d);
          dD = fmaf(DY[i], xv, dD);
        }
        // dB, dC: sums over the warp's 8 channels (lanes with the same quarter q)
        float* rrow = red + ((size_t)warp * kBwdLc + i) * rw;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            vB[s] += __shfl_xor_sync(0xffffffffu, vB[s], o);
            vC[s] += __shfl_xor_sync(0xffffffffu, vC[s], o);
          }
        }
        if (lane < 4) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const int n = 4 * q + s;
            if (n < p.N) {
              rrow[n] = vB[s];
              rrow[p.N + n] = vC[s];
            }
          }
        }
        // dA per expert slot, and the slot's gate gradient (a sum over the warp's channels and states)
        for (int j = 0; j < p.k; ++j) {
          const int e = min(max(p.idx[bt * p.k + j], 0), p.E - 1);
          const float g = p.gates[bt * p.k + j];
          const float4 a4 = reinterpret_cast<const float4*>(As)[(e * kBwdCh + c) * 4 + q];
          float4* acc = reinterpret_cast<float4*>(dAacc) + (size_t)e * 256 + tid;
          float4 v = *acc;
          v.x = fmaf(g, dA[0], v.x);
          v.y = fmaf(g, dA[1], v.y);
          v.z = fmaf(g, dA[2], v.z);
          v.w = fmaf(g, dA[3], v.w);
          *acc = v;
          float dg = dA[0] * a4.x + dA[1] * a4.y + dA[2] * a4.z + dA[3] * a4.w;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) dg += __shfl_xor_sync(0xffffffffu, dg, o);
          if (lane == 0) rrow[2 * p.N + j] = dg;
        }
      }
    }
    __syncthreads();
    // the chunk's per-token sums over the CTA's warps -> this tile's partial
    for (int v = tid; v < nt * rw; v += 256) {
      const int i = v / rw, w = v % rw;
      float sum = 0.f;
      for (int wp = 0; wp < kBwdWarps; ++wp) sum += red[((size_t)wp * kBwdLc + i) * rw + w];
      const size_t tok = (size_t)b * p.L + t0 + i;
      p.part[((size_t)tile * p.B * p.L + tok) * rw + w] = sum;
    }
    __syncthreads();
  }
  if (valid) {
    if (p.dh0 != nullptr) {
#pragma unroll
      for (int s = 0; s < 4; ++s)
        if (4 * q + s < p.N) p.dh0[((size_t)b * p.D + d) * p.N + 4 * q + s] = carry[s];
    }
    for (int e = 0; e < p.E; ++e) {
      const float4 v = reinterpret_cast<const float4*>(dAacc)[(size_t)e * 256 + tid];
      const float vv[4] = {v.x, v.y, v.z, v.w};
      float* dst = p.part_A + (((size_t)b * p.E + e) * p.D + d) * p.N;
#pragma unroll
      for (int s = 0; s < 4; ++s)
        if (4 * q + s < p.N) dst[4 * q + s] = vv[s];
    }
    if (q == 0) p.part_D[(size_t)b * p.D + d] = dD;
  }
}

// Sums of the partials in a fixed order: dB, dC, dgates over channel tiles; dA, dD over sequences.
__global__ void scan_bwd_reduce_kernel(ScanBwdParams p, int tiles) {
  const int rw = 2 * p.N + p.k;
  const int64_t n_tok = (int64_t)p.B * p.L * rw;
  const int64_t n_A = (int64_t)p.E * p.D * p.N;
  const int64_t total = n_tok + n_A + p.D;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    if (i < n_tok) {
      float s = 0.f;
      for (int t = 0; t < tiles; ++t) s += p.part[(size_t)t * n_tok + i];
      const int64_t tok = i / rw;
      const int w = (int)(i % rw);
      if (w < p.N) p.dB[tok * p.N + w] = s;
      else if (w < 2 * p.N) p.dC[tok * p.N + w - p.N] = s;
      else p.dgates[tok * p.k + w - 2 * p.N] = s;
    } else if (i < n_tok + n_A) {
      const int64_t r = i - n_tok;
      float s = 0.f;
      for (int b = 0; b < p.B; ++b) s += p.part_A[(size_t)b * n_A + r];
      p.dA[r] = s;
    } else {
      const int64_t r = i - n_tok - n_A;
      float s = 0.f;
      for (int b = 0; b < p.B; ++b) s += p.part_D[(size_t)b * p.D + r];
      p.dD[r] = s;
    }
  }
}

size_t scan_bwd_workspace(int64_t B, int64_t L, int D, int N, int E, int k) {
  const int64_t tiles = (D + kBwdCh - 1) / kBwdCh;
  const int64_t nck = (L + kBwdLc - 1) / kBwdLc;
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  return up((size_t)B * nck * D * N * 4) + up((size_t)tiles * B * L * (2 * N + k) * 4) +
         up((size_t)B * E * D * N * 4) + up((size_t)B * D * 4);
}

cudaError_t run_scan_bwd(ScanBwdParams p, bool io_bf16, void* ws, cudaStream_t s) {
  const int tiles = (p.D + kBwdCh - 1) / kBwdCh;
  p.nck = (int)((p.L + kBwdLc - 1) / kBwdLc);
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ckpt = reinterpret_cast<float*>(w);
  w += up((size_t)p.B * p.nck * p.D * p.N * 4);
  p.part = reinterpret_cast<float*>(w);
  w += up((size_t)tiles * p.B * p.L * (2 * p.N + p.k) * 4);
  p.part_A = reinterpret_cast<float*>(w);
  w += up((size_t)p.B * p.E * p.D * p.N * 4);
  p.part_D = reinterpret_cast<float*>(w);
  const unsigned grid = (unsigned)(tiles * p.B);
  const size_t smem_ck = sizeof(float) * (size_t)p.E * kBwdCh * 16;
  const size_t smem_bw = smem_ck + sizeof(float) * ((size_t)p.E * 256 * 4 + (size_t)kBwdWarps * kBwdLc * (2 * p.N + p.k));
  cudaError_t e;
  if (io_bf16) {
    if ((e = cudaFuncSetAttribute(scan_bwd_ckpt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_ck)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(scan_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_bw)) != cudaSuccess)
      return e;
    scan_bwd_ckpt_kernel<__nv_bfloat16><<<grid, 256, smem_ck, s>>>(p);
    scan_bwd_kernel<__nv_bfloat16><<<grid, 256, smem_bw, s>>>(p);
  } else {
    if ((e = cudaFuncSetAttribute(scan_bwd_ckpt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_ck)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(scan_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_bw)) != cudaSuccess)
      return e;
    scan_bwd_ckpt_kernel<float><<<grid, 256, smem_ck, s>>>(p);
    scan_bwd_kernel<float><<<grid, 256, smem_bw, s>>>(p);
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  scan_bwd_reduce_kernel<<<(unsigned)(4 * sms), 256, 0, s>>>(p, tiles);
  note_launch(3);
  return cudaGetLastError();
}

}  // namespace swimba
