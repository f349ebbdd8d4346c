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
//           from the last: runs forward through the chunk from its checkpoint (writing dz, and the
//           state before every 4-token sub-block to shared memory), then runs the adjoint back
//           one sub-block at a time, recomputing the sub-block's 4 states into registers (a short
//           unrolled body: with a 16-token body the kernel stalled on instruction fetch). The
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

// A chunk of up to 16 tokens of the CTA's 64 channels, staged in shared memory by all 256 threads
// with 16-byte loads (the inner loops then read on-chip memory, not a chain of global loads).
template <typename IO>
struct ChunkTile {
  float dl[kBwdLc][kBwdCh];
  IO x[kBwdLc][kBwdCh];
  IO z[kBwdLc][kBwdCh];
  IO go[kBwdLc][kBwdCh];
  float B[kBwdLc][16];
  float C[kBwdLc][16];
  int e[kBwdLc][16];
  float g[kBwdLc][16];
};

template <typename IO>
__device__ __forceinline__ void load_chunk(ChunkTile<IO>& ct, const ScanBwdParams& p, int b, int64_t t0, int nt,
                                           int d0, int nc, bool with_zg) {
  const int tid = threadIdx.x;
  constexpr int per16 = 16 / (int)sizeof(IO);
  const int v4 = nc / 4, vio = nc / per16;  // nc % 8 == 0
  for (int i = tid; i < nt * v4; i += 256) {
    const int r = i / v4, c = (i % v4) * 4;
    *reinterpret_cast<float4*>(&ct.dl[r][c]) =
        *reinterpret_cast<const float4*>(p.delta + ((size_t)b * p.L + t0 + r) * p.D + d0 + c);
  }
  for (int i = tid; i < nt * vio; i += 256) {
    const int r = i / vio, c = (i % vio) * per16;
    const size_t g = ((size_t)b * p.L + t0 + r) * p.D + d0 + c;
    *reinterpret_cast<uint4*>(&ct.x[r][c]) = *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.x) + g);
    if (with_zg) {
      *reinterpret_cast<uint4*>(&ct.z[r][c]) = *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.z) + g);
      *reinterpret_cast<uint4*>(&ct.go[r][c]) =
          *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.g_out) + g);
    }
  }
  for (int i = tid; i < nt * 16; i += 256) {
    const int r = i / 16, n = i % 16;
    const size_t bt = (size_t)b * p.L + t0 + r;
    ct.B[r][n] = n < p.N ? p.B_mix[bt * p.N + n] : 0.f;
    ct.C[r][n] = (with_zg && n < p.N) ? p.C_mix[bt * p.N + n] : 0.f;
    // every slot holds an expert in [0, E) (zero gate past k), so no index read from the tile can
    // leave the A tables
    ct.e[r][n] = n < p.k ? min(max(p.idx[bt * p.k + n], 0), p.E - 1) : 0;
    ct.g[r][n] = n < p.k ? p.gates[bt * p.k + n] : 0.f;
  }
}

// The mixed transition row quarter of token r for this thread's channel c and quarter q.
template <int K, typename IO>
__device__ __forceinline__ void mix_a(const ChunkTile<IO>& ct, const float* As, int r, int k_rt, int c, int q,
                                     float (&at)[4]) {
  at[0] = at[1] = at[2] = at[3] = 0.f;
  const int k = K > 0 ? K : k_rt;  // K > 0: unrolled; K == 0: a runtime loop
#pragma unroll
  for (int j = 0; j < k; ++j) {
    const float g = ct.g[r][j];
    const float4 a4 = reinterpret_cast<const float4*>(As)[(ct.e[r][j] * kBwdCh + c) * 4 + q];
    at[0] = fmaf(g, a4.x, at[0]);
    at[1] = fmaf(g, a4.y, at[1]);
    at[2] = fmaf(g, a4.z, at[2]);
    at[3] = fmaf(g, a4.w, at[3]);
  }
}

template <typename IO, int K>
__global__ void __launch_bounds__(256) scan_bwd_ckpt_kernel(ScanBwdParams p) {
  extern __shared__ __align__(16) float smem_ck[];
  float* As = smem_ck;                                                        // [E][64][16]
  ChunkTile<IO>& ct = *reinterpret_cast<ChunkTile<IO>*>(As + p.E * kBwdCh * 16);
  const int tid = threadIdx.x, c = tid >> 2, q = tid & 3;
  const int tiles = (p.D + kBwdCh - 1) / kBwdCh;
  const int tile = blockIdx.x % tiles, b = blockIdx.x / tiles;
  const int d0 = tile * kBwdCh, nc = min(kBwdCh, p.D - d0);
  const bool valid = c < nc;
  const int d = d0 + (valid ? c : 0);
  load_a_rows(As, p.A, p.E, p.D, p.N, d0, nc);
  float h[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int n = 4 * q + s;
    h[s] = (valid && p.h0 != nullptr && n < p.N) ? p.h0[((size_t)b * p.D + d) * p.N + n] : 0.f;
  }
  for (int ck = 0; ck < p.nck; ++ck) {
    const int64_t t0 = (int64_t)ck * kBwdLc;
    const int nt = (int)(p.L - t0 < kBwdLc ? p.L - t0 : kBwdLc);
    if (valid) {
      float* dst = p.ckpt + (((size_t)b * p.nck + ck) * p.D + d) * p.N;
#pragma unroll
      for (int s = 0; s < 4; ++s)
        if (4 * q + s < p.N) dst[4 * q + s] = h[s];
    }
    __syncthreads();  // the previous chunk's tile is no longer read
    load_chunk(ct, p, b, t0, nt, d0, nc, false);
    __syncthreads();
    for (int i = 0; i < nt; ++i) {
      float at[4];
      mix_a<K>(ct, As, i, p.k, c, q, at);
      const float dl = ct.dl[i][c], c0 = dl * kLog2e, dxv = dl * to_f32(ct.x[i][c]);
#pragma unroll
      for (int s = 0; s < 4; ++s) h[s] = fmaf(ex2_approx(c0 * at[s]), h[s], dxv * ct.B[i][4 * q + s]);
    }
  }
}

constexpr int kBwdSub = 4;  // tokens per sub-block of the adjoint pass

// The adjoint back through tokens [i0, i0 + ni) of the staged chunk (ni <= 4), from the state h_in
// before token i0: recomputes the sub-block's states and dy into registers (a 4-token unrolled
// body keeps the code small), then walks it backwards, updating `carry` (a_{t+1} λ_{t+1}).
template <int K, typename IO>
__device__ __forceinline__ void adjoint_sub(const ScanBwdParams& p, const ChunkTile<IO>& ct, const float* As,
                                            float* dAacc, float* red, int rw, int i0, int ni, const float (&h_in)[4],
                                            int64_t t0, int b, int d, int cc, bool valid, float dsk, int tid,
                                            int warp, int lane, int q, float (&carry)[4], float& dD) {
  float H[kBwdSub][4], DY[kBwdSub], AT[kBwdSub][4], AB[kBwdSub][4];  // states, dy, A_t, exp(Δ A_t)
  {
    float h[4] = {h_in[0], h_in[1], h_in[2], h_in[3]};
#pragma unroll
    for (int u = 0; u < kBwdSub; ++u) {
      if (u < ni) {
        const int i = i0 + u;
        float at[4];
        mix_a<K>(ct, As, i, p.k, cc, q, at);
        const float dl = valid ? ct.dl[i][cc] : 0.f;
        const float xv = valid ? to_f32(ct.x[i][cc]) : 0.f;
        const float zv = valid ? to_f32(ct.z[i][cc]) : 0.f;
        const float go = valid ? to_f32(ct.go[i][cc]) : 0.f;
        const float c0 = dl * kLog2e, dxv = dl * xv;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          AT[u][s] = at[s];
          AB[u][s] = ex2_approx(c0 * at[s]);
          h[s] = fmaf(AB[u][s], h[s], dxv * ct.B[i][4 * q + s]);
          H[u][s] = h[s];
        }
        DY[u] = go * zv * sigmoid_f(zv);
      }
    }
  }
#pragma unroll
  for (int u = kBwdSub - 1; u >= 0; --u) {
    if (u < ni) {
      const int i = i0 + u;
      const size_t bt = (size_t)b * p.L + t0 + i;
      const float dl = valid ? ct.dl[i][cc] : 0.f;
      const float xv = valid ? to_f32(ct.x[i][cc]) : 0.f;
      const float dlx = dl * xv;
      float dA[4], vB[4], vC[4];
      float sum_b = 0.f, sum_d = 0.f;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const float bn = ct.B[i][4 * q + s], cn = ct.C[i][4 * q + s];
        const float a = AB[u][s];
        const float hp = u > 0 ? H[u > 0 ? u - 1 : 0][s] : h_in[s];
        const float lam = fmaf(cn, DY[u], carry[s]);
        const float ahp = a * hp;
        dA[s] = lam * dl * ahp;
        sum_b = fmaf(lam, bn, sum_b);
        sum_d = fmaf(lam, AT[u][s] * ahp, sum_d);
        vB[s] = lam * dlx;
        vC[s] = DY[u] * H[u][s];
        carry[s] = a * lam;
      }
      sum_b += __shfl_xor_sync(0xffffffffu, sum_b, 1);
      sum_b += __shfl_xor_sync(0xffffffffu, sum_b, 2);
      sum_d += __shfl_xor_sync(0xffffffffu, sum_d, 1);
      sum_d += __shfl_xor_sync(0xffffffffu, sum_d, 2);
      if (valid && q == 0) {
        p.dx[bt * p.D + d] = fmaf(dsk, DY[u], dl * sum_b);
        p.ddelta[bt * p.D + d] = fmaf(sum_b, xv, sum_d);
        dD = fmaf(DY[u], xv, dD);
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
      const int kk = K > 0 ? K : p.k;
#pragma unroll
      for (int j = 0; j < kk; ++j) {
        const int e = ct.e[i][j];
        const float g = ct.g[i][j];
        const float4 a4 = reinterpret_cast<const float4*>(As)[(e * kBwdCh + cc) * 4 + q];
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
}

template <typename IO, int K>
__global__ void __launch_bounds__(256, 2) scan_bwd_kernel(ScanBwdParams p) {
  extern __shared__ __align__(16) float smem[];
  float* As = smem;                                  // [E][64][16]
  float* dAacc = As + p.E * kBwdCh * 16;             // [E][256 threads][4]
  float4* sub = reinterpret_cast<float4*>(dAacc + p.E * 256 * 4);  // [4 sub-blocks][256 threads]
  float* red = reinterpret_cast<float*>(sub + (kBwdLc / kBwdSub) * 256);  // [8 warps][16 tokens][rw]
  const int rw = 2 * p.N + p.k;                      // per token: dB[N], dC[N], dgates[k]
  ChunkTile<IO>& ct = *reinterpret_cast<ChunkTile<IO>*>(red + kBwdWarps * kBwdLc * rw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, c = tid >> 2, q = tid & 3;
  const int tiles = (p.D + kBwdCh - 1) / kBwdCh;
  const int tile = blockIdx.x % tiles, b = blockIdx.x / tiles;
  const int d0 = tile * kBwdCh, nc = min(kBwdCh, p.D - d0);
  const bool valid = c < nc;  // whole warps (8 channels; nc % 8 == 0)
  const int cc = valid ? c : 0;
  const int d = d0 + cc;
  load_a_rows(As, p.A, p.E, p.D, p.N, d0, nc);
  for (int i = tid; i < p.E * 256 * 4; i += 256) dAacc[i] = 0.f;
  const float dsk = p.D_skip[d];
  float carry[4] = {0.f, 0.f, 0.f, 0.f};
  float dD = 0.f;

  for (int ck = p.nck - 1; ck >= 0; --ck) {
    const int64_t t0 = (int64_t)ck * kBwdLc;
    const int nt = (int)(p.L - t0 < kBwdLc ? p.L - t0 : kBwdLc);
    __syncthreads();  // the previous chunk's tile and partial sums are no longer read
    load_chunk(ct, p, b, t0, nt, d0, nc, true);
    float h[4];
    {
      const float* src = p.ckpt + (((size_t)b * p.nck + ck) * p.D + d) * p.N;
#pragma unroll
      for (int s = 0; s < 4; ++s) h[s] = (valid && 4 * q + s < p.N) ? src[4 * q + s] : 0.f;
    }
    __syncthreads();
    // ---- forward through the chunk: the state before every 4-token sub-block (shared memory),
    // and dz (which needs y) ----
    for (int i = 0; i < nt; ++i) {
      if ((i & (kBwdSub - 1)) == 0) sub[(i / kBwdSub) * 256 + tid] = make_float4(h[0], h[1], h[2], h[3]);
      float at[4];
      mix_a<K>(ct, As, i, p.k, cc, q, at);
      const float dl = valid ? ct.dl[i][cc] : 0.f;
      const float xv = valid ? to_f32(ct.x[i][cc]) : 0.f;
      const float c0 = dl * kLog2e, dxv = dl * xv;
      float y = 0.f;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        h[s] = fmaf(ex2_approx(c0 * at[s]), h[s], dxv * ct.B[i][4 * q + s]);
        y = fmaf(ct.C[i][4 * q + s], h[s], y);
      }
      y += __shfl_xor_sync(0xffffffffu, y, 1);
      y += __shfl_xor_sync(0xffffffffu, y, 2);
      if (valid && q == 0) {
        const float zv = to_f32(ct.z[i][cc]), go = to_f32(ct.go[i][cc]);
        const float sg = sigmoid_f(zv);
        p.dz[((size_t)b * p.L + t0 + i) * p.D + d] = go * fmaf(dsk, xv, y) * sg * fmaf(zv, 1.f - sg, 1.f);
      }
    }
    // ---- the adjoint back through the chunk, one 4-token sub-block at a time ----
    for (int sb = (nt - 1) / kBwdSub; sb >= 0; --sb) {
      const int i0 = sb * kBwdSub;
      const int ni = nt - i0 < kBwdSub ? nt - i0 : kBwdSub;
      const float4 hv = sub[sb * 256 + tid];
      const float h_in[4] = {hv.x, hv.y, hv.z, hv.w};
      adjoint_sub<K>(p, ct, As, dAacc, red, rw, i0, ni, h_in, t0, b, d, cc, valid, dsk, tid, warp, lane, q, carry, dD);
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

template <typename IO, int K>
cudaError_t launch_bwd_pair(const ScanBwdParams& p, unsigned grid, size_t smem_ck, size_t smem_bw, cudaStream_t s) {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(scan_bwd_ckpt_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_ck)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(scan_bwd_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bw)) !=
      cudaSuccess)
    return e;
  scan_bwd_ckpt_kernel<IO, K><<<grid, 256, smem_ck, s>>>(p);
  scan_bwd_kernel<IO, K><<<grid, 256, smem_bw, s>>>(p);
  return cudaGetLastError();
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
  const size_t a_bytes = sizeof(float) * (size_t)p.E * kBwdCh * 16;
  const size_t tile_bytes = io_bf16 ? sizeof(ChunkTile<__nv_bfloat16>) : sizeof(ChunkTile<float>);
  const size_t smem_ck = a_bytes + tile_bytes;
  const size_t smem_bw = a_bytes + sizeof(float) * ((size_t)p.E * 256 * 4 + (size_t)kBwdWarps * kBwdLc * (2 * p.N + p.k)) +
                         sizeof(float4) * (kBwdLc / kBwdSub) * 256 + tile_bytes;
  cudaError_t e;
  if (io_bf16) {
    if (p.k == 1) e = launch_bwd_pair<__nv_bfloat16, 1>(p, grid, smem_ck, smem_bw, s);
    else if (p.k == 2) e = launch_bwd_pair<__nv_bfloat16, 2>(p, grid, smem_ck, smem_bw, s);
    else e = launch_bwd_pair<__nv_bfloat16, 0>(p, grid, smem_ck, smem_bw, s);
  } else {
    if (p.k == 1) e = launch_bwd_pair<float, 1>(p, grid, smem_ck, smem_bw, s);
    else if (p.k == 2) e = launch_bwd_pair<float, 2>(p, grid, smem_ck, smem_bw, s);
    else e = launch_bwd_pair<float, 0>(p, grid, smem_ck, smem_bw, s);
  }
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  scan_bwd_reduce_kernel<<<(unsigned)(4 * sms), 256, 0, s>>>(p, tiles);
  note_launch(3);
  return cudaGetLastError();
}

}  // namespace swimba
