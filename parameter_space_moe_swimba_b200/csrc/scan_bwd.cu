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
// Shapes: N <= 16, any k <= E <= 16, io fp32 or bf16. For N = 16, k <= 2 and D % 16 == 0 the bwd
// kernel runs in a packed layout (two channels per lane, f32x2 arithmetic, the A rows in tensor
// memory, the sub-block states in an L2-resident global scratch and the adjoint's exponentials
// recomputed rather than kept, so four CTAs fit on an SM; scan_bwd_pk_kernel), and with bf16 io the
// checkpoints come from the forward's fast scan (its recurrence-only pass in checkpoint mode,
// run_scan_fast_ckpt) instead of the ckpt kernel.
#include "common.cuh"
#include "scan.cuh"
#include "sm100.cuh"

namespace swimba {

namespace {

constexpr int kBwdCh = 64;    // channels per CTA
constexpr int kBwdLc = 16;    // tokens per checkpoint chunk
constexpr int kBwdWarps = 8;  // 256 threads

__device__ __forceinline__ float sigmoid_f(float v) { return __fdividef(1.f, 1.f + ex2_approx(-v * kLog2e)); }

// The A rows of every expert for the CTA's channels: As[e][c][16], zero beyond N.
__device__ __forceinline__ void load_a_rows(float* As, const float* A, int E, int D, int N, int d0, int nc) {
  for (int i = threadIdx.x; i < E * kBwdCh * 16; i += blockDim.x) {
    const int e = i / (kBwdCh * 16), r = i % (kBwdCh * 16), c = r / 16, n = r % 16;
    As[i] = (c < nc && n < N) ? A[((size_t)e * D + d0 + c) * N + n] : 0.f;
  }
}

}  // namespace

// A chunk of up to 16 tokens of the CTA's 64 channels, staged in shared memory by all the CTA's
// threads with 16-byte loads (the inner loops then read on-chip memory, not a chain of global loads).
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
  for (int i = tid; i < nt * v4; i += blockDim.x) {
    const int r = i / v4, c = (i % v4) * 4;
    *reinterpret_cast<float4*>(&ct.dl[r][c]) =
        *reinterpret_cast<const float4*>(p.delta + ((size_t)b * p.L + t0 + r) * p.D + d0 + c);
  }
  for (int i = tid; i < nt * vio; i += blockDim.x) {
    const int r = i / vio, c = (i % vio) * per16;
    const size_t g = ((size_t)b * p.L + t0 + r) * p.D + d0 + c;
    *reinterpret_cast<uint4*>(&ct.x[r][c]) = *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.x) + g);
    if (with_zg) {
      *reinterpret_cast<uint4*>(&ct.z[r][c]) = *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.z) + g);
      *reinterpret_cast<uint4*>(&ct.go[r][c]) =
          *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.g_out) + g);
    }
  }
  for (int i = tid; i < nt * 16; i += blockDim.x) {
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

// ---- packed layout for N = 16, k <= 2, D % 16 == 0 ---------------------------------------------
// A CTA of 4 warps owns 64 channels; lane l of warp w holds the channel pair c0 = 16 w + 2 (l >> 2),
// c1 = c0 + 1 and the state quarter q = l & 3 (states 4q .. 4q + 3), every per-state value a
// float2 over the two channels (packed f32x2 arithmetic, as in the forward scan). Against the
// one-channel layout above it halves the arithmetic and the per-channel loads per state element,
// and the per-token sums over channels (dB, dC, the gate gradients) leave each lane with one value
// of a reduce-scatter instead of every lane with every value.
constexpr int kPkThreads = 128;
constexpr int kPkWarps = 4;

__device__ __forceinline__ float2 f2s(float v) { return make_float2(v, v); }

// The A rows (4 states) of token r's expert slots for the lane's two channels. Lanes of odd channel
// pairs read their second channel first, so every 8-lane phase of the 16-byte loads touches 8
// distinct bank groups.
template <int K, typename IO>
__device__ __forceinline__ void load_a2(const ChunkTile<IO>& ct, const float* As, int r, int c0, int q,
                                       float4 (&a0)[K], float4 (&a1)[K]) {
  const bool sw = (c0 >> 1) & 1;
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const float4* row = reinterpret_cast<const float4*>(As) + (ct.e[r][j] * kBwdCh + c0) * 4 + q;
    const float4 f = row[sw ? 4 : 0], t = row[sw ? 0 : 4];
    a0[j] = sw ? t : f;
    a1[j] = sw ? f : t;
  }
}

// The mixed transition rows A_t = Σ_j g_j A^{e_j} (4 states, both channels) of staged token r.
template <int K, typename IO>
__device__ __forceinline__ void mix_a2(const ChunkTile<IO>& ct, const float4 (&a0)[K], const float4 (&a1)[K], int r,
                                      float2 (&at)[4]) {
#pragma unroll
  for (int s = 0; s < 4; ++s) at[s] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const float2 g = f2s(ct.g[r][j]);
    at[0] = __ffma2_rn(g, make_float2(a0[j].x, a1[j].x), at[0]);
    at[1] = __ffma2_rn(g, make_float2(a0[j].y, a1[j].y), at[1]);
    at[2] = __ffma2_rn(g, make_float2(a0[j].z, a1[j].z), at[2]);
    at[3] = __ffma2_rn(g, make_float2(a0[j].w, a1[j].w), at[3]);
  }
}

template <int K, typename IO>
__device__ __forceinline__ void mix_a2(const ChunkTile<IO>& ct, const float* As, int r, int c0, int q,
                                      float2 (&at)[4]) {
  float4 a0[K], a1[K];
  load_a2<K>(ct, As, r, c0, q, a0, a1);
  mix_a2<K>(ct, a0, a1, r, at);
}

// The same rows from tensor memory: in the warp's lane quarter (tm_lane = its address), column 8e of
// lane l holds (A[e][c0][4q .. 4q+3], A[e][c0+1][4q .. 4q+3]) for the lane's channels and quarter.
// The expert of a token is uniform over the warp, so the load is one warp-wide tcgen05.ld per slot.
template <int K, typename IO>
__device__ __forceinline__ void load_a2_tm(const ChunkTile<IO>& ct, uint32_t tm_lane, int r, float4 (&a0)[K],
                                          float4 (&a1)[K]) {
  uint32_t v[K][8];
#pragma unroll
  for (int j = 0; j < K; ++j) sm100::tmem_ld8_nowait(tm_lane + (uint32_t)ct.e[r][j] * 8u, v[j]);
  sm100::tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < K; ++j) {
    a0[j] = make_float4(__uint_as_float(v[j][0]), __uint_as_float(v[j][1]), __uint_as_float(v[j][2]),
                        __uint_as_float(v[j][3]));
    a1[j] = make_float4(__uint_as_float(v[j][4]), __uint_as_float(v[j][5]), __uint_as_float(v[j][6]),
                        __uint_as_float(v[j][7]));
  }
}

__device__ __forceinline__ float2 ld2(const float (&row)[kBwdCh], int c0) {
  return *reinterpret_cast<const float2*>(&row[c0]);
}
__device__ __forceinline__ float2 ld2(const __nv_bfloat16 (&row)[kBwdCh], int c0) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&row[c0]));
}

// One exp2 per component (the special-function unit has no packed form).
__device__ __forceinline__ float2 ex2_2(float2 v) { return make_float2(ex2_approx(v.x), ex2_approx(v.y)); }

template <typename IO, int K>
__global__ void __launch_bounds__(kPkThreads) scan_bwd_ckpt_pk_kernel(ScanBwdParams p) {
  extern __shared__ __align__(16) float smem_pk[];
  float* As = smem_pk;  // [E][64][16]
  ChunkTile<IO>& ct = *reinterpret_cast<ChunkTile<IO>*>(As + p.E * kBwdCh * 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q = lane & 3;
  const int c0 = 16 * warp + 2 * (lane >> 2);
  const int tiles = (p.D + kBwdCh - 1) / kBwdCh;
  const int tile = blockIdx.x % tiles, b = blockIdx.x / tiles;
  const int d0 = tile * kBwdCh, nc = min(kBwdCh, p.D - d0);  // nc % 16 == 0
  const bool valid = 16 * warp < nc;                         // whole warps
  load_a_rows(As, p.A, p.E, p.D, p.N, d0, nc);
  float2 h[4];
  {
    float4 u0 = make_float4(0.f, 0.f, 0.f, 0.f), u1 = u0;
    if (valid && p.h0 != nullptr) {
      u0 = *reinterpret_cast<const float4*>(p.h0 + ((size_t)b * p.D + d0 + c0) * 16 + 4 * q);
      u1 = *reinterpret_cast<const float4*>(p.h0 + ((size_t)b * p.D + d0 + c0 + 1) * 16 + 4 * q);
    }
    h[0] = make_float2(u0.x, u1.x);
    h[1] = make_float2(u0.y, u1.y);
    h[2] = make_float2(u0.z, u1.z);
    h[3] = make_float2(u0.w, u1.w);
  }
  for (int ck = 0; ck < p.nck; ++ck) {
    const int64_t t0 = (int64_t)ck * kBwdLc;
    const int nt = (int)(p.L - t0 < kBwdLc ? p.L - t0 : kBwdLc);
    if (valid) {
      float* dst = p.ckpt + (((size_t)b * p.nck + ck) * p.D + d0 + c0) * 16 + 4 * q;
      *reinterpret_cast<float4*>(dst) = make_float4(h[0].x, h[1].x, h[2].x, h[3].x);
      *reinterpret_cast<float4*>(dst + 16) = make_float4(h[0].y, h[1].y, h[2].y, h[3].y);
    }
    __syncthreads();  // the previous chunk's tile is no longer read
    load_chunk(ct, p, b, t0, nt, d0, nc, false);
    __syncthreads();
    for (int i = 0; i < nt; ++i) {
      float2 at[4];
      mix_a2<K>(ct, As, i, c0, q, at);
      const float2 dl = ld2(ct.dl[i], c0);
      const float2 c2 = __fmul2_rn(dl, f2s(kLog2e)), dx = __fmul2_rn(dl, ld2(ct.x[i], c0));
#pragma unroll
      for (int s = 0; s < 4; ++s)
        h[s] = __ffma2_rn(ex2_2(__fmul2_rn(c2, at[s])), h[s], __fmul2_rn(dx, f2s(ct.B[i][4 * q + s])));
    }
  }
}

// The adjoint back through tokens [i0, i0 + ni) of the staged chunk (ni <= 4), packed layout: the
// sub-block's states, transitions and dy are recomputed into registers from h_in (the state
// before token i0), then walked backwards, updating `carry` (a_{t+1} λ_{t+1}).
// FULL: the sub-block holds kBwdSub tokens (every sub-block but a ragged tail), so its token loops
// carry no bounds test and the compiler may interleave the tokens' independent work.
template <int K, bool FULL, typename IO>
__device__ __forceinline__ void adjoint_sub_pk(const ScanBwdParams& p, const ChunkTile<IO>& ct, uint32_t tm_lane,
                                               float* dAacc, float* red, int rw, int i0, int ni,
                                               const float2 (&h_in)[4], int64_t t0, int b, int d0, int c0,
                                               bool valid, float2 dsk, int tid, int warp, int lane, int q,
                                               float2 (&carry)[4], float2& dD) {
  float2 H[kBwdSub][4], DY[kBwdSub];
  {
    float2 h[4] = {h_in[0], h_in[1], h_in[2], h_in[3]};
#pragma unroll
    for (int u = 0; u < kBwdSub; ++u) {
      if (FULL || u < ni) {
        const int i = i0 + u;
        float4 a0[K], a1[K];
        load_a2_tm<K>(ct, tm_lane, i, a0, a1);
        float2 at[4];
        mix_a2<K>(ct, a0, a1, i, at);
        const float2 dl = ld2(ct.dl[i], c0), xv = ld2(ct.x[i], c0);
        const float2 c2 = __fmul2_rn(dl, f2s(kLog2e)), dx = __fmul2_rn(dl, xv);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          h[s] = __ffma2_rn(ex2_2(__fmul2_rn(c2, at[s])), h[s], __fmul2_rn(dx, f2s(ct.B[i][4 * q + s])));
          H[u][s] = h[s];
        }
        const float2 zv = ld2(ct.z[i], c0), go = ld2(ct.go[i], c0);
        DY[u] = __fmul2_rn(__fmul2_rn(go, zv), make_float2(sigmoid_f(zv.x), sigmoid_f(zv.y)));
      }
    }
  }
#pragma unroll
  for (int u = kBwdSub - 1; u >= 0; --u) {
    if (FULL || u < ni) {
      const int i = i0 + u;
      float4 a0[K], a1[K];
      load_a2_tm<K>(ct, tm_lane, i, a0, a1);
      float2 at[4];
      mix_a2<K>(ct, a0, a1, i, at);
      const float2 dl = ld2(ct.dl[i], c0), xv = ld2(ct.x[i], c0);
      const float2 dlx = __fmul2_rn(dl, xv), c2 = __fmul2_rn(dl, f2s(kLog2e));
      float2 dA[4], sum_b = make_float2(0.f, 0.f), sum_d = make_float2(0.f, 0.f);
      float vB[4], vC[4];
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const float2 hp = u > 0 ? H[u > 0 ? u - 1 : 0][s] : h_in[s];
        const float2 lam = __ffma2_rn(f2s(ct.C[i][4 * q + s]), DY[u], carry[s]);
        const float2 ab = ex2_2(__fmul2_rn(c2, at[s]));  // recomputed: not kept from the forward above
        const float2 ahp = __fmul2_rn(ab, hp);
        dA[s] = __fmul2_rn(__fmul2_rn(lam, dl), ahp);
        sum_b = __ffma2_rn(lam, f2s(ct.B[i][4 * q + s]), sum_b);
        sum_d = __ffma2_rn(__fmul2_rn(lam, at[s]), ahp, sum_d);
        vB[s] = fmaf(lam.x, dlx.x, lam.y * dlx.y);               // this lane's 2 channels
        vC[s] = fmaf(DY[u].x, H[u][s].x, DY[u].y * H[u][s].y);
        carry[s] = __fmul2_rn(ab, lam);
      }
      // dx, dΔ: sums over the channel's 4 state quarters
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        sum_b.x += __shfl_xor_sync(0xffffffffu, sum_b.x, o);
        sum_b.y += __shfl_xor_sync(0xffffffffu, sum_b.y, o);
        sum_d.x += __shfl_xor_sync(0xffffffffu, sum_d.x, o);
        sum_d.y += __shfl_xor_sync(0xffffffffu, sum_d.y, o);
      }
      // every lane of a quarter group now holds both channels' sums: lane q writes one of the four
      // values (dx of c0, c0 + 1; dΔ of c0, c0 + 1), so no branch
      {
        const bool odd = q & 1;
        const float sb = odd ? sum_b.y : sum_b.x;
        const float vdx = fmaf(odd ? dsk.y : dsk.x, odd ? DY[u].y : DY[u].x, (odd ? dl.y : dl.x) * sb);
        const float vdd = fmaf(sb, odd ? xv.y : xv.x, odd ? sum_d.y : sum_d.x);
        const size_t g = ((size_t)b * p.L + t0 + i) * p.D + d0 + c0 + (odd ? 1 : 0);
        if (valid) (q < 2 ? p.dx : p.ddelta)[g] = q < 2 ? vdx : vdd;
        dD = __ffma2_rn(DY[u], xv, dD);  // every lane alike; the q == 0 lanes' sums are written
      }
      // dB, dC: the 8 values (vB[0..3], vC[0..3]) summed over the warp's 8 channel pairs (lane
      // bits 2-4) by recursive halving; lane l ends with the value of type (l >> 4) & 1 (B, C) and
      // state 4q + 2((l >> 3) & 1) + ((l >> 2) & 1)
      float v4[4], v2[2], v1;
      {
        const bool hi = lane & 16;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float keep = hi ? vC[m] : vB[m], send = hi ? vB[m] : vC[m];
          v4[m] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
      }
      {
        const bool hi = lane & 8;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const float keep = hi ? v4[m + 2] : v4[m], send = hi ? v4[m] : v4[m + 2];
          v2[m] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
      }
      {
        const bool hi = lane & 4;
        const float keep = hi ? v2[1] : v2[0], send = hi ? v2[0] : v2[1];
        v1 = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      float* rrow = red + ((size_t)warp * kBwdLc + i) * rw;
      rrow[((lane >> 4) & 1) * 16 + 4 * q + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1)] = v1;
      // dA per expert slot, and the slots' gate gradients (sums over the warp's channels and states)
      float pj[K];
#pragma unroll
      for (int j = 0; j < K; ++j) {
        const int e = ct.e[i][j];
        const float2 g = f2s(ct.g[i][j]);
        float4* acc = reinterpret_cast<float4*>(dAacc) + (size_t)e * 2 * kPkThreads + tid;
        float4 w0 = acc[0], w1 = acc[kPkThreads];
        w0.x = fmaf(g.x, dA[0].x, w0.x);
        w0.y = fmaf(g.x, dA[1].x, w0.y);
        w0.z = fmaf(g.x, dA[2].x, w0.z);
        w0.w = fmaf(g.x, dA[3].x, w0.w);
        w1.x = fmaf(g.x, dA[0].y, w1.x);
        w1.y = fmaf(g.x, dA[1].y, w1.y);
        w1.z = fmaf(g.x, dA[2].y, w1.z);
        w1.w = fmaf(g.x, dA[3].y, w1.w);
        acc[0] = w0;
        acc[kPkThreads] = w1;
        pj[j] = dA[0].x * a0[j].x + dA[1].x * a0[j].y + dA[2].x * a0[j].z + dA[3].x * a0[j].w + dA[0].y * a1[j].x +
                dA[1].y * a1[j].y + dA[2].y * a1[j].z + dA[3].y * a1[j].w;
      }
      float gsum;
      if (K == 2) {  // first level of a reduce-scatter: lanes with bit 4 set carry slot 1
        const bool hi = lane & 16;
        gsum = (hi ? pj[K - 1] : pj[0]) + __shfl_xor_sync(0xffffffffu, hi ? pj[0] : pj[K - 1], 16);
      } else {
        gsum = pj[0] + __shfl_xor_sync(0xffffffffu, pj[0], 16);
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
      if (lane == 0) rrow[32] = gsum;
      if (K == 2 && lane == 16) rrow[33] = gsum;
    }
  }
}

// The packed kernel's chunk load for a full chunk (16 tokens) of a full tile (64 channels), k == K:
// every thread issues all of its global loads (Δ 2 x 16 B; x, z, g_out 16 B each; a quarter row of
// B_mix or C_mix; one expert index and gate for threads < 16K) before its first shared-memory store,
// so the chunk costs one memory round trip instead of one per loop trip of load_chunk. Only the
// first K expert slots of each token are written; the packed kernel reads no other.
template <int K, typename IO>
__device__ __forceinline__ void load_chunk_pk_full(ChunkTile<IO>& ct, const ScanBwdParams& p, int b, int64_t t0,
                                                   int d0) {
  static_assert(kPkThreads == 128 && kBwdLc == 16 && kBwdCh == 64, "thread-to-item map below");
  const int tid = threadIdx.x;
  const size_t row0 = (size_t)b * p.L + t0;
  const int r0 = tid >> 4, cd = (tid & 15) * 4;  // Δ: items tid and tid + 128 of 16 x 16 float4
  const float4 dl0 = *reinterpret_cast<const float4*>(p.delta + (row0 + r0) * p.D + d0 + cd);
  const float4 dl1 = *reinterpret_cast<const float4*>(p.delta + (row0 + r0 + 8) * p.D + d0 + cd);
  constexpr int per16 = 16 / (int)sizeof(IO), vio = kBwdCh / per16;  // 16-byte items per row
  uint4 xv[2], zv[2], gv[2];
  int rio[2], cio[2];
  constexpr int nio = (kBwdLc * vio + kPkThreads - 1) / kPkThreads;  // 1 (bf16) or 2 (fp32)
#pragma unroll
  for (int a = 0; a < nio; ++a) {
    const int it = tid + a * kPkThreads;
    rio[a] = it / vio;
    cio[a] = (it % vio) * per16;
    const size_t g = (row0 + rio[a]) * p.D + d0 + cio[a];
    xv[a] = *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.x) + g);
    zv[a] = *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.z) + g);
    gv[a] = *reinterpret_cast<const uint4*>(reinterpret_cast<const IO*>(p.g_out) + g);
  }
  // B_mix / C_mix rows of the chunk's 16 tokens are 256 contiguous floats each (N = 16)
  const int bc = tid & 63;
  const float4 bcv = *reinterpret_cast<const float4*>((tid < 64 ? p.B_mix : p.C_mix) + row0 * 16 + 4 * bc);
  int ev = 0;
  float gw = 0.f;
  if (tid < kBwdLc * K) {
    ev = min(max(p.idx[row0 * K + tid], 0), p.E - 1);
    gw = p.gates[row0 * K + tid];
  }
  *reinterpret_cast<float4*>(&ct.dl[r0][cd]) = dl0;
  *reinterpret_cast<float4*>(&ct.dl[r0 + 8][cd]) = dl1;
#pragma unroll
  for (int a = 0; a < nio; ++a) {
    *reinterpret_cast<uint4*>(&ct.x[rio[a]][cio[a]]) = xv[a];
    *reinterpret_cast<uint4*>(&ct.z[rio[a]][cio[a]]) = zv[a];
    *reinterpret_cast<uint4*>(&ct.go[rio[a]][cio[a]]) = gv[a];
  }
  *reinterpret_cast<float4*>(tid < 64 ? &ct.B[bc >> 2][4 * (bc & 3)] : &ct.C[bc >> 2][4 * (bc & 3)]) = bcv;
  if (tid < kBwdLc * K) {
    ct.e[tid / K][tid % K] = ev;
    ct.g[tid / K][tid % K] = gw;
  }
}

// Tensor-memory columns for the packed kernel's A rows: 8 per expert, rounded up to a power of two
// of at least 32 (the allocation unit).
__host__ __device__ constexpr uint32_t pk_tmem_cols(int E) { return E * 8 <= 32 ? 32u : (E * 8 <= 64 ? 64u : 128u); }

// The chunk walk of the packed layout (same order as scan_bwd_kernel: the forward through each chunk
// from its checkpoint, then the adjoint one sub-block at a time). Shared memory:
// dAacc[E][2][128 threads] float4 | red[4 warps][16][rw] | tile (thread-fastest layouts: the
// 16-byte accesses are free of bank conflicts), 55 KB at E = 8 with bf16 io; the A rows live in
// tensor memory (load_a2_tm) and the state before each sub-block in a per-CTA global scratch
// (p.sub, [4][2][128 threads] float4, written and read back by the same thread; 16 KB per CTA, so
// it stays in L2). The adjoint recomputes each token's exp(Δ A) instead of keeping the sub-block's
// 16 float2 of them: at most 128 registers. Four CTAs per SM (16 warps) against three with the sub-block
// states in shared memory and the exponentials kept (156 registers): 10.4 -> 8.3 ms on the
// Mamba-1.4B-like shape, for one more exponential per state element.
template <typename IO, int K>
__global__ void __launch_bounds__(kPkThreads, 4) scan_bwd_pk_kernel(ScanBwdParams p) {
  extern __shared__ __align__(16) float smem_pk[];
  __shared__ uint32_t tm_slot;
  float* dAacc = smem_pk;
  float* red = dAacc + p.E * kPkThreads * 8;
  float4* sub = reinterpret_cast<float4*>(p.sub) + (size_t)blockIdx.x * (kBwdLc / kBwdSub) * kPkThreads * 2;
  const int rw = 2 * 16 + K;  // per token: dB[16], dC[16], dgates[K]
  ChunkTile<IO>& ct = *reinterpret_cast<ChunkTile<IO>*>(red + kPkWarps * kBwdLc * rw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q = lane & 3;
  const int c0 = 16 * warp + 2 * (lane >> 2);
  const int tiles = (p.D + kBwdCh - 1) / kBwdCh;
  const int tile = blockIdx.x % tiles, b = blockIdx.x / tiles;
  const int d0 = tile * kBwdCh, nc = min(kBwdCh, p.D - d0);  // nc % 16 == 0
  const bool valid = 16 * warp < nc;                         // whole warps
  // the A rows of every expert for the lane's channels and quarter in tensor memory (8 columns per
  // expert), which keeps the shared memory of a CTA small enough for four CTAs per SM
  const uint32_t tm_cols = pk_tmem_cols(p.E);
  if (warp == 0) {
    sm100::tmem_alloc(&tm_slot, tm_cols);
    sm100::tmem_relinquish();
  }
  for (int i = tid; i < p.E * kPkThreads * 8; i += kPkThreads) dAacc[i] = 0.f;
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tm_lane = tm_slot + ((uint32_t)(32 * warp) << 16);
  for (int e = 0; e < p.E; ++e) {
    float4 u0 = make_float4(0.f, 0.f, 0.f, 0.f), u1 = u0;
    if (valid) {
      const float* src = p.A + ((size_t)e * p.D + d0 + c0) * 16 + 4 * q;
      u0 = __ldg(reinterpret_cast<const float4*>(src));
      u1 = __ldg(reinterpret_cast<const float4*>(src + 16));
    }
    const uint32_t r[8] = {__float_as_uint(u0.x), __float_as_uint(u0.y), __float_as_uint(u0.z), __float_as_uint(u0.w),
                           __float_as_uint(u1.x), __float_as_uint(u1.y), __float_as_uint(u1.z), __float_as_uint(u1.w)};
    sm100::tmem_st8(tm_lane + (uint32_t)e * 8u, r);
  }
  sm100::tmem_wait_st();  // each warp reads back only what its own lanes wrote
  const float2 dsk = valid ? *reinterpret_cast<const float2*>(p.D_skip + d0 + c0) : make_float2(0.f, 0.f);
  float2 carry[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 dD = make_float2(0.f, 0.f);

  for (int ck = p.nck - 1; ck >= 0; --ck) {
    const int64_t t0 = (int64_t)ck * kBwdLc;
    const int nt = (int)(p.L - t0 < kBwdLc ? p.L - t0 : kBwdLc);
    __syncthreads();  // the previous chunk's tile and partial sums are no longer read
    if (nt == kBwdLc && nc == kBwdCh && p.k == K) load_chunk_pk_full<K>(ct, p, b, t0, d0);
    else load_chunk(ct, p, b, t0, nt, d0, nc, true);
    float2 h[4];
    {
      float4 u0 = make_float4(0.f, 0.f, 0.f, 0.f), u1 = u0;
      if (valid) {
        const float* src = p.ckpt + (((size_t)b * p.nck + ck) * p.D + d0 + c0) * 16 + 4 * q;
        u0 = *reinterpret_cast<const float4*>(src);
        u1 = *reinterpret_cast<const float4*>(src + 16);
      }
      h[0] = make_float2(u0.x, u1.x);
      h[1] = make_float2(u0.y, u1.y);
      h[2] = make_float2(u0.z, u1.z);
      h[3] = make_float2(u0.w, u1.w);
    }
    __syncthreads();
    if (valid) {
      // ---- forward through the chunk: the state before every sub-block, and dz ----
      // (one token; lanes q = 0, 1 write dz of channel c0 + q, lanes 2, 3 compute the same and skip
      // the store, so the body has no branch)
      auto fwd_token = [&](int i) {
        float4 a0[K], a1[K];
        load_a2_tm<K>(ct, tm_lane, i, a0, a1);
        float2 at[4];
        mix_a2<K>(ct, a0, a1, i, at);
        const float2 dl = ld2(ct.dl[i], c0), xv = ld2(ct.x[i], c0);
        const float2 c2 = __fmul2_rn(dl, f2s(kLog2e)), dx = __fmul2_rn(dl, xv);
        float2 y = make_float2(0.f, 0.f);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          h[s] = __ffma2_rn(ex2_2(__fmul2_rn(c2, at[s])), h[s], __fmul2_rn(dx, f2s(ct.B[i][4 * q + s])));
          y = __ffma2_rn(f2s(ct.C[i][4 * q + s]), h[s], y);
        }
        y.x += __shfl_xor_sync(0xffffffffu, y.x, 1);
        y.y += __shfl_xor_sync(0xffffffffu, y.y, 1);
        y.x += __shfl_xor_sync(0xffffffffu, y.x, 2);
        y.y += __shfl_xor_sync(0xffffffffu, y.y, 2);
        const int ch = c0 + (q & 1);
        const float zv = to_f32(ct.z[i][ch]), go = to_f32(ct.go[i][ch]);
        const float yy = fmaf(q & 1 ? dsk.y : dsk.x, q & 1 ? xv.y : xv.x, q & 1 ? y.y : y.x);
        const float sg = sigmoid_f(zv);
        if (q < 2) p.dz[((size_t)b * p.L + t0 + i) * p.D + d0 + ch] = go * yy * sg * fmaf(zv, 1.f - sg, 1.f);
      };
      for (int i0 = 0; i0 < nt; i0 += kBwdSub) {
        float4* sv = sub + (i0 / kBwdSub) * 2 * kPkThreads + tid;
        sv[0] = make_float4(h[0].x, h[0].y, h[1].x, h[1].y);
        sv[kPkThreads] = make_float4(h[2].x, h[2].y, h[3].x, h[3].y);
        if (nt - i0 >= kBwdSub) {
#pragma unroll
          for (int u = 0; u < kBwdSub; ++u) fwd_token(i0 + u);
        } else {
          for (int i = i0; i < nt; ++i) fwd_token(i);
        }
      }
      // ---- the adjoint back through the chunk, one sub-block at a time ----
      for (int sb = (nt - 1) / kBwdSub; sb >= 0; --sb) {
        const int i0 = sb * kBwdSub;
        const int ni = nt - i0 < kBwdSub ? nt - i0 : kBwdSub;
        const float4* sv = sub + sb * 2 * kPkThreads + tid;
        const float4 v0 = sv[0], v1 = sv[kPkThreads];
        const float2 h_in[4] = {make_float2(v0.x, v0.y), make_float2(v0.z, v0.w), make_float2(v1.x, v1.y),
                                make_float2(v1.z, v1.w)};
        if (ni == kBwdSub)
          adjoint_sub_pk<K, true>(p, ct, tm_lane, dAacc, red, rw, i0, ni, h_in, t0, b, d0, c0, valid, dsk, tid, warp,
                                  lane, q, carry, dD);
        else
          adjoint_sub_pk<K, false>(p, ct, tm_lane, dAacc, red, rw, i0, ni, h_in, t0, b, d0, c0, valid, dsk, tid, warp,
                                   lane, q, carry, dD);
      }
    } else {
      for (int v = lane; v < nt * rw; v += 32) red[(size_t)warp * kBwdLc * rw + v] = 0.f;
    }
    __syncthreads();
    // the chunk's per-token sums over the CTA's warps -> this tile's partial
    for (int v = tid; v < nt * rw; v += kPkThreads) {
      const int i = v / rw, w = v % rw;
      float sum = 0.f;
#pragma unroll
      for (int wp = 0; wp < kPkWarps; ++wp) sum += red[((size_t)wp * kBwdLc + i) * rw + w];
      const size_t tok = (size_t)b * p.L + t0 + i;
      p.part[((size_t)tile * p.B * p.L + tok) * rw + w] = sum;
    }
  }
  if (valid) {
    if (p.dh0 != nullptr) {
      float* dst = p.dh0 + ((size_t)b * p.D + d0 + c0) * 16 + 4 * q;
      *reinterpret_cast<float4*>(dst) = make_float4(carry[0].x, carry[1].x, carry[2].x, carry[3].x);
      *reinterpret_cast<float4*>(dst + 16) = make_float4(carry[0].y, carry[1].y, carry[2].y, carry[3].y);
    }
    for (int e = 0; e < p.E; ++e) {
      const float4* acc = reinterpret_cast<const float4*>(dAacc) + (size_t)e * 2 * kPkThreads + tid;
      float* dst = p.part_A + (((size_t)b * p.E + e) * p.D + d0 + c0) * 16 + 4 * q;
      *reinterpret_cast<float4*>(dst) = acc[0];
      *reinterpret_cast<float4*>(dst + 16) = acc[kPkThreads];
    }
    if (q == 0) *reinterpret_cast<float2*>(p.part_D + (size_t)b * p.D + d0 + c0) = dD;
  }
  sm100::tc_fence_before();
  __syncthreads();  // every warp's tensor-memory loads have completed (each waited for its own)
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tm_slot, tm_cols);
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

// The packed pair; fast_ckpt: the checkpoints come from the forward's fast scan (bf16 x), whose
// chunk walk (TMA ring, A rows in tensor memory, one warp per 16 channels) runs the recurrence in
// about half the time of scan_bwd_ckpt_pk_kernel.
template <typename IO, int K>
cudaError_t launch_bwd_pk(const ScanBwdParams& p, unsigned grid, size_t smem_ck, size_t smem_bw, bool fast_ckpt,
                          cudaStream_t s) {
  cudaError_t e;
  if (fast_ckpt) {
    ScanParams sp{};
    sp.x = p.x;
    sp.z = p.z;
    sp.delta = p.delta;
    sp.B_mix = p.B_mix;
    sp.C_mix = p.C_mix;
    sp.idx = p.idx;
    sp.gates = p.gates;
    sp.A = p.A;
    sp.D_skip = p.D_skip;
    sp.h0 = p.h0;
    sp.L = p.L;
    sp.B = p.B;
    sp.D = p.D;
    sp.N = p.N;
    sp.E = p.E;
    sp.k = p.k;
    if ((e = run_scan_fast_ckpt(sp, p.ckpt, p.nck, p.status, s)) != cudaSuccess) return e;
  } else {
    if ((e = cudaFuncSetAttribute(scan_bwd_ckpt_pk_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem_ck)) != cudaSuccess)
      return e;
    scan_bwd_ckpt_pk_kernel<IO, K><<<grid, kPkThreads, smem_ck, s>>>(p);
  }
  if ((e = cudaFuncSetAttribute(scan_bwd_pk_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_bw)) != cudaSuccess)
    return e;
  scan_bwd_pk_kernel<IO, K><<<grid, kPkThreads, smem_bw, s>>>(p);
  return cudaGetLastError();
}

// The packed kernel's per-CTA scratch: the state before each 4-token sub-block of the current chunk
// (written by the forward through the chunk, read back by the same thread in the adjoint; it stays in
// L2).
static size_t sub_bytes(int64_t ctas) { return (size_t)ctas * (kBwdLc / kBwdSub) * kPkThreads * 2 * sizeof(float4); }

size_t scan_bwd_workspace(int64_t B, int64_t L, int D, int N, int E, int k) {
  const int64_t tiles = (D + kBwdCh - 1) / kBwdCh;
  const int64_t nck = (L + kBwdLc - 1) / kBwdLc;
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  return up((size_t)B * nck * D * N * 4) + up((size_t)tiles * B * L * (2 * N + k) * 4) +
         up((size_t)B * E * D * N * 4) + up((size_t)B * D * 4) + up(sub_bytes(tiles * B));
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
  w += up((size_t)p.B * p.D * 4);
  p.sub = reinterpret_cast<float*>(w);
  const unsigned grid = (unsigned)(tiles * p.B);
  const size_t a_bytes = sizeof(float) * (size_t)p.E * kBwdCh * 16;
  const size_t tile_bytes = io_bf16 ? sizeof(ChunkTile<__nv_bfloat16>) : sizeof(ChunkTile<float>);
  const size_t smem_ck = a_bytes + tile_bytes;
  const size_t smem_bw = a_bytes + sizeof(float) * ((size_t)p.E * 256 * 4 + (size_t)kBwdWarps * kBwdLc * (2 * p.N + p.k)) +
                         sizeof(float4) * (kBwdLc / kBwdSub) * 256 + tile_bytes;
  cudaError_t e;
  // packed layout: N = 16, k <= 2, whole 16-channel warps
  const bool packed = p.N == 16 && (p.k == 1 || p.k == 2) && p.D % 16 == 0;
  const size_t smem_pk = sizeof(float) * ((size_t)p.E * kPkThreads * 8 + (size_t)kPkWarps * kBwdLc * (32 + p.k)) +
                         tile_bytes;
  const bool fast_ckpt = packed && io_bf16 && scan_fast_plan(p.B, p.L, p.D, p.N, p.E, p.k, true).fast;
  if (packed) {
    if (io_bf16) {
      e = p.k == 1 ? launch_bwd_pk<__nv_bfloat16, 1>(p, grid, smem_ck, smem_pk, fast_ckpt, s)
                   : launch_bwd_pk<__nv_bfloat16, 2>(p, grid, smem_ck, smem_pk, fast_ckpt, s);
    } else {
      e = p.k == 1 ? launch_bwd_pk<float, 1>(p, grid, smem_ck, smem_pk, false, s)
                   : launch_bwd_pk<float, 2>(p, grid, smem_ck, smem_pk, false, s);
    }
  } else if (io_bf16) {
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
  note_launch(fast_ckpt ? 2 : 3);  // (the fast scan's checkpoint pass counts itself)
  return cudaGetLastError();
}

}  // namespace swimba
