// Backward pass of the mixed expert projection and of the router.
//
// Source of the forward: "Swimba: Switch Mamba Model Scales State Space Models", §2 "Generación de
// Parámetros" / "Mezcla en el Espacio de Parámetros" (es), "Kernmechanisme van Swimba" (nl): per
// active expert e_j of token t, v_j = x_t W_x^{e_j} = [dt_low_j | B_j | C_j],
// dt_j = dt_low_j W_dt^{e_j} + b_dt^{e_j}; the streams mix with the gates g_j; Δ = softplus(Σ g_j dt_j).
// The router's gates are the softmax of the k selected logits of x W_r. The pages give no training
// details; these are the exact gradients of that forward (reverse mode), with bf16 MMA operands:
//   g_dt      = ∂L/∂Δ σ(dt_mix) = ∂L/∂Δ (1 − e^{−Δ})               (Δ = softplus(dt_mix))
//   q_j       = W_dt^{e_j} g_dt                                     [R]
//   ∂L/∂g_j   = dt_low_j · q_j + b_dt^{e_j} · g_dt + B_j · ∂L/∂B_mix + C_j · ∂L/∂C_mix
//   dV_j      = [g_j q_j | g_j ∂L/∂B_mix | g_j ∂L/∂C_mix]            [R + 2N]
//   ∂L/∂x    += Σ_j W_x^{e_j} dV_j;   ∂L/∂W_x^e = Σ_{(t,j): e} x_tᵀ dV_j
//   ∂L/∂W_dt^e = Σ_{(t,j): e} (g_j dt_low_j)ᵀ g_dt;   ∂L/∂b_dt^e = Σ_{(t,j): e} g_j g_dt
//   router: ∂L/∂s_j = g_j (∂L/∂g_j − Σ_i g_i ∂L/∂g_i) on the selected logits s;
//           ∂L/∂x += Σ_e ∂L/∂logit_e W_r[:, e];  ∂L/∂W_r = Σ_t x_tᵀ ∂L/∂logits_t.
//
// Layout of the work: the (token, slot) pairs are sorted by expert (a stable counting sort), so
// every product above is a dense GEMM per expert on contiguous rows, run by the library's tcgen05
// GEMM (gemm.cu) in its transposed-operand forms: the rows' x and g_dt are gathered once into bf16
// matrices Xg and G; v (recomputed, fp32) = Xg W_x^e and q = G W_dt^eᵀ; then a per-pair kernel forms
// dV, g_j dt_low (with g_j appended as an extra column, so that the W_dt GEMM also yields the bias
// gradient) and the gate gradient; then Xgᵀ dV = ∂L/∂W_x^e, (g dt_low | g)ᵀ G = [∂L/∂W_dt^e ; ∂L/∂b_dt^e],
// dV W_x^eᵀ = the pairs' input gradients, scattered straight into ∂L/∂x rows by the GEMM's epilogue
// (expert after expert: deterministic). The experts' independent GEMMs run side by side on a few
// internal streams. The expert sizes are read back to the host once per call (so the GEMM shapes
// are exact); that makes this entry point synchronise its stream, unlike the forward ones.
#include <mutex>

#include <type_traits>

#include "common.cuh"

namespace swimba {

cudaError_t run_gemm_tc(bool a_t, bool b_t, bool f32_out, int M, int N, int K, const void* A, int lda, const void* B,
                        int ldb, void* C0, int ldc0, void* C1, int ldc1, int split, const void* R, int ldr,
                        void* status, cudaStream_t s, const int* rows, int rows_div);

namespace {

constexpr int kMaxE = 16;

// Stable counting sort of the P = T k pairs by expert over blocks of kPairBlock pairs, three
// kernels: per-block counts per expert; one CTA turning them into the experts' sizes and offsets and
// every block's first row per expert; each block placing its pairs at that row plus their rank
// among the block's earlier pairs of the expert (warp match + per-warp counts). perm[row] = pair,
// inv[pair] = row, counts[e] = pairs of expert e, offsets[e] = first row of expert e; inside an
// expert the rows keep ascending pair order, whatever the scheduling.
constexpr int kPairBlock = 1024;

__global__ void __launch_bounds__(kPairBlock) pair_count_kernel(const int32_t* idx, int64_t P, int E, int* bhist) {
  __shared__ int hist[kMaxE];
  if (threadIdx.x < kMaxE) hist[threadIdx.x] = 0;
  __syncthreads();
  const int64_t p = (int64_t)blockIdx.x * kPairBlock + threadIdx.x;
  if (p < P) atomicAdd(&hist[min(max(idx[p], 0), E - 1)], 1);
  __syncthreads();
  if (threadIdx.x < E) bhist[(size_t)blockIdx.x * E + threadIdx.x] = hist[threadIdx.x];
}

// One CTA, a warp per expert: the expert's total over the blocks, then (after the offsets) an
// exclusive scan of its per-block counts, 32 blocks at a time.
__global__ void __launch_bounds__(32 * kMaxE) pair_scan_kernel(const int* bhist, int nb, int E, int* counts,
                                                              int* offsets, int* bbase) {
  __shared__ int s_cnt[kMaxE], s_off[kMaxE];
  const int lane = threadIdx.x & 31, e = threadIdx.x >> 5;
  if (e < E) {
    int c = 0;
    for (int bb = lane; bb < nb; bb += 32) c += bhist[(size_t)bb * E + e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) s_cnt[e] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0;
    for (int x = 0; x < E; ++x) {
      s_off[x] = o;
      counts[x] = s_cnt[x];
      offsets[x] = o;
      o += s_cnt[x];
    }
    offsets[E] = o;
  }
  __syncthreads();
  if (e < E) {
    int carry = s_off[e];
    for (int b0 = 0; b0 < nb; b0 += 32) {
      const int bb = b0 + lane;
      const int v = bb < nb ? bhist[(size_t)bb * E + e] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (bb < nb) bbase[(size_t)bb * E + e] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

__global__ void __launch_bounds__(kPairBlock) pair_scatter_kernel(const int32_t* idx, int64_t P, int E,
                                                                 const int* bbase, int* perm, int* inv) {
  __shared__ int warpcnt[kPairBlock / 32][kMaxE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kPairBlock / 32) * kMaxE; i += kPairBlock) (&warpcnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t p = (int64_t)blockIdx.x * kPairBlock + threadIdx.x;
  const bool valid = p < P;
  const int e = valid ? min(max(idx[p], 0), E - 1) : -1;
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int lane_rank = __popc(same & ((1u << lane) - 1u));
  if (valid && lane_rank == 0) warpcnt[warp][e] = __popc(same);
  __syncthreads();
  if (!valid) return;
  int row = bbase[(size_t)blockIdx.x * E + e] + lane_rank;
  for (int w = 0; w < warp; ++w) row += warpcnt[w][e];
  perm[row] = (int)p;
  inv[p] = row;
}

// One CTA per token: g_dt = ∂L/∂Δ (1 − e^{−Δ}) is formed once, and each of the token's k pairs gets
// its sorted row: Xg[row] = x[t] (bf16), G[row] = bf16(g_dt), bg[row] = b_dt^e · g_dt (fp32).
constexpr int kMaxK = 16;
// 8 consecutive weights as floats, in one 16-byte load (bf16) or two (fp32); 16-byte aligned.
__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* src, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 4);
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}

template <typename WT>
__global__ void __launch_bounds__(256) proj_bwd_gather_kernel(const __nv_bfloat16* x, const float* delta,
                                                              const float* g_delta, const int32_t* idx,
                                                              const WT* b_dt, const int* inv, int k, int D, int E,
                                                              __nv_bfloat16* Xg, __nv_bfloat16* G, float* bg) {
  const int64_t t = blockIdx.x;
  const __nv_bfloat16* xr = x + t * D;
  float part[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) part[j] = 0.f;
  for (int c = threadIdx.x * 8; c < D; c += 256 * 8) {  // D % 8 == 0
    const uint4 xv = *reinterpret_cast<const uint4*>(xr + c);
    const float4 d0 = *reinterpret_cast<const float4*>(delta + t * D + c);
    const float4 d1 = *reinterpret_cast<const float4*>(delta + t * D + c + 4);
    const float4 g0 = *reinterpret_cast<const float4*>(g_delta + t * D + c);
    const float4 g1 = *reinterpret_cast<const float4*>(g_delta + t * D + c + 4);
    const float dl[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    const float gd[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    float gdt[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) gdt[i] = -gd[i] * expm1f(-dl[i]);
    __nv_bfloat162 hb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) hb[i] = __floats2bfloat162_rn(gdt[2 * i], gdt[2 * i + 1]);
    const uint4 gv = *reinterpret_cast<const uint4*>(hb);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        const int row = inv[t * k + j];
        const int e = min(max(idx[t * k + j], 0), E - 1);
        *reinterpret_cast<uint4*>(Xg + (size_t)row * D + c) = xv;
        *reinterpret_cast<uint4*>(G + (size_t)row * D + c) = gv;
        float bv[8];
        load8(b_dt + (size_t)e * D + c, bv);
#pragma unroll
        for (int i = 0; i < 8; ++i) part[j] = fmaf(gdt[i], bv[i], part[j]);
      }
    }
  }
  __shared__ float wsum[8][kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j < k) {
      float v = part[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5][j] = v;
    }
  }
  __syncthreads();
  if (threadIdx.x < k) {
    float v = 0.f;
    for (int w = 0; w < 8; ++w) v += wsum[w][threadIdx.x];
    bg[inv[t * k + threadIdx.x]] = v;
  }
}

// One CTA (128 threads) per sorted row, after v = Xg W_x^e (XD, fp32 [R + 2N]) and q = G W_dt^eᵀ
// (Q, fp32 [R]): dV[row] = bf16[g q | g ∂L/∂B | g ∂L/∂C]; DTs[row] = bf16[g dt_low | g | 0 x 7];
// the pair's gate gradient dt_low·q + bg + B·∂L/∂B + C·∂L/∂C.
__global__ void __launch_bounds__(128) proj_bwd_pair_kernel(const float* XD, const float* Q, const float* bg,
                                                            const float* gB, const float* gC, const float* gates,
                                                            const int* perm, int k, int R, int N, __nv_bfloat16* dV,
                                                            __nv_bfloat16* DTs, float* dgates) {
  const int row = blockIdx.x;
  const int p = perm[row];
  const int64_t t = p / k;
  const float g = gates[p];
  const int W = R + 2 * N;
  const float* xd = XD + (size_t)row * W;
  const float* q = Q + (size_t)row * R;
  float part = 0.f;
  for (int i = threadIdx.x; i < W; i += 128) {
    float dv;
    if (i < R) {
      dv = g * q[i];
      part = fmaf(xd[i], q[i], part);
    } else if (i < R + N) {
      const float gb = gB[t * N + i - R];
      dv = g * gb;
      part = fmaf(xd[i], gb, part);
    } else {
      const float gc = gC[t * N + i - R - N];
      dv = g * gc;
      part = fmaf(xd[i], gc, part);
    }
    dV[(size_t)row * W + i] = __float2bfloat16_rn(dv);
  }
  for (int i = threadIdx.x; i < R + 8; i += 128)
    DTs[(size_t)row * (R + 8) + i] = __float2bfloat16_rn(i < R ? g * xd[i] : (i == R ? g : 0.f));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  __shared__ float wsum[4];
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x == 0) dgates[p] = wsum[0] + wsum[1] + wsum[2] + wsum[3] + bg[row];
}

// [∂L/∂W_dt^e ; ∂L/∂b_dt^e] (TMP rows 0..R-1 and R of expert e) -> the caller's arrays.
__global__ void proj_bwd_split_kernel(const float* TMP, int E, int R, int D, float* dW_dt, float* db) {
  const int64_t n = (int64_t)E * (R + 1) * D;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i / ((int64_t)(R + 1) * D), r = (i / D) % (R + 1), d = i % D;
    const float v = TMP[(e * (R + 8) + r) * D + d];
    if (r < R) dW_dt[(e * R + r) * D + d] = v;
    else db[e * D + d] = v;
  }
}

// Router: ∂L/∂logits per token from the gate gradients (the sum of up to two contributions):
// ∂L/∂s_j = g_j (G_j − Σ_i g_i G_i) on the selected logits, zero elsewhere. One thread per token.
__global__ void route_bwd_logits_kernel(const int32_t* idx, const float* gates, const float* gg_a, const float* gg_b,
                                        int64_t T, int E, int k, float* dlogits) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= T) return;
  float mean = 0.f;
  for (int j = 0; j < k; ++j) mean = fmaf(gates[t * k + j], gg_a[t * k + j] + (gg_b ? gg_b[t * k + j] : 0.f), mean);
  for (int e = 0; e < E; ++e) dlogits[t * E + e] = 0.f;
  for (int j = 0; j < k; ++j) {
    const float gg = gg_a[t * k + j] + (gg_b ? gg_b[t * k + j] : 0.f);
    const int e = min(max(idx[t * k + j], 0), E - 1);
    dlogits[t * E + e] += gates[t * k + j] * (gg - mean);
  }
}

// ∂L/∂x[t, d] (+)= Σ_e ∂L/∂logits[t, e] W_r[d, e]: a CTA owns 256 channels (a thread each, its
// W_r row in registers) and a run of 64 tokens, whose ∂L/∂logits rows it stages in shared memory
// (EP = E rounded up to 4 columns, zero-padded, read back as float4 broadcasts); every dx access
// is a coalesced row segment.
constexpr int kDxTok = 64;
template <int EP>
__global__ void __launch_bounds__(256) route_bwd_dx_kernel(const float* W_r, const float* dlogits, int64_t T, int D,
                                                           int E, float* dx, int accumulate) {
  __shared__ __align__(16) float dl[kDxTok][EP];
  const int d = blockIdx.x * 256 + threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.y * kDxTok;
  const int nt = (int)(T - t0 < kDxTok ? T - t0 : kDxTok);
  for (int i = threadIdx.x; i < kDxTok * EP; i += 256) {
    const int r = i / EP, e = i % EP;
    dl[r][e] = (r < nt && e < E) ? dlogits[(t0 + r) * E + e] : 0.f;
  }
  float w[EP];
#pragma unroll
  for (int e = 0; e < EP; ++e) w[e] = (d < D && e < E) ? W_r[(size_t)d * E + e] : 0.f;
  __syncthreads();
  if (d >= D) return;
  // dx is read and written in place, so the compiler may not move a load above an earlier store
  // (one memory round trip per row otherwise): rows go in batches of 8, the next batch's values
  // loaded before the current one is stored
  constexpr int kB = 8;
  float a[kB], an[kB];
#pragma unroll
  for (int i = 0; i < kB; ++i) a[i] = (accumulate && i < nt) ? dx[(t0 + i) * D + d] : 0.f;
  for (int r0 = 0; r0 < nt; r0 += kB) {
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int r = r0 + kB + i;
      an[i] = (accumulate && r < nt) ? dx[(t0 + r) * D + d] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int r = r0 + i;
      if (r < nt) {
        float acc = a[i];
#pragma unroll
        for (int e4 = 0; e4 < EP; e4 += 4) {
          const float4 g = *reinterpret_cast<const float4*>(&dl[r][e4]);
          acc = fmaf(g.x, w[e4], acc);
          acc = fmaf(g.y, w[e4 + 1], acc);
          acc = fmaf(g.z, w[e4 + 2], acc);
          acc = fmaf(g.w, w[e4 + 3], acc);
        }
        dx[(t0 + r) * D + d] = acc;
      }
    }
#pragma unroll
    for (int i = 0; i < kB; ++i) a[i] = an[i];
  }
}

constexpr int kDwTok = 256;  // tokens per partial of ∂L/∂W_r

__device__ __forceinline__ float2 ld2f(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ float2 ld2f(const float* p) { return *reinterpret_cast<const float2*>(p); }

// Partial ∂L/∂W_r over a block of 256 tokens: a CTA owns 512 channels (two per thread, one 2-element
// load per token) and the block's tokens, whose ∂L/∂logits rows it stages in shared memory (EP
// columns, zero-padded, read back as float4 broadcasts); eight tokens' x loads are issued before
// their multiply-adds. The partial goes to part[block][d][e].
template <typename IO, int EP>
__global__ void __launch_bounds__(256) route_bwd_dw_kernel(const IO* x, const float* dlogits, int64_t T, int D, int E,
                                                           float* part) {
  __shared__ __align__(16) float dls[kDwTok][EP];
  const int64_t tb = blockIdx.y, t0 = tb * kDwTok;
  const int nt = (int)(T - t0 < kDwTok ? T - t0 : kDwTok);
  for (int i = threadIdx.x; i < kDwTok * EP; i += 256) {
    const int r = i / EP, e = i % EP;
    dls[r][e] = (r < nt && e < E) ? dlogits[(t0 + r) * E + e] : 0.f;
  }
  __syncthreads();
  const int d = (blockIdx.x * 256 + threadIdx.x) * 2;  // D % 8 == 0: d < D means d + 1 < D
  if (d >= D) return;
  float a0[EP], a1[EP];
#pragma unroll
  for (int e = 0; e < EP; ++e) a0[e] = a1[e] = 0.f;
  constexpr int U = 8;  // divides kDwTok, so rows r0 .. r0 + 7 stay inside dls
  for (int r0 = 0; r0 < nt; r0 += U) {
    float2 xv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) xv[u] = r0 + u < nt ? ld2f(x + (t0 + r0 + u) * D + d) : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int e4 = 0; e4 < EP; e4 += 4) {
        const float4 g = *reinterpret_cast<const float4*>(&dls[r0 + u][e4]);
        a0[e4] = fmaf(xv[u].x, g.x, a0[e4]);
        a0[e4 + 1] = fmaf(xv[u].x, g.y, a0[e4 + 1]);
        a0[e4 + 2] = fmaf(xv[u].x, g.z, a0[e4 + 2]);
        a0[e4 + 3] = fmaf(xv[u].x, g.w, a0[e4 + 3]);
        a1[e4] = fmaf(xv[u].y, g.x, a1[e4]);
        a1[e4 + 1] = fmaf(xv[u].y, g.y, a1[e4 + 1]);
        a1[e4 + 2] = fmaf(xv[u].y, g.z, a1[e4 + 2]);
        a1[e4 + 3] = fmaf(xv[u].y, g.w, a1[e4 + 3]);
      }
    }
  }
  float* dst = part + (tb * D + d) * E;
#pragma unroll
  for (int e = 0; e < EP; ++e)
    if (e < E) {
      dst[e] = a0[e];
      dst[E + e] = a1[e];
    }
}

// ∂L/∂W_r = Σ over the token blocks' partials, in block order.
__global__ void route_bwd_dw_reduce_kernel(const float* part, int64_t nblk, int D, int E, float* dW_r) {
  const int64_t n = (int64_t)D * E;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int64_t b = 0; b < nblk; ++b) s += part[b * n + i];
    dW_r[i] = s;
  }
}

size_t up256(size_t v) { return (v + 255) & ~size_t(255); }

struct ProjBwdLayout {
  size_t counts, offsets, perm, inv, bhist, bbase, bg, Xg, G, XD, Q, dV, DTs, TMP, total;
};

ProjBwdLayout proj_bwd_layout(int64_t T, int D, int R, int N, int E, int k) {
  ProjBwdLayout l{};
  const size_t P = (size_t)T * k, W = (size_t)R + 2 * N;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = up256(o + bytes);
    return at;
  };
  l.counts = take(4 * (kMaxE + 1));
  l.offsets = take(4 * (kMaxE + 1));
  l.perm = take(4 * P);
  l.inv = take(4 * P);
  const size_t nb = (P + kPairBlock - 1) / kPairBlock;
  l.bhist = take(4 * nb * E);
  l.bbase = take(4 * nb * E);
  l.bg = take(4 * P);
  l.Xg = take(2 * P * D);
  l.G = take(2 * P * D);
  l.XD = take(4 * P * W);
  l.Q = take(4 * P * R);
  l.dV = take(2 * P * W);
  l.DTs = take(2 * P * (R + 8));
  l.TMP = take(4 * (size_t)E * (R + 8) * D);
  l.total = o;
  return l;
}


// Side streams (per device, created once) on which the experts' independent GEMMs run side by
// side: one expert's product fills only part of the GPU when its K or N is small.
constexpr int kSideStreams = 4;
struct SideStreams {
  cudaStream_t s[kSideStreams];
  cudaEvent_t fork, join[kSideStreams];
  bool ok = false;
};
SideStreams* side_streams() {
  static std::mutex mu;
  static SideStreams per_dev[16];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  SideStreams& ss = per_dev[dev];
  if (!ss.ok) {
    bool good = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < kSideStreams && good; ++i)
      good = cudaStreamCreateWithFlags(&ss.s[i], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&ss.join[i], cudaEventDisableTiming) == cudaSuccess;
    if (!good) return nullptr;
    ss.ok = true;
  }
  return &ss;
}

cudaError_t fork_to(SideStreams* ss, cudaStream_t s) {
  cudaError_t e = cudaEventRecord(ss->fork, s);
  for (int i = 0; i < kSideStreams && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(ss->s[i], ss->fork, 0);
  return e;
}

cudaError_t join_from(SideStreams* ss, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < kSideStreams && e == cudaSuccess; ++i) {
    e = cudaEventRecord(ss->join[i], ss->s[i]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join[i], 0);
  }
  return e;
}

}  // namespace

size_t proj_bwd_workspace(int64_t T, int D, int R, int N, int E, int k) { return proj_bwd_layout(T, D, R, N, E, k).total; }

cudaError_t run_proj_bwd(const void* x, const float* delta, const float* g_delta, const float* gB, const float* gC,
                         const int32_t* idx, const float* gates, const void* W_x, const void* W_dt, const void* b_dt,
                         bool b_bf16, float* dx, int accumulate, float* dgates, float* dW_x, float* dW_dt, float* db,
                         int64_t T, int D, int R, int N, int E, int k, void* ws, void* status, cudaStream_t s) {
  const ProjBwdLayout l = proj_bwd_layout(T, D, R, N, E, k);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* counts = reinterpret_cast<int*>(w + l.counts);
  int* offsets = reinterpret_cast<int*>(w + l.offsets);
  int* perm = reinterpret_cast<int*>(w + l.perm);
  int* inv = reinterpret_cast<int*>(w + l.inv);
  float* bg = reinterpret_cast<float*>(w + l.bg);
  __nv_bfloat16* Xg = reinterpret_cast<__nv_bfloat16*>(w + l.Xg);
  __nv_bfloat16* G = reinterpret_cast<__nv_bfloat16*>(w + l.G);
  float* XD = reinterpret_cast<float*>(w + l.XD);
  float* Q = reinterpret_cast<float*>(w + l.Q);
  __nv_bfloat16* dV = reinterpret_cast<__nv_bfloat16*>(w + l.dV);
  __nv_bfloat16* DTs = reinterpret_cast<__nv_bfloat16*>(w + l.DTs);
  float* TMP = reinterpret_cast<float*>(w + l.TMP);
  const int64_t P = T * k;
  const int W = R + 2 * N;
  SideStreams* ss = side_streams();
  if (ss == nullptr) return cudaErrorNotReady;
  cudaError_t e;
  const int nb = (int)((P + kPairBlock - 1) / kPairBlock);
  int* bhist = reinterpret_cast<int*>(w + l.bhist);
  int* bbase = reinterpret_cast<int*>(w + l.bbase);
  pair_count_kernel<<<(unsigned)nb, kPairBlock, 0, s>>>(idx, P, E, bhist);
  pair_scan_kernel<<<1, 32 * kMaxE, 0, s>>>(bhist, nb, E, counts, offsets, bbase);
  pair_scatter_kernel<<<(unsigned)nb, kPairBlock, 0, s>>>(idx, P, E, bbase, perm, inv);
  if (b_bf16)
    proj_bwd_gather_kernel<__nv_bfloat16><<<(unsigned)T, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), delta, g_delta, idx, static_cast<const __nv_bfloat16*>(b_dt), inv, k,
        D, E, Xg, G, bg);
  else
    proj_bwd_gather_kernel<float><<<(unsigned)T, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), delta, g_delta,
                                                              idx, static_cast<const float*>(b_dt), inv, k, D, E, Xg,
                                                              G, bg);
  note_launch(4);  // the three sorting kernels and the gather
  if (!accumulate && (e = cudaMemsetAsync(dx, 0, sizeof(float) * (size_t)T * D, s)) != cudaSuccess) return e;
  int h_off[kMaxE + 1];
  if ((e = cudaMemcpyAsync(h_off, offsets, sizeof(int) * (E + 1), cudaMemcpyDeviceToHost, s)) != cudaSuccess) return e;
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const __nv_bfloat16* Wx = static_cast<const __nv_bfloat16*>(W_x);
  const __nv_bfloat16* Wdt = static_cast<const __nv_bfloat16*>(W_dt);
  // v = Xg W_x^e and q = G W_dt^eᵀ per expert, the experts side by side
  if ((e = fork_to(ss, s)) != cudaSuccess) return e;
  for (int ex = 0; ex < E; ++ex) {
    const int o = h_off[ex], n = h_off[ex + 1] - h_off[ex];
    if (n == 0) continue;
    cudaStream_t se = ss->s[ex % kSideStreams];
    if ((e = run_gemm_tc(false, false, true, n, W, D, Xg + (size_t)o * D, D, Wx + (size_t)ex * D * W, W,
                         XD + (size_t)o * W, W, nullptr, 0, W, nullptr, 0, status, se, nullptr, 1)) != cudaSuccess)
      return e;
    if ((e = run_gemm_tc(false, true, true, n, R, D, G + (size_t)o * D, D, Wdt + (size_t)ex * R * D, D,
                         Q + (size_t)o * R, R, nullptr, 0, R, nullptr, 0, status, se, nullptr, 1)) != cudaSuccess)
      return e;
  }
  if ((e = join_from(ss, s)) != cudaSuccess) return e;
  proj_bwd_pair_kernel<<<(unsigned)P, 128, 0, s>>>(XD, Q, bg, gB, gC, gates, perm, k, R, N, dV, DTs, dgates);
  note_launch();
  // the weight gradients, the experts side by side: ∂L/∂W_x^e = Xgᵀ dV (Xg stored [pairs, D] = [K, M]);
  // [∂L/∂W_dt^e ; ∂L/∂b_dt^e] = [g dt_low | g]ᵀ G
  if ((e = fork_to(ss, s)) != cudaSuccess) return e;
  for (int ex = 0; ex < E; ++ex) {
    const int o = h_off[ex], n = h_off[ex + 1] - h_off[ex];
    cudaStream_t se = ss->s[ex % kSideStreams];
    if (n == 0) {  // an expert no token chose has zero weight gradients
      if ((e = cudaMemsetAsync(dW_x + (size_t)ex * D * W, 0, sizeof(float) * (size_t)D * W, se)) != cudaSuccess) return e;
      if ((e = cudaMemsetAsync(TMP + (size_t)ex * (R + 8) * D, 0, sizeof(float) * (size_t)(R + 8) * D, se)) !=
          cudaSuccess)
        return e;
      continue;
    }
    if ((e = run_gemm_tc(true, false, true, D, W, n, Xg + (size_t)o * D, D, dV + (size_t)o * W, W,
                         dW_x + (size_t)ex * D * W, W, nullptr, 0, W, nullptr, 0, status, se, nullptr, 1)) !=
        cudaSuccess)
      return e;
    if ((e = run_gemm_tc(true, false, true, R + 8, D, n, DTs + (size_t)o * (R + 8), R + 8, G + (size_t)o * D, D,
                         TMP + (size_t)ex * (R + 8) * D, D, nullptr, 0, D, nullptr, 0, status, se, nullptr, 1)) !=
        cudaSuccess)
      return e;
  }
  // meanwhile, on the caller's stream, the input gradients dV W_x^eᵀ (W_x^e stored [D, R + 2N] = [N, K]),
  // added straight into dx rows (a token's pairs belong to distinct experts, so one expert's rows
  // never repeat a token; the experts go one after another, in expert order)
  for (int ex = 0; ex < E; ++ex) {
    const int o = h_off[ex], n = h_off[ex + 1] - h_off[ex];
    if (n == 0) continue;
    if ((e = run_gemm_tc(false, true, true, n, D, W, dV + (size_t)o * W, W, Wx + (size_t)ex * D * W, W, dx, D, nullptr,
                         0, D, dx, D, status, s, perm + o, k)) != cudaSuccess)
      return e;
  }
  if ((e = join_from(ss, s)) != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  proj_bwd_split_kernel<<<(unsigned)(2 * sms), 256, 0, s>>>(TMP, E, R, D, dW_dt, db);
  note_launch();
  return cudaGetLastError();
}

size_t route_bwd_workspace(int64_t T, int D, int E) {
  const int64_t nblk = (T + kDwTok - 1) / kDwTok;
  return up256((size_t)T * E * 4) + (size_t)nblk * D * E * 4;
}

cudaError_t run_route_bwd(const void* x, bool io_bf16, const float* W_r, const int32_t* idx, const float* gates,
                          const float* gg_a, const float* gg_b, void* ws, float* dx, int accumulate, float* dW_r,
                          int64_t T, int D, int E, int k, cudaStream_t s) {
  float* dlogits = static_cast<float*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + up256((size_t)T * E * 4));
  const int64_t nblk = (T + kDwTok - 1) / kDwTok;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  route_bwd_logits_kernel<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(idx, gates, gg_a, gg_b, T, E, k, dlogits);
  const dim3 gx((unsigned)((D + 255) / 256), (unsigned)((T + kDxTok - 1) / kDxTok));
  const dim3 gw((unsigned)((D + 511) / 512), (unsigned)nblk);
  auto both = [&](auto ep) {
    constexpr int EP = decltype(ep)::value;
    route_bwd_dx_kernel<EP><<<gx, 256, 0, s>>>(W_r, dlogits, T, D, E, dx, accumulate);
    if (io_bf16)
      route_bwd_dw_kernel<__nv_bfloat16, EP><<<gw, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), dlogits, T, D,
                                                                 E, part);
    else
      route_bwd_dw_kernel<float, EP><<<gw, 256, 0, s>>>(static_cast<const float*>(x), dlogits, T, D, E, part);
  };
  if (E <= 4) both(std::integral_constant<int, 4>{});
  else if (E <= 8) both(std::integral_constant<int, 8>{});
  else if (E <= 12) both(std::integral_constant<int, 12>{});
  else both(std::integral_constant<int, 16>{});
  route_bwd_dw_reduce_kernel<<<(unsigned)(2 * sms), 256, 0, s>>>(part, nblk, D, E, dW_r);
  note_launch(4);
  return cudaGetLastError();
}

}  // namespace swimba
