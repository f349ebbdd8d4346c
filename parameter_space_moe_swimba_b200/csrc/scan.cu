// Fused discretise + selective scan + readout + skip + SiLU gate, and the decode step.
//
// Sources: "Swimba: Switch Mamba Model Scales State Space Models" -- one state trajectory and one
// recurrence whatever the number of experts (§2 "Resultado", Teorema 2); the injection and the
// readout use the gate-mixed streams. "Mamba y las SSMs: el retorno del estado persistente",
// "Mamba": selective SSM with Ā = exp(Δ_t A); Figura 2: the state stays on chip while inputs
// stream from HBM; "Estado interno puramente lineal": the linear state admits a scan.
//
// Per token t and channel d (Δ = delta[t, d] already holds softplus(dt_mix)):
//   A_t[d, n] = Σ_j g_j A^{e_j}[d, n]          (per-expert A tables of this CTA's channels in smem)
//   h[d, n]  = exp(Δ A_t[d, n]) h[d, n] + Δ B_mix[t, n] x[t, d]
//   y[t, d]  = Σ_n C_mix[t, n] h[d, n] + D_skip[d] x[t, d];   out = y z σ(z)
//
// Thread layout: a CTA owns 32 channels of one sequence; 4 lanes share a channel and hold 4 of
// its 16 fp32 states each, in registers, for the whole sequence. All lanes of a warp read the
// same token, so the expert indices are warp-uniform. exp is evaluated as 2^(Δ g_j log2(e) A).
#include "common.cuh"
#include "scan.cuh"

namespace swimba {

namespace {
constexpr int kNS = 4;   // states per thread
constexpr int kG = 4;    // threads per channel (16 states / kNS)
constexpr int kDT = 32;  // channels per CTA
constexpr int kNMax = 16;

__device__ __forceinline__ float silu_gate(float y, float z) { return y * z * (1.f / (1.f + __expf(-z))); }

__device__ __forceinline__ void fill_A_table(float* As, const ScanParams& p, int d0) {
  const int total = p.E * kDT * kNMax;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int e = i / (kDT * kNMax);
    const int r = i - e * (kDT * kNMax);
    const int dd = d0 + r / kNMax;
    const int n = r % kNMax;
    As[i] = (dd < p.D && n < p.N) ? __ldg(p.A + ((size_t)e * p.D + dd) * p.N + n) : 0.f;
  }
}

// One token of the recurrence for the 4 states (n0 .. n0+3) of channel d held by this thread.
// Returns the partial readout Σ_{n in thread} C[n] h[n].
template <int K>
__device__ __forceinline__ float token_update(float (&h)[kNS], const float* As, int dl, int n0, float dlt, float xv,
                                              const float (&Bv)[kNS], const float (&Cv)[kNS],
                                              const int32_t* idx_t, const float* g_t, int k, int E, bool zoh) {
  float arg[kNS] = {0.f, 0.f, 0.f, 0.f};
  const int kk = K > 0 ? K : k;
#pragma unroll
  for (int j = 0; j < (K > 0 ? K : 16); ++j) {
    if (K == 0 && j >= kk) break;
    const int e = min(max(__ldg(idx_t + j), 0), E - 1);  // indices outside [0, E) are clamped
    const float c = dlt * __ldg(g_t + j) * kLog2e;
    const float4 a4 = *reinterpret_cast<const float4*>(As + (e * kDT + dl) * kNMax + n0);
    arg[0] = fmaf(c, a4.x, arg[0]);
    arg[1] = fmaf(c, a4.y, arg[1]);
    arg[2] = fmaf(c, a4.z, arg[2]);
    arg[3] = fmaf(c, a4.w, arg[3]);
  }
  const float dx = dlt * xv;
  float y = 0.f;
#pragma unroll
  for (int s = 0; s < kNS; ++s) {
    const float a = ex2_approx(arg[s]);
    const float u = zoh ? dx * Bv[s] * zoh_phi(arg[s], a) : dx * Bv[s];
    h[s] = fmaf(a, h[s], u);
    y = fmaf(Cv[s], h[s], y);
  }
  return y;
}

__device__ __forceinline__ void load_bc(const ScanParams& p, size_t tok, int n0, float (&Bv)[kNS], float (&Cv)[kNS]) {
  if (p.N == kNMax) {
    const float4 b4 = __ldg(reinterpret_cast<const float4*>(p.B_mix + tok * kNMax + n0));
    const float4 c4 = __ldg(reinterpret_cast<const float4*>(p.C_mix + tok * kNMax + n0));
    Bv[0] = b4.x; Bv[1] = b4.y; Bv[2] = b4.z; Bv[3] = b4.w;
    Cv[0] = c4.x; Cv[1] = c4.y; Cv[2] = c4.z; Cv[3] = c4.w;
  } else {
#pragma unroll
    for (int s = 0; s < kNS; ++s) {
      const int n = n0 + s;
      Bv[s] = n < p.N ? __ldg(p.B_mix + tok * p.N + n) : 0.f;
      Cv[s] = n < p.N ? __ldg(p.C_mix + tok * p.N + n) : 0.f;
    }
  }
}
}  // namespace

template <typename IO, int K>
__global__ void __launch_bounds__(128) scan_fwd_kernel(ScanParams p) {
  extern __shared__ float As[];  // [E][kDT][16]
  const int tid = threadIdx.x;
  const int dl = tid / kG, gi = tid % kG;
  const int d0 = blockIdx.x * kDT;
  const int d = d0 + dl;
  const int b = blockIdx.y;
  const int n0 = gi * kNS;
  const bool dvalid = d < p.D;
  const int dc = dvalid ? d : 0;  // clamped channel for loads
  fill_A_table(As, p, d0);
  __syncthreads();

  float h[kNS];
#pragma unroll
  for (int s = 0; s < kNS; ++s)
    h[s] = (p.h0 != nullptr && dvalid && n0 + s < p.N) ? p.h0[((size_t)b * p.D + d) * p.N + n0 + s] : 0.f;
  const float dsk = p.D_skip[dc];
  const IO* x = reinterpret_cast<const IO*>(p.x);
  const IO* z = reinterpret_cast<const IO*>(p.z);
  IO* out = reinterpret_cast<IO*>(p.out);

#pragma unroll 2
  for (int64_t t = 0; t < p.L; ++t) {
    const size_t tok = (size_t)b * p.L + t;
    const float dlt = __ldg(p.delta + tok * p.D + dc);
    const float xv = to_f32(x[tok * p.D + dc]);
    const float zv = to_f32(z[tok * p.D + dc]);
    float Bv[kNS], Cv[kNS];
    load_bc(p, tok, n0, Bv, Cv);
    float y = token_update<K>(h, As, dl, n0, dlt, xv, Bv, Cv, p.idx + tok * p.k, p.gates + tok * p.k, p.k, p.E,
                              p.zoh != 0);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    if (gi == 0 && dvalid) {
      y = fmaf(dsk, xv, y);
      if (p.y_pre != nullptr) p.y_pre[tok * p.D + d] = y;
      from_f32(out[tok * p.D + d], silu_gate(y, zv));
    }
  }
  if (p.h_final != nullptr && dvalid) {
#pragma unroll
    for (int s = 0; s < kNS; ++s)
      if (n0 + s < p.N) p.h_final[((size_t)b * p.D + d) * p.N + n0 + s] = h[s];
  }
}

// Decode step: one token per sequence, state read from and written back to p.h_final (= p.h0).
// The step moves each sequence's state through HBM once (read, then written back), so the kernel
// is built for memory parallelism: one thread per (sequence, channel, 4 states), no shared-memory
// staging, every load of the thread issued before any arithmetic. The selected experts' A rows
// are read straight from the A tables (a few MB, L2-resident across the grid).
template <typename IO, int K>
__global__ void __launch_bounds__(128) step_kernel(ScanParams p) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over (b, d, state group)
  const int gi = (int)(i % kG);
  const int64_t bd = i / kG;
  const bool valid = bd < (int64_t)p.B * p.D;
  const int64_t bdc = valid ? bd : 0;
  const int d = (int)(bdc % p.D);
  const size_t tok = (size_t)(bdc / p.D);  // seqlen == 1: token = sequence
  const int n0 = gi * kNS;
  float* hp = p.h_final + (size_t)bdc * p.N + n0;
  float h[kNS];
  if (p.N == kNMax) {
    const float4 h4 = *reinterpret_cast<const float4*>(hp);
    h[0] = h4.x; h[1] = h4.y; h[2] = h4.z; h[3] = h4.w;
  } else {
#pragma unroll
    for (int s = 0; s < kNS; ++s) h[s] = (n0 + s < p.N) ? hp[s] : 0.f;
  }
  const float dlt = __ldg(p.delta + tok * p.D + d);
  const float xv = to_f32(reinterpret_cast<const IO*>(p.x)[tok * p.D + d]);
  const float zv = to_f32(reinterpret_cast<const IO*>(p.z)[tok * p.D + d]);
  float Bv[kNS], Cv[kNS];
  load_bc(p, tok, n0, Bv, Cv);
  // arg = Σ_j (Δ g_j log2 e) A^{e_j}[d, n]
  float arg[kNS] = {0.f, 0.f, 0.f, 0.f};
  const int kk = K > 0 ? K : p.k;
#pragma unroll
  for (int j = 0; j < (K > 0 ? K : 16); ++j) {
    if (K == 0 && j >= kk) break;
    const int e = min(max(__ldg(p.idx + tok * p.k + j), 0), p.E - 1);
    const float c = dlt * __ldg(p.gates + tok * p.k + j) * kLog2e;
    const float* ar = p.A + ((size_t)e * p.D + d) * p.N + n0;
    float a[kNS];
    if (p.N == kNMax) {
      const float4 a4 = __ldg(reinterpret_cast<const float4*>(ar));
      a[0] = a4.x; a[1] = a4.y; a[2] = a4.z; a[3] = a4.w;
    } else {
#pragma unroll
      for (int s = 0; s < kNS; ++s) a[s] = (n0 + s < p.N) ? __ldg(ar + s) : 0.f;
    }
#pragma unroll
    for (int s = 0; s < kNS; ++s) arg[s] = fmaf(c, a[s], arg[s]);
  }
  const float dx = dlt * xv;
  float y = 0.f;
#pragma unroll
  for (int s = 0; s < kNS; ++s) {
    h[s] = fmaf(ex2_approx(arg[s]), h[s], dx * Bv[s]);
    y = fmaf(Cv[s], h[s], y);
  }
  // the 4 state groups of a channel are 4 consecutive lanes
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  y += __shfl_xor_sync(0xffffffffu, y, 2);
  if (valid) {
    if (p.N == kNMax) {
      *reinterpret_cast<float4*>(hp) = make_float4(h[0], h[1], h[2], h[3]);
    } else {
#pragma unroll
      for (int s = 0; s < kNS; ++s)
        if (n0 + s < p.N) hp[s] = h[s];
    }
    if (gi == 0) {
      y = fmaf(p.D_skip[d], xv, y);
      if (p.y_pre != nullptr) p.y_pre[tok * p.D + d] = y;
      from_f32(reinterpret_cast<IO*>(p.out)[tok * p.D + d], silu_gate(y, zv));
    }
  }
}

// Summary of a whole sequence (the hand-off of one piece of a longer one), for the shapes outside
// the fast path: one thread per (b, d, n) runs the recurrence from zero over every token and sums
// the log decays, h_zero = h_L(0), log_decay = Σ_t Δ_t A_t.
template <typename IO>
__global__ void __launch_bounds__(128) summary_kernel(ScanParams p, float* h_zero, float* log_decay) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over (b, d, n)
  if (i >= (int64_t)p.B * p.D * p.N) return;
  const int n = (int)(i % p.N);
  const int d = (int)((i / p.N) % p.D);
  const int b = (int)(i / ((int64_t)p.N * p.D));
  const IO* x = reinterpret_cast<const IO*>(p.x);
  float h = 0.f, lsum = 0.f;
  for (int64_t t = 0; t < p.L; ++t) {
    const size_t tok = (size_t)b * p.L + t;
    const float dlt = __ldg(p.delta + tok * p.D + d);
    float At = 0.f;
    for (int j = 0; j < p.k; ++j) {
      const int e = min(max(__ldg(p.idx + tok * p.k + j), 0), p.E - 1);
      At = fmaf(__ldg(p.gates + tok * p.k + j), __ldg(p.A + ((size_t)e * p.D + d) * p.N + n), At);
    }
    const float arg = dlt * At;
    lsum += arg;
    h = fmaf(ex2_approx(arg * kLog2e), h, dlt * __ldg(p.B_mix + tok * p.N + n) * to_f32(x[tok * p.D + d]));
  }
  h_zero[i] = h;
  log_decay[i] = lsum;
}

// Start states of consecutive pieces: one thread per (b, d, n) walks the pieces in order.
__global__ void chain_kernel(int64_t BDN, int P, const float* h_zero, const float* log_decay, const float* h0,
                             float* h_start) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BDN) return;
  float H = h0 != nullptr ? h0[i] : 0.f;
  h_start[i] = H;
  for (int q = 0; q < P; ++q) {
    H = fmaf(ex2_approx(log_decay[q * BDN + i] * kLog2e), H, h_zero[q * BDN + i]);
    h_start[(q + 1) * BDN + i] = H;
  }
}

cudaError_t run_scan_summary(const ScanParams& p, bool io_bf16, float* h_zero, float* log_decay, cudaStream_t s) {
  const int64_t n = (int64_t)p.B * p.D * p.N;
  const unsigned grid = (unsigned)((n + 127) / 128);
  if (io_bf16)
    summary_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(p, h_zero, log_decay);
  else
    summary_kernel<float><<<grid, 128, 0, s>>>(p, h_zero, log_decay);
  note_launch();
  return cudaGetLastError();
}

cudaError_t run_scan_chain(int64_t BDN, int P, const float* h_zero, const float* log_decay, const float* h0,
                           float* h_start, cudaStream_t s) {
  chain_kernel<<<(unsigned)((BDN + 255) / 256), 256, 0, s>>>(BDN, P, h_zero, log_decay, h0, h_start);
  note_launch();
  return cudaGetLastError();
}

// Decode step, N = 16, k <= 2: a CTA owns a tile of up to 256 channels of one sequence. Its 256
// threads first put the whole tile's inputs in flight with cp.async 16-byte copies into shared memory
// -- the state tile (16 KB), Δ, x, z, B_mix, C_mix -- then, once thread 0 has read the token's
// experts, the two selected experts' A tiles (16 KB each, L2-resident tables). The copies need no
// registers, so every SM keeps tens of KB of the state stream in flight (the per-thread loads of
// step_kernel above kept a few KB). Then thread i computes 4 (channel, state quarter) items of the
// tile from shared memory, the four quarters of a channel reduce the readout with two shuffles,
// and the new state goes back to HBM with coalesced 16-byte stores. The waits are the hardware's
// cp.async group waits (no spin).
constexpr int kStepTile = 256;  // channels per CTA

__device__ __forceinline__ void cp_async16_s(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}

template <typename IO, int K>
__global__ void __launch_bounds__(256) step_bulk_kernel(ScanParams p) {
  extern __shared__ __align__(16) uint8_t ssm[];
  float* hs = reinterpret_cast<float*>(ssm);             // [256][16]
  float* a0s = hs + kStepTile * 16;                        // [256][16]
  float* a1s = a0s + kStepTile * 16;                       // [256][16]
  float* ds = a1s + kStepTile * 16;                        // [256]
  float* bcs = ds + kStepTile;                             // [32]: B_mix, C_mix
  IO* xs = reinterpret_cast<IO*>(bcs + 32);                // [256]
  IO* zs = xs + kStepTile;                                 // [256]
  __shared__ int sel[2];
  __shared__ float gsel[2];
  const int tid = threadIdx.x;
  const int tiles = (p.D + kStepTile - 1) / kStepTile;
  const int b = blockIdx.x / tiles;
  const int d0 = (blockIdx.x % tiles) * kStepTile;
  const int nc = min(kStepTile, p.D - d0);  // channels of this tile (a multiple of 8)
  const size_t tok = (size_t)b;             // seqlen == 1
  float* hg = p.h_final + ((size_t)b * p.D + d0) * 16;
  // group 0: everything that does not depend on the token's experts
  for (int i = tid; i < nc * 4; i += 256) cp_async16_s(hs + 4 * i, hg + 4 * i);
  for (int i = tid; i < nc / 4; i += 256) cp_async16_s(ds + 4 * i, p.delta + tok * p.D + d0 + 4 * i);
  constexpr int per16 = 16 / (int)sizeof(IO);
  for (int i = tid; i < nc / per16; i += 256) {
    cp_async16_s(xs + per16 * i, reinterpret_cast<const IO*>(p.x) + tok * p.D + d0 + per16 * i);
    cp_async16_s(zs + per16 * i, reinterpret_cast<const IO*>(p.z) + tok * p.D + d0 + per16 * i);
  }
  if (tid < 4) cp_async16_s(bcs + 4 * tid, p.B_mix + tok * 16 + 4 * tid);
  else if (tid < 8) cp_async16_s(bcs + 16 + 4 * (tid - 4), p.C_mix + tok * 16 + 4 * (tid - 4));
  asm volatile("cp.async.commit_group;" ::: "memory");
  if (tid < K) {
    sel[tid] = min(max(__ldg(p.idx + tok * K + tid), 0), p.E - 1);  // indices outside [0, E) are clamped
    gsel[tid] = __ldg(p.gates + tok * K + tid);
  }
  __syncthreads();
  // group 1: the selected experts' A tiles
  const float* A0 = p.A + ((size_t)sel[0] * p.D + d0) * 16;
  for (int i = tid; i < nc * 4; i += 256) cp_async16_s(a0s + 4 * i, A0 + 4 * i);
  if (K == 2) {
    const float* A1 = p.A + ((size_t)sel[1] * p.D + d0) * 16;
    for (int i = tid; i < nc * 4; i += 256) cp_async16_s(a1s + 4 * i, A1 + 4 * i);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  const float g0 = gsel[0], g1 = K == 2 ? gsel[1] : 0.f;
  const int q = tid & 3;
  const float4 bq = reinterpret_cast<const float4*>(bcs)[q];
  const float4 cq = reinterpret_cast<const float4*>(bcs + 16)[q];
  const float bv[4] = {bq.x, bq.y, bq.z, bq.w}, cv[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
  for (int r = 0; r < kStepTile / 64; ++r) {
    const int c = (tid >> 2) + 64 * r;  // channel within the tile
    if (c >= nc) break;                  // nc % 8 == 0: whole quads leave together
    const float4 h4 = reinterpret_cast<const float4*>(hs)[c * 4 + q];
    const float4 x0 = reinterpret_cast<const float4*>(a0s)[c * 4 + q];
    const float dlt = ds[c];
    const float xv = to_f32(xs[c]);
    const float c0 = dlt * g0 * kLog2e;
    float arg[4] = {c0 * x0.x, c0 * x0.y, c0 * x0.z, c0 * x0.w};
    if (K == 2) {
      const float4 x1 = reinterpret_cast<const float4*>(a1s)[c * 4 + q];
      const float c1 = dlt * g1 * kLog2e;
      arg[0] = fmaf(c1, x1.x, arg[0]);
      arg[1] = fmaf(c1, x1.y, arg[1]);
      arg[2] = fmaf(c1, x1.z, arg[2]);
      arg[3] = fmaf(c1, x1.w, arg[3]);
    }
    float h[4] = {h4.x, h4.y, h4.z, h4.w};
    const float dx = dlt * xv;
    float y = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      h[s] = fmaf(ex2_approx(arg[s]), h[s], dx * bv[s]);
      y = fmaf(cv[s], h[s], y);
    }
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    reinterpret_cast<float4*>(hg)[c * 4 + q] = make_float4(h[0], h[1], h[2], h[3]);
    if (q == 0) {
      const int d = d0 + c;
      y = fmaf(p.D_skip[d], xv, y);
      if (p.y_pre != nullptr) p.y_pre[tok * p.D + d] = y;
      from_f32(reinterpret_cast<IO*>(p.out)[tok * p.D + d], silu_gate(y, to_f32(zs[c])));
    }
  }
}

template <typename IO, int K>
static cudaError_t launch_step_bulk(const ScanParams& p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (3 * kStepTile * 16 + kStepTile + 32) + 2 * kStepTile * sizeof(IO);
  cudaError_t e = cudaFuncSetAttribute(step_bulk_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = (p.D + kStepTile - 1) / kStepTile;
  step_bulk_kernel<IO, K><<<(unsigned)(p.B * tiles), 256, smem, s>>>(p);
  note_launch();
  return cudaGetLastError();
}

template <typename IO, int K>
static cudaError_t launch_scan(const ScanParams& p, bool step, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)p.E * kDT * kNMax;
  const unsigned gx = (unsigned)((p.D + kDT - 1) / kDT);
  if (step && p.N == kNMax && (K == 1 || K == 2)) return launch_step_bulk<IO, (K == 2 ? 2 : 1)>(p, s);
  if (step) {
    const int64_t threads = (int64_t)p.B * p.D * kG;
    step_kernel<IO, K><<<(unsigned)((threads + 127) / 128), 128, 0, s>>>(p);
    note_launch();
  } else {
    if (smem > 48 * 1024) {
      cudaError_t e =
          cudaFuncSetAttribute(scan_fwd_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    dim3 grid(gx, (unsigned)p.B);
    scan_fwd_kernel<IO, K><<<grid, 128, smem, s>>>(p);
    note_launch();
  }
  return cudaGetLastError();
}

template <typename IO>
static cudaError_t scan_dispatch(const ScanParams& p, bool step, cudaStream_t s) {
  switch (p.k) {
    case 1: return launch_scan<IO, 1>(p, step, s);
    case 2: return launch_scan<IO, 2>(p, step, s);
    default: return launch_scan<IO, 0>(p, step, s);
  }
}

cudaError_t run_scan(const ScanParams& p, bool io_bf16, bool step, cudaStream_t s) {
  return io_bf16 ? scan_dispatch<__nv_bfloat16>(p, step, s) : scan_dispatch<float>(p, step, s);
}

}  // namespace swimba
