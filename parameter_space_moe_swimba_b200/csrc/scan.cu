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

// Decode step, N = 16, k <= 2. The state stream (h read and written, 128 bytes per channel and
// sequence) is the step's traffic; the A tables are small and shared by every sequence. So a CTA
// owns a tile of 64 channels and a group of sequences: it stages the A rows of ALL E experts for
// its channels in shared memory once (E x 4 KB, read from L2 once per CTA instead of once per
// sequence), then streams its sequences past them. Thread i owns (channel i / 4, state quarter
// i % 4); it puts two sequences' state quarters, Δ, x, z, B/C quarters and experts in flight
// before it computes any of them, and the four quarters of a channel reduce the readout with two
// shuffles. Two sequences per thread at four CTAs per SM (60 registers) keep more warps in flight
// than four sequences at three CTAs (80 registers): 35.5 against 40.8 µs for 256 sequences in a
// timing probe of the same loop. The grid is one wave: tiles x groups <= the CTAs the SMs hold
// at once, so no CTA waits for a second wave.
constexpr int kStepCh = 64;  // channels per CTA
constexpr int kStepU = 2;    // sequences in flight per thread

template <typename IO, int K>
__global__ void __launch_bounds__(256, 4) step_stream_kernel(ScanParams p, int seq_per_cta) {
  extern __shared__ float4 a_rows[];  // [E][kStepCh][4] float4 = the E experts' A rows of the tile
  const int tid = threadIdx.x, c = tid >> 2, q = tid & 3;
  const int tiles = (p.D + kStepCh - 1) / kStepCh;
  const int tile = blockIdx.x % tiles, grp = blockIdx.x / tiles;
  const int d0 = tile * kStepCh, nc = min(kStepCh, p.D - d0);  // nc % 8 == 0
  for (int i = tid; i < p.E * nc * 4; i += 256) {
    const int e = i / (nc * 4), r = i - e * nc * 4;
    a_rows[e * kStepCh * 4 + r] = __ldg(reinterpret_cast<const float4*>(p.A + ((size_t)e * p.D + d0) * 16) + r);
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // Δ, B_mix, C_mix, the experts and gates of this step have been written
  if (c >= nc) return;  // whole warps (8 channels each) leave together; nothing below synchronises
  const int d = d0 + c;
  const float dsk = p.D_skip[d];
  const int b_begin = grp * seq_per_cta, b_end = min(p.B, b_begin + seq_per_cta);
  for (int bb = b_begin; bb < b_end; bb += kStepU) {
    float4 h4[kStepU], bq[kStepU], cq[kStepU];
    float dl[kStepU], xv[kStepU], zv[kStepU], g0[kStepU], g1[kStepU];
    int e0[kStepU], e1[kStepU];
#pragma unroll
    for (int u = 0; u < kStepU; ++u) {
      const int b = min(bb + u, b_end - 1);  // past the group's end: a repeat of its last sequence, not stored
      const size_t bd = (size_t)b * p.D + d;
      h4[u] = reinterpret_cast<const float4*>(p.h_final)[bd * 4 + q];
      dl[u] = p.delta[bd];
      xv[u] = to_f32(reinterpret_cast<const IO*>(p.x)[bd]);
      zv[u] = to_f32(reinterpret_cast<const IO*>(p.z)[bd]);
      bq[u] = __ldg(reinterpret_cast<const float4*>(p.B_mix + (size_t)b * 16) + q);
      cq[u] = __ldg(reinterpret_cast<const float4*>(p.C_mix + (size_t)b * 16) + q);
      e0[u] = min(max(__ldg(p.idx + (size_t)b * K), 0), p.E - 1);  // indices outside [0, E) are clamped
      g0[u] = __ldg(p.gates + (size_t)b * K);
      if (K == 2) {
        e1[u] = min(max(__ldg(p.idx + (size_t)b * K + 1), 0), p.E - 1);
        g1[u] = __ldg(p.gates + (size_t)b * K + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < kStepU; ++u) {
      if (bb + u >= b_end) break;
      const size_t bd = (size_t)(bb + u) * p.D + d;
      const float4 a0 = a_rows[(e0[u] * kStepCh + c) * 4 + q];
      const float c0 = dl[u] * g0[u] * kLog2e;
      float arg[4] = {c0 * a0.x, c0 * a0.y, c0 * a0.z, c0 * a0.w};
      if (K == 2) {
        const float4 a1 = a_rows[(e1[u] * kStepCh + c) * 4 + q];
        const float c1 = dl[u] * g1[u] * kLog2e;
        arg[0] = fmaf(c1, a1.x, arg[0]);
        arg[1] = fmaf(c1, a1.y, arg[1]);
        arg[2] = fmaf(c1, a1.z, arg[2]);
        arg[3] = fmaf(c1, a1.w, arg[3]);
      }
      float h[4] = {h4[u].x, h4[u].y, h4[u].z, h4[u].w};
      const float bv[4] = {bq[u].x, bq[u].y, bq[u].z, bq[u].w}, cv[4] = {cq[u].x, cq[u].y, cq[u].z, cq[u].w};
      const float dx = dl[u] * xv[u];
      float y = 0.f;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        h[s] = fmaf(ex2_approx(arg[s]), h[s], dx * bv[s]);
        y = fmaf(cv[s], h[s], y);
      }
      y += __shfl_xor_sync(0xffffffffu, y, 1);
      y += __shfl_xor_sync(0xffffffffu, y, 2);
      reinterpret_cast<float4*>(p.h_final)[bd * 4 + q] = make_float4(h[0], h[1], h[2], h[3]);
      if (q == 0) {
        y = fmaf(dsk, xv[u], y);
        if (p.y_pre != nullptr) p.y_pre[bd] = y;
        from_f32(reinterpret_cast<IO*>(p.out)[bd], silu_gate(y, zv[u]));
      }
    }
  }
}

template <typename IO, int K>
static cudaError_t launch_step_stream(const ScanParams& p, cudaStream_t s) {
  const size_t smem = sizeof(float4) * (size_t)p.E * kStepCh * 4;
  cudaError_t e = cudaFuncSetAttribute(step_stream_kernel<IO, K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, step_stream_kernel<IO, K>, 256, smem)) != cudaSuccess)
    return e;
  // every CTA resident at once (one wave): the groups of a tile split the sequences evenly
  const int tiles = (p.D + kStepCh - 1) / kStepCh;
  int groups = std::max(1, std::min(p.B, std::max(1, per_sm) * sms / tiles));
  const int spc = (p.B + groups - 1) / groups;
  groups = (p.B + spc - 1) / spc;
  if ((e = launch_pdl(step_stream_kernel<IO, K>, dim3((unsigned)(tiles * groups)), dim3(256), smem, s, p, spc)) !=
      cudaSuccess)
    return e;
  note_launch();
  return cudaGetLastError();
}

template <typename IO, int K>
static cudaError_t launch_scan(const ScanParams& p, bool step, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)p.E * kDT * kNMax;
  const unsigned gx = (unsigned)((p.D + kDT - 1) / kDT);
  if (step && p.N == kNMax && (K == 1 || K == 2)) return launch_step_stream<IO, (K == 2 ? 2 : 1)>(p, s);
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
