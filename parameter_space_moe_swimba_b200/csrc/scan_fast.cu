// Selective scan over the mixed parameters, B200 fast path (bf16 x/z/out, N = 16, k <= 2, E <= 16).
//
// Sources: "Swimba: Switch Mamba Model Scales State Space Models" -- one state trajectory and ONE
// recurrence whatever the number of experts (§2 "Resultado"; Teorema 2: the recurrence cost does
// not grow with E); "Mamba y las SSMs: el retorno del estado persistente", "Mamba" (Ā = exp(Δ_t A);
// Figura 2: the state stays on chip, inputs stream from HBM) and "Estado interno puramente lineal"
// (the linear state admits a scan, used here to split long sequences into segments).
//
// Per token and state:  arg = Σ_j (Δ g_j) A^{e_j};  ā = 2^arg;  h = ā h + (Δ x) B;  y += C h.
// At N = 16 every (token, channel) costs 16 exponentials and ~80 FP32 operations against 10 bytes
// of HBM traffic, so the kernel is bound by the special-function unit and by instruction issue, not
// by HBM. The design therefore aims at the issue rate: as many resident warps as the SM holds
// (16, at <= 128 registers), the fewest instructions per state element, and packed f32x2 math.
//
// Work unit = one warp = 16 channels of one sequence segment. Lane l holds the channel pair
// (2*(l>>2), 2*(l>>2)+1) and the 4 states 4*(l&3) .. +3 of both channels: state register s is the
// float2 (h[c0][s], h[c1][s]), so every packed operation works on the two channels at once and the
// readout Σ_s C[s] h[s] comes out as the float2 of the two channels' partial sums. B_mix / C_mix
// loads are one 16-byte broadcast per token (8 lanes share each quarter).
// The per-expert transition rows (pre-multiplied by log2 e) live in tensor memory: each warp owns a
// window of its lane quarter, expert e at columns 8e..8e+7 holding (A[c0][s], A[c1][s]) for s = 0..3.
// Every lane of a warp reads the same token, so the selected expert is warp-uniform and one
// tcgen05.ld.32x32b.x8 at column 8e fetches the lane's 8 values: a dynamically indexed, branch-free
// lookup that costs no registers and no shared-memory bandwidth.
//
// A chunk of 16 tokens runs in two passes. The recurrence pass keeps only the state chain; each
// lane leaves its float2 partial readout per token in shared memory. The readout pass then changes
// the lane layout: lane l takes token l/2 and 8 channels, adds the four state quarters' partials,
// the skip term D_skip x and the gate z σ(z) = hz + hz tanh(hz) (hz = z/2), and writes 8 bf16
// outputs; one TMA store per chunk moves the warp's [16 x 16] output tile to HBM (it clips rows
// past L).
//
// Each warp streams its inputs through its own 2-stage ring filled by TMA (x, z, Δ tiles of
// [16 tokens x 16 channels], the tokens' B_mix and C_mix rows) plus the tokens' expert columns and
// gates, which the lanes load one chunk ahead and write into the stage. A chunk's
// compute takes several microseconds, so one chunk in flight hides the HBM latency. Units are
// spread evenly over one persistent CTA per SM.
//
// Segments (when B*D alone cannot fill the GPU): pass 1 computes, per segment, the end state from
// zero and log2 of the decay product Σ_t Δ_t A_t; a carry pass chains them into each segment's
// start state; the main pass then runs every segment from its true start state.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "scan.cuh"
#include "sm100.cuh"

// Tuning knobs, fixed at build time: the warps per SM the segment plan aims at, and the warp count
// per SM below which a sequence is split into segments.
#ifndef SWIMBA_SCAN_TARGET_WARPS
#define SWIMBA_SCAN_TARGET_WARPS 14
#endif
#ifndef SWIMBA_SCAN_MIN_WARPS
#define SWIMBA_SCAN_MIN_WARPS 8
#endif

namespace swimba {

using namespace sm100;

namespace {

constexpr int LC = 16;            // tokens per chunk
constexpr int kStages = 2;        // ring depth per warp
constexpr int kCPW = 16;          // channels per warp
constexpr int kSPL = 4;           // states per lane and channel
constexpr int kMaxWarps = 16;     // warps per CTA (128 registers per thread)
constexpr int kPRow = 4 * kCPW + 4;  // floats per token row of the partial-readout buffer (padded)

// Byte offsets inside one ring stage of one warp (TMA destinations, 128-byte aligned).
struct Stage {
  static constexpr int X = 0;                    // bf16 [LC][16]
  static constexpr int Z = X + LC * kCPW * 2;    // bf16 [LC][16]
  static constexpr int DL = Z + LC * kCPW * 2;   // f32  [LC][16]
  static constexpr int B = DL + LC * kCPW * 4;   // f32  [LC][16]
  static constexpr int C = B + LC * 16 * 4;      // f32  [LC][16]
  static constexpr int META = C + LC * 16 * 4;   // int4 [LC] {TMEM column of e0, of e1, g0, g1}
  static constexpr int BYTES = META + LC * 16;
  static_assert(X % 128 == 0 && Z % 128 == 0 && DL % 128 == 0 && B % 128 == 0 && C % 128 == 0 && META % 128 == 0 &&
                    BYTES % 128 == 0,
                "TMA destinations must be 128-byte aligned");
};

// Per-warp area after the rings: partial readouts and two output tiles (the TMA store of one may
// still be reading while the next is written).
struct Epi {
  static constexpr int P = 0;                        // f32 [LC][kPRow]: [token][channel pair][state quarter][2]
  static constexpr int O = P + LC * kPRow * 4;       // bf16 [2][LC][16]
  static constexpr int BYTES = O + 2 * LC * kCPW * 2;
  static_assert(O % 128 == 0 && BYTES % 128 == 0, "readout area layout");
};

constexpr int kWarpBytes = kStages * Stage::BYTES + Epi::BYTES;

// TMEM columns one warp needs (8 per expert, rounded up to the 32-column allocation granule).
__host__ __device__ constexpr int tmem_cols_per_warp(int E) { return ((E * 8 + 31) / 32) * 32; }

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 8 bf16 (one 16-byte word) as 4 float2 pairs.
__device__ __forceinline__ void bf16x8_to_float2(const uint4 q, float2 (&f)[4]) {
  f[0] = make_float2(bf16lo(q.x), bf16hi(q.x));
  f[1] = make_float2(bf16lo(q.y), bf16hi(q.y));
  f[2] = make_float2(bf16lo(q.z), bf16hi(q.z));
  f[3] = make_float2(bf16lo(q.w), bf16hi(q.w));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float2 v) {
  const __nv_bfloat162 b = __float22bfloat162_rn(v);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }

// One token's scan inputs as the recurrence pass holds them (lane view: channels c0, c1 as the two
// halves of every float2; states 4q .. 4q+3).
struct TokIn {
  int4 m;             // {TMEM column of e0, of e1, g0, g1}
  uint32_t ar[2][8];  // A rows of the selected experts (x log2 e), from TMEM: (c0, c1) per state
  float2 dl, xv;      // Δ and x of the two channels
  float4 bq, cq;      // B_mix, C_mix of the lane's 4 states
  float2 dx;          // Δ x
  float2 a[kSPL];     // 2^arg per state, both channels
  float2 phi[kSPL];   // zero-order-hold factor per state (ZOH only)
};

struct FastParams {
  const int32_t* idx;   // [B, L, k]
  const float* gates;   // [B, L, k]
  const float* A;       // [E, D, 16]
  const float* D_skip;  // [D]
  const float* h0;      // [B, D, 16] or null (start state of segment 0)
  const float* h_seg;   // [B, S, D, 16] start state of every segment (segmented main pass) or null
  float* y_pre;         // [B, L, D] or null
  float* h_final;       // [B, D, 16] or null
  float* agg_h;         // pass 1: [B, S, D, 16] end state from zero
  float* agg_logp;      // pass 1: [B, S, D, 16] log2 of the decay product
  float* ckpt;          // checkpoint pass (AGG kernel, one segment from h0): [B, nck, D, 16] the state at
                        // the start of every 16-token chunk, or null
  int nck;
  void* status;
  int64_t L, Lseg;
  int B, D, E, S;
  int seg_count;        // segments this pass visits (S, or S - 1 for pass 1)
  int units;            // B * seg_count * (D / 16)
  int tmem_cols;        // TMEM columns the CTA allocates
};

// AGG = true: pass 1 (segments 0 .. S-2 only; no readout, no output), or the checkpoint pass of the
// backward (p.ckpt set). ZOH = true: zero-order-hold injection (φ Δ B x, φ = (ā - 1) / (Δ A_t))
// instead of Euler's Δ B x.
template <int K, bool AGG, bool ZOH>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
    scan_fast_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                     const __grid_constant__ CUtensorMap tm_dl, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_o,
                     const FastParams p) {
  using St = Stage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  uint8_t* ring = smem + (size_t)warp * kWarpBytes;
  uint8_t* epi = ring + kStages * St::BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nwarps * kWarpBytes);
  uint64_t* full = bars + warp * kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + nwarps * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + nwarps * kStages) + 1;
  float* psm = reinterpret_cast<float*>(epi + Epi::P);

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    if (warp == 0) {
      *abort_flag = 0;
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_dl);
      prefetch_tmap(&tm_b);
      if (!AGG) {
        prefetch_tmap(&tm_z);
        prefetch_tmap(&tm_c);
        prefetch_tmap(&tm_o);
      }
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  // this warp's TMEM window: its lane quarter, tmem_cols_per_warp(E) columns
  const uint32_t tbase =
      *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(warp >> 2) * (uint32_t)tmem_cols_per_warp(p.E);

  const int cp = lane >> 2;        // recurrence pass: channel pair 2cp, 2cp+1 of the warp's 16
  const int q = lane & 3;          //                  state quarter: states 4q .. 4q+3
  // readout pass: lane = (token rt of the chunk, channels rc .. rc+7 of the warp's 16); the eight
  // lanes of a 16-byte load phase take eight consecutive tokens of one channel half, so their reads
  // of the partial-readout rows (stride 68 floats) fall in eight distinct bank groups (with the two
  // halves of one token in a phase they collided two by two: 10 % of the kernel's shared-memory
  // wavefronts); the x, z and output tile rows (32 bytes) then conflict two ways instead, for a
  // quarter of those wavefronts
  const int rt = lane & 15;
  const int rc = (lane >> 4) * 8;
  const int ntiles = p.D / kCPW;
  const int u_begin = (int)((int64_t)p.units * blockIdx.x / gridDim.x);
  const int u_end = (int)((int64_t)p.units * (blockIdx.x + 1) / gridDim.x);
  uint32_t phase_bits = 0;  // one parity bit per stage
  int ochunk = 0;           // output tiles written by this warp (selects the double buffer)
  constexpr uint32_t tx_bytes = AGG ? (LC * kCPW * 2 + LC * kCPW * 4 + LC * 16 * 4)
                                    : (2 * LC * kCPW * 2 + LC * kCPW * 4 + 2 * LC * 16 * 4);
  const uint32_t emax = (uint32_t)(p.E - 1);

  for (int u = u_begin + warp; u < u_end; u += nwarps) {
    const int tile = u % ntiles;
    const int bs = u / ntiles;  // b * seg_count + seg
    const int seg = bs % p.seg_count;
    const int b = bs / p.seg_count;
    const int dA = tile * kCPW + 2 * cp;  // this lane's channels dA, dA + 1
    const int64_t t_begin = (int64_t)seg * p.Lseg;
    const int64_t t_end = std::min<int64_t>(p.L, t_begin + p.Lseg);
    const int nchunks = (int)((t_end - t_begin + LC - 1) / LC);

    // per-expert transition rows of this lane's 2 channels x 4 states, times log2(e), into TMEM
    // columns 8e + 2s + channel (a copy of the rows in registers behind a warp-uniform switch ran
    // the Mamba-1.4B-like scan in 1627 against 961 µs: spills and branches)
    for (int e = 0; e < p.E; ++e) {
      const float4 a0 = __ldg(reinterpret_cast<const float4*>(p.A + ((size_t)e * p.D + dA) * 16 + 4 * q));
      const float4 a1 = __ldg(reinterpret_cast<const float4*>(p.A + ((size_t)e * p.D + dA + 1) * 16 + 4 * q));
      const uint32_t r[8] = {__float_as_uint(a0.x * kLog2e), __float_as_uint(a1.x * kLog2e),
                             __float_as_uint(a0.y * kLog2e), __float_as_uint(a1.y * kLog2e),
                             __float_as_uint(a0.z * kLog2e), __float_as_uint(a1.z * kLog2e),
                             __float_as_uint(a0.w * kLog2e), __float_as_uint(a1.w * kLog2e)};
      tmem_st8(tbase + (uint32_t)(e * 8), r);
    }
    tmem_wait_st();
    float2 dsk[4];  // readout pass: D_skip of channels rc .. rc+7
    if (!AGG) {
      const float4 d0 = __ldg(reinterpret_cast<const float4*>(p.D_skip + tile * kCPW + rc));
      const float4 d1 = __ldg(reinterpret_cast<const float4*>(p.D_skip + tile * kCPW + rc + 4));
      dsk[0] = make_float2(d0.x, d0.y);
      dsk[1] = make_float2(d0.z, d0.w);
      dsk[2] = make_float2(d1.x, d1.y);
      dsk[3] = make_float2(d1.z, d1.w);
    }

    // start state: (h[c0][s], h[c1][s])
    float2 h[kSPL];
    {
      const float* hs = nullptr;
      if (!AGG || p.ckpt != nullptr) {
        if (p.h_seg != nullptr) hs = p.h_seg + (((size_t)b * p.S + seg) * p.D + dA) * 16;
        else if (p.h0 != nullptr && seg == 0) hs = p.h0 + ((size_t)b * p.D + dA) * 16;
      }
      if (hs != nullptr) {
        const float4 u0 = *reinterpret_cast<const float4*>(hs + 4 * q);
        const float4 u1 = *reinterpret_cast<const float4*>(hs + 16 + 4 * q);
        h[0] = make_float2(u0.x, u1.x);
        h[1] = make_float2(u0.y, u1.y);
        h[2] = make_float2(u0.z, u1.z);
        h[3] = make_float2(u0.w, u1.w);
      } else {
#pragma unroll
        for (int s = 0; s < kSPL; ++s) h[s] = f2(0.f);
      }
    }
    float2 lsum[kSPL];
#pragma unroll
    for (int s = 0; s < kSPL; ++s) lsum[s] = f2(0.f);

    // meta of one chunk: lane t (< LC) holds token t's {TMEM column of e0, of e1, g0, g1}; expert
    // indices outside [0, E) are clamped into the table, tokens past the segment get gate 0
    auto load_meta = [&](int c) -> int4 {
      int4 m = make_int4(0, 0, 0, 0);
      const int64_t t = t_begin + (int64_t)c * LC + lane;
      if (lane < LC && c < nchunks && t < t_end) {
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
    // fill stage (c % kStages) with chunk c: meta from registers, the rest by TMA
    auto issue = [&](int c, int4 m) {
      uint8_t* st = ring + (c % kStages) * St::BYTES;
      if (lane < LC) reinterpret_cast<int4*>(st + St::META)[lane] = m;
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_smem();
        uint64_t* bar = &full[c % kStages];
        mbar_arrive_expect_tx(bar, tx_bytes);
        const int t0 = (int)(t_begin + (int64_t)c * LC);
        tma_load_3d(st + St::X, &tm_x, bar, tile * kCPW, t0, b);
        tma_load_3d(st + St::DL, &tm_dl, bar, tile * kCPW, t0, b);
        tma_load_3d(st + St::B, &tm_b, bar, 0, t0, b);
        if (!AGG) {
          tma_load_3d(st + St::Z, &tm_z, bar, tile * kCPW, t0, b);
          tma_load_3d(st + St::C, &tm_c, bar, 0, t0, b);
        }
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
    int issued = pre;
    int failed_chunk = 0;
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
      const float2* ds2 = reinterpret_cast<const float2*>(st + St::DL);
      const float4* bsm = reinterpret_cast<const float4*>(st + St::B);
      const float4* csm = reinterpret_cast<const float4*>(st + St::C);
      const int64_t t0 = t_begin + (int64_t)c * LC;
      if (AGG && p.ckpt != nullptr) {  // the state before this chunk
        float* ck = p.ckpt + (((size_t)b * p.nck + t0 / LC) * p.D + dA) * 16 + 4 * q;
        *reinterpret_cast<float4*>(ck) = make_float4(h[0].x, h[1].x, h[2].x, h[3].x);
        *reinterpret_cast<float4*>(ck + 16) = make_float4(h[0].y, h[1].y, h[2].y, h[3].y);
      }

      // issue token t's loads (TMEM loads are waited for by the caller)
      auto load_tok = [&](TokIn& tk, int t) {
        tk.m = meta[t];  // (handing it over by warp shuffles from the lanes that load it ran slower)
        tmem_ld8_nowait(tbase + (uint32_t)tk.m.x, tk.ar[0]);
        if (K == 2) tmem_ld8_nowait(tbase + (uint32_t)tk.m.y, tk.ar[1]);
        tk.dl = ds2[t * (kCPW / 2) + cp];
        const uint32_t xw = xs2[t * (kCPW / 2) + cp];
        tk.xv = make_float2(bf16lo(xw), bf16hi(xw));
        tk.bq = bsm[t * 4 + q];
        if (!AGG) tk.cq = csm[t * 4 + q];
      };
      // decay factors of a loaded token (independent of the state)
      auto decay = [&](TokIn& tk) {
        tk.dx = __fmul2_rn(tk.dl, tk.xv);
        const float2 dg0 = __fmul2_rn(tk.dl, f2(__int_as_float(tk.m.z)));
        const float2 dg1 = __fmul2_rn(tk.dl, f2(__int_as_float(tk.m.w)));
#pragma unroll
        for (int s = 0; s < kSPL; ++s) {
          float2 arg =
              __fmul2_rn(dg0, make_float2(__uint_as_float(tk.ar[0][2 * s]), __uint_as_float(tk.ar[0][2 * s + 1])));
          if (K == 2)
            arg = __ffma2_rn(dg1, make_float2(__uint_as_float(tk.ar[1][2 * s]), __uint_as_float(tk.ar[1][2 * s + 1])),
                             arg);
          if (AGG) lsum[s] = __fadd2_rn(lsum[s], arg);  // Σ_t log2 ā_t
          // every exponential on the special-function unit (moving one per lane and token to a
          // polynomial on the FMA pipe ran slower: 1029 against 961 µs)
          const float ax = ex2_approx(arg.x);
          const float ay = ex2_approx(arg.y);
          tk.a[s] = make_float2(ax, ay);
          if (ZOH) tk.phi[s] = make_float2(zoh_phi(arg.x, ax), zoh_phi(arg.y, ay));
        }
      };

      // ---- recurrence pass: the state chain only; partial readouts go to shared memory ----
      // Software-pipelined by one token: while token t updates the state, token t+1's inputs are
      // loaded (its A rows from TMEM, Δ, x, B, C from the ring) and its decay factors computed.
      TokIn cur, nxt;
      load_tok(cur, 0);
      tmem_wait_ld();
      decay(cur);
#pragma unroll
      for (int t = 0; t < LC; ++t) {
        if (t + 1 < LC) load_tok(nxt, t + 1);
        const float bsv[4] = {cur.bq.x, cur.bq.y, cur.bq.z, cur.bq.w};
#pragma unroll
        for (int s = 0; s < kSPL; ++s) {
          float2 u = __fmul2_rn(cur.dx, f2(bsv[s]));
          if (ZOH) u = __fmul2_rn(u, cur.phi[s]);
          h[s] = __ffma2_rn(cur.a[s], h[s], u);
        }
        if (!AGG) {
          float2 y = __fmul2_rn(f2(cur.cq.x), h[0]);
          y = __ffma2_rn(f2(cur.cq.y), h[1], y);
          y = __ffma2_rn(f2(cur.cq.z), h[2], y);
          y = __ffma2_rn(f2(cur.cq.w), h[3], y);
          *reinterpret_cast<float2*>(psm + t * kPRow + cp * 8 + q * 2) = y;
        }
        if (t + 1 < LC) {
          tmem_wait_ld();
          decay(nxt);
          cur = nxt;
        }
      }

      // ---- readout pass: lane = (token rt, channels rc..rc+7) ----
      if (!AGG) {
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
        float2 xf[4], zf[4];
        bf16x8_to_float2(*reinterpret_cast<const uint4*>(st + St::X + (rt * kCPW + rc) * 2), xf);
        bf16x8_to_float2(*reinterpret_cast<const uint4*>(st + St::Z + (rt * kCPW + rc) * 2), zf);
        uint32_t packed[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          yv[i] = __ffma2_rn(dsk[i], xf[i], yv[i]);  // y + D_skip x
          const float2 hz = __fmul2_rn(zf[i], f2(0.5f));
          const float2 th = make_float2(tanh_approx(hz.x), tanh_approx(hz.y));
          const float2 silu = __ffma2_rn(hz, th, hz);  // z σ(z)
          packed[i] = pack_bf16x2(__fmul2_rn(yv[i], silu));
        }
        if (p.y_pre != nullptr && t0 + rt < t_end) {
          float4* yp = reinterpret_cast<float4*>(p.y_pre + ((size_t)b * p.L + t0 + rt) * p.D + tile * kCPW + rc);
          yp[0] = make_float4(yv[0].x, yv[0].y, yv[1].x, yv[1].y);
          yp[1] = make_float4(yv[2].x, yv[2].y, yv[3].x, yv[3].y);
        }
        // the TMA store issued two chunks ago from this output buffer must have read it
        uint8_t* obuf = epi + Epi::O + (ochunk & 1) * (LC * kCPW * 2);
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
      }
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
      if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 31, blockIdx.x, u);
      // let the copies this warp still has in flight (chunks failed_chunk .. issued-1) land before
      // the CTA exits (bounded, ignores the flag)
      for (int c = failed_chunk; c < issued; ++c) {
        const int sidx = c % kStages;
        const uint64_t w0 = globaltimer_ns();
        while (!mbar_try_wait(&full[sidx], (phase_bits >> sidx) & 1u) && globaltimer_ns() - w0 < kWaitLimitNs) {
        }
        phase_bits ^= 1u << sidx;
      }
      break;
    }
    // end state (segment aggregates in pass 1, h_final after the last segment)
    float* hout = nullptr;
    float* lout = nullptr;
    if (AGG && p.ckpt == nullptr) {
      hout = p.agg_h + (((size_t)b * p.S + seg) * p.D + dA) * 16;
      lout = p.agg_logp + (((size_t)b * p.S + seg) * p.D + dA) * 16;
    } else if (p.h_final != nullptr && seg == p.S - 1) {
      hout = p.h_final + ((size_t)b * p.D + dA) * 16;
    }
    if (hout != nullptr) {
      *reinterpret_cast<float4*>(hout + 4 * q) = make_float4(h[0].x, h[1].x, h[2].x, h[3].x);
      *reinterpret_cast<float4*>(hout + 16 + 4 * q) = make_float4(h[0].y, h[1].y, h[2].y, h[3].y);
    }
    if (lout != nullptr) {
      *reinterpret_cast<float4*>(lout + 4 * q) = make_float4(lsum[0].x, lsum[1].x, lsum[2].x, lsum[3].x);
      *reinterpret_cast<float4*>(lout + 16 + 4 * q) = make_float4(lsum[0].y, lsum[1].y, lsum[2].y, lsum[3].y);
    }
    __syncwarp();
  }
  // the output stores must have read their shared-memory tiles before the CTA's memory goes away
  if (!AGG && lane == 0) bulk_wait<0>();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, (uint32_t)p.tmem_cols);
  }
}

// Chain the segments: Hin[s] = start state of segment s; Hin[s+1] = 2^{logp[s]} Hin[s] + h_end[s].
__global__ void scan_carry_kernel(const float* h0, const float* agg_h, const float* agg_logp, float* h_seg, int B,
                                  int S, int D) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over (b, d, n)
  if (i >= (int64_t)B * D * 16) return;
  const int n = (int)(i % 16);
  const int d = (int)((i / 16) % D);
  const int b = (int)(i / (16 * (int64_t)D));
  float H = h0 != nullptr ? h0[((size_t)b * D + d) * 16 + n] : 0.f;
  for (int s = 0; s < S; ++s) {
    const size_t o = (((size_t)b * S + s) * D + d) * 16 + n;
    h_seg[o] = H;
    if (s + 1 < S) H = fmaf(ex2_approx(agg_logp[o]), H, agg_h[o]);
  }
}

// Summary of a whole sequence from its segments' aggregates: the state after the last segment when
// the first starts from zero, H = 2^{logp[s]} H + h_end[s] over s, and the total log decay
// Σ_s logp[s] (log2 units in, natural log out).
__global__ void summary_combine_kernel(const float* agg_h, const float* agg_logp, float* h_zero, float* log_decay,
                                       int B, int S, int D) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // over (b, d, n)
  if (i >= (int64_t)B * D * 16) return;
  const int n = (int)(i % 16);
  const int d = (int)((i / 16) % D);
  const int b = (int)(i / (16 * (int64_t)D));
  float H = 0.f, lp = 0.f;
  for (int s = 0; s < S; ++s) {
    const size_t o = (((size_t)b * S + s) * D + d) * 16 + n;
    H = fmaf(ex2_approx(agg_logp[o]), H, agg_h[o]);
    lp += agg_logp[o];
  }
  h_zero[i] = H;
  log_decay[i] = lp * 0.6931471805599453f;  // ln 2
}

// ---- host ------------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 3-D map over a [B, L, inner] row-major tensor, box {box_inner, LC, 1}.
bool map3(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int64_t inner, int64_t L, int64_t B,
          int box_inner) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t str[2] = {(cuuint64_t)(inner * esize), (cuuint64_t)(inner * L * esize)};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)LC, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int device_sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

// ---- segment plan and workspace ---------------------------------------------------------------------
ScanPlan scan_fast_plan(int64_t B, int64_t L, int D, int N, int E, int k, bool io_bf16) {
  ScanPlan pl{};
  pl.fast = io_bf16 && N == 16 && (k == 1 || k == 2) && E >= 1 && E <= 16;
  if (!pl.fast) return pl;
  if (D % kCPW != 0 || B * L > (int64_t(1) << 31)) {
    pl.fast = false;
    return pl;
  }
  const int64_t sms = device_sms();
  const int64_t base_units = B * (D / kCPW);
  int64_t S = 1;
  if (base_units < sms * SWIMBA_SCAN_MIN_WARPS) {
    const int64_t target = sms * SWIMBA_SCAN_TARGET_WARPS;
    S = std::min<int64_t>((target + base_units - 1) / base_units, (L + LC - 1) / LC);
    S = std::max<int64_t>(S, 1);
  }
  int64_t Lseg = (L + S - 1) / S;
  Lseg = (Lseg + LC - 1) / LC * LC;
  S = (L + Lseg - 1) / Lseg;
  pl.S = (int)S;
  pl.Lseg = Lseg;
  pl.ws_bytes = S > 1 ? (size_t)3 * B * S * D * 16 * sizeof(float) : 0;
  return pl;
}

using FastKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           const CUtensorMap, const CUtensorMap, const FastParams);

template <int K, bool AGG>
static FastKernel pick_kernel(int E, bool zoh) {
  (void)E;
  return zoh ? scan_fast_kernel<K, AGG, true> : scan_fast_kernel<K, AGG, false>;
}

struct FastLaunch {
  CUtensorMap tx, tz, td, tb, tc, to;
  FastParams p;
  int sms, win;
  bool zoh;
};

static bool fast_setup(const ScanParams& sp, const ScanPlan& pl, void* status, FastLaunch& f) {
  if (!map3(&f.tx, sp.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, kCPW) ||
      !map3(&f.td, sp.delta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, sp.D, sp.L, sp.B, kCPW) ||
      !map3(&f.tb, sp.B_mix, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 16, sp.L, sp.B, 16))
    return false;
  // the summary pass reads no z, C_mix or output: its maps repeat x and B_mix
  const void* z = sp.z != nullptr ? sp.z : sp.x;
  const float* C = sp.C_mix != nullptr ? sp.C_mix : sp.B_mix;
  void* out = sp.out != nullptr ? sp.out : const_cast<void*>(sp.x);
  if (!map3(&f.tz, z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, kCPW) ||
      !map3(&f.tc, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 16, sp.L, sp.B, 16) ||
      !map3(&f.to, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, kCPW))
    return false;
  FastParams& p = f.p;
  p = FastParams{};
  p.idx = sp.idx;
  p.gates = sp.gates;
  p.A = sp.A;
  p.D_skip = sp.D_skip;
  p.h0 = sp.h0;
  p.y_pre = sp.y_pre;
  p.h_final = sp.h_final;
  p.status = status;
  p.L = sp.L;
  p.Lseg = pl.Lseg;
  p.B = sp.B;
  p.D = sp.D;
  p.E = sp.E;
  p.S = pl.S;
  p.seg_count = pl.S;
  p.units = sp.B * pl.S * (sp.D / kCPW);
  f.sms = device_sms();
  f.win = tmem_cols_per_warp(sp.E);
  f.zoh = sp.zoh != 0;
  return true;
}

// One persistent CTA per SM; the warps per CTA cover the units (at most kMaxWarps, and at most 4
// windows of `win` TMEM columns per lane quarter); the TMEM allocation covers the CTA's windows.
static cudaError_t fast_shape(const void* fn, int units, int sms, int win, int& ctas, int& warps, int& cols) {
  cudaFuncAttributes fa;
  cudaError_t err = cudaFuncGetAttributes(&fa, fn);
  if (err != cudaSuccess) return err;
  const int wmax = std::max(1, std::min({kMaxWarps, fa.maxThreadsPerBlock / 32, 4 * (512 / win)}));
  ctas = std::max(1, std::min(sms, units));
  warps = std::min(wmax, (units + ctas - 1) / ctas);
  if ((int64_t)ctas * warps < units) ctas = (int)std::min<int64_t>((units + warps - 1) / warps, 65535);
  const int need = ((warps + 3) / 4) * win;
  cols = 32;
  while (cols < need) cols *= 2;
  return cudaSuccess;
}

static size_t fast_smem(int warps) { return 128 + (size_t)warps * (kWarpBytes + kStages * 8) + 16; }

// Pass 1 over `seg_count` segments (from segment 0): end state from zero and log2 decay sums into
// agg_h / agg_logp [B, S, D, 16].
template <int K>
static cudaError_t launch_agg(FastLaunch& f, int seg_count, float* agg_h, float* agg_logp, cudaStream_t s) {
  FastParams a = f.p;
  a.agg_h = agg_h;
  a.agg_logp = agg_logp;
  a.h0 = nullptr;
  a.h_seg = nullptr;
  a.seg_count = seg_count;
  a.units = a.B * seg_count * (a.D / kCPW);
  auto kagg = pick_kernel<K, true>(a.E, f.zoh);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(kagg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fast_smem(kMaxWarps))) !=
      cudaSuccess)
    return e;
  int ctas, warps;
  if ((e = fast_shape((const void*)kagg, a.units, f.sms, f.win, ctas, warps, a.tmem_cols)) != cudaSuccess) return e;
  kagg<<<ctas, warps * 32, fast_smem(warps), s>>>(f.tx, f.tz, f.td, f.tb, f.tc, f.to, a);
  note_launch();
  return cudaGetLastError();
}

template <int K>
static cudaError_t launch_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, cudaStream_t s) {
  FastLaunch f;
  if (!fast_setup(sp, pl, status, f)) return cudaErrorInvalidValue;
  FastParams& p = f.p;
  cudaError_t e;
  if (pl.S > 1) {
    float* agg_h = reinterpret_cast<float*>(seg_ws);
    float* agg_logp = agg_h + (size_t)sp.B * pl.S * sp.D * 16;
    float* h_seg = agg_logp + (size_t)sp.B * pl.S * sp.D * 16;
    if ((e = launch_agg<K>(f, pl.S - 1, agg_h, agg_logp, s)) != cudaSuccess) return e;  // the last needs none
    const int64_t n = (int64_t)sp.B * sp.D * 16;
    scan_carry_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(sp.h0, agg_h, agg_logp, h_seg, sp.B, pl.S, sp.D);
    note_launch();
    p.h_seg = h_seg;
  }
  auto kmain = pick_kernel<K, false>(p.E, sp.zoh != 0);
  if ((e = cudaFuncSetAttribute(kmain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fast_smem(kMaxWarps))) !=
      cudaSuccess)
    return e;
  int ctas, warps;
  if ((e = fast_shape((const void*)kmain, p.units, f.sms, f.win, ctas, warps, p.tmem_cols)) != cudaSuccess) return e;
  kmain<<<ctas, warps * 32, fast_smem(warps), s>>>(f.tx, f.tz, f.td, f.tb, f.tc, f.to, p);
  note_launch();
  return cudaGetLastError();
}

template <int K>
static cudaError_t launch_summary(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status,
                                  float* h_zero, float* log_decay, cudaStream_t s) {
  FastLaunch f;
  if (!fast_setup(sp, pl, status, f)) return cudaErrorInvalidValue;
  float* agg_h = reinterpret_cast<float*>(seg_ws);
  float* agg_logp = agg_h + (size_t)sp.B * pl.S * sp.D * 16;
  cudaError_t e;
  if ((e = launch_agg<K>(f, pl.S, agg_h, agg_logp, s)) != cudaSuccess) return e;
  const int64_t n = (int64_t)sp.B * sp.D * 16;
  summary_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(agg_h, agg_logp, h_zero, log_decay, sp.B, pl.S,
                                                                       sp.D);
  note_launch();
  return cudaGetLastError();
}

// The checkpoint pass of the scan backward: the recurrence alone (no readout) over each whole
// sequence from h0, writing the state at the start of every 16-token chunk into ckpt [B, nck, D, 16].
template <int K>
static cudaError_t launch_ckpt(const ScanParams& sp, float* ckpt, int nck, void* status, cudaStream_t s) {
  const ScanPlan pl{true, 1, sp.L, 0};
  FastLaunch f;
  if (!fast_setup(sp, pl, status, f)) return cudaErrorInvalidValue;
  FastParams a = f.p;
  a.ckpt = ckpt;
  a.nck = nck;
  a.h_seg = nullptr;
  auto kagg = pick_kernel<K, true>(a.E, f.zoh);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(kagg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fast_smem(kMaxWarps))) !=
      cudaSuccess)
    return e;
  int ctas, warps;
  if ((e = fast_shape((const void*)kagg, a.units, f.sms, f.win, ctas, warps, a.tmem_cols)) != cudaSuccess) return e;
  kagg<<<ctas, warps * 32, fast_smem(warps), s>>>(f.tx, f.tz, f.td, f.tb, f.tc, f.to, a);
  note_launch();
  return cudaGetLastError();
}

cudaError_t run_scan_fast_ckpt(const ScanParams& sp, float* ckpt, int nck, void* status, cudaStream_t s) {
  return sp.k == 1 ? launch_ckpt<1>(sp, ckpt, nck, status, s) : launch_ckpt<2>(sp, ckpt, nck, status, s);
}

cudaError_t run_scan_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, cudaStream_t s) {
  return sp.k == 1 ? launch_fast<1>(sp, pl, seg_ws, status, s) : launch_fast<2>(sp, pl, seg_ws, status, s);
}

size_t scan_fast_summary_ws(const ScanPlan& pl, int64_t B, int D) {
  return (size_t)2 * B * pl.S * D * 16 * sizeof(float);
}

cudaError_t run_scan_summary_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, float* h_zero,
                                  float* log_decay, cudaStream_t s) {
  return sp.k == 1 ? launch_summary<1>(sp, pl, seg_ws, status, h_zero, log_decay, s)
                   : launch_summary<2>(sp, pl, seg_ws, status, h_zero, log_decay, s);
}

// ---- scratch for callers that cannot allocate device memory ----------------------------------------
// Some callers of the scan have no way to hand the library a workspace: a plugin inside a host
// framework that owns every byte of device memory and exposes no allocator to it, or a latency-
// critical loop where a cudaMalloc (which can synchronise the device) is not acceptable. For them
// swimba_scan_fwd_noalloc uses this fixed array instead of a caller workspace. It lives in the
// library's module, so every GPU that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_scan_noalloc_scratch[kScanNoAllocScratchBytes];

// Device address of the fixed scratch on the current device. In host code the array's name is only
// a host-side stand-in, so the address comes from cudaGetSymbolAddress with the device current. It
// is looked up on every call (cheap once the module is loaded), so a context that was reset and
// re-created never sees a stale address.
cudaError_t scan_noalloc_scratch(void** addr) {
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_scan_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *addr = ptr;
  return cudaSuccess;
}

}  // namespace swimba
