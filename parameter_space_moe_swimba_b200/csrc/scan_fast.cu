// Selective scan over the mixed parameters, B200 fast path (bf16 x/z/out, N = 16, k <= 2, E <= 16).
//
// Sources: "Swimba: Switch Mamba Model Scales State Space Models" -- one state trajectory and ONE
// recurrence whatever the number of experts (§2 "Resultado"; Teorema 2: the recurrence cost does
// not grow with E); "Mamba y las SSMs: el retorno del estado persistente", "Mamba" (Ā = exp(Δ_t A);
// Figura 2: the state stays on chip, inputs stream from HBM) and "Estado interno puramente lineal"
// (the linear state admits a scan, used here to split long sequences into segments).
//
// Work unit = one warp = 32 channels of one sequence segment. Lane l holds the channel pair
// (2*(l>>1), 2*(l>>1)+1) of the warp and the 8 states (l&1)*8 .. +7 of both channels, 16 fp32 states
// in registers; the two lanes of a pair together hold all 16 states of the two channels. So every
// B_mix / C_mix value a lane loads serves two channels, and one shuffle finishes the readout.
// The per-expert transition rows (pre-multiplied by log2 e) live in tensor memory: each warp owns
// E*16 TMEM columns of its lane quarter and keeps expert e's 16 values of every lane at columns
// 16e..16e+15. Every lane of a warp reads the same token, so the selected expert is warp-uniform
// and one tcgen05.ld.32x32b.x16 at column 16e fetches it: a dynamically indexed, branch-free lookup
// that costs no registers and no shared-memory bandwidth.
// Per token and state:  arg = Σ_j (Δ g_j) A^{e_j};  ā = 2^arg;  h = ā h + (Δ x) B;  y += C h.
// The two lanes of a pair swap one partial readout so that each finishes one channel's token:
// y += D_skip x, out = y z σ(z) (σ via tanh.approx for bf16 outputs).
//
// Each warp streams its inputs through its own 3-stage shared-memory ring filled by TMA (x, z, Δ
// tiles of [16 tokens x 32 channels] and B_mix, C_mix rows of 16 tokens) plus the tokens' expert
// indices and gates written by the warp's lanes one chunk ahead. Units are spread evenly over one
// persistent CTA per SM, so no SM gets a whole extra sequence.
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

namespace swimba {

using namespace sm100;

namespace {

constexpr int LC = 16;          // tokens per chunk
constexpr int kStages = 3;      // ring depth per warp

// Lane geometry, by G = lanes per channel pair (2 or 4): each lane holds NS = 16 / G states of two
// channels; a warp covers CPW = 64 / G channels; a CTA holds up to 8 (G = 2, up to 255 registers a
// thread) or 16 (G = 4, up to 128) warps.
template <int G>
struct Geo {
  static_assert(G == 2 || G == 4, "2 or 4 lanes per channel pair");
  static constexpr int NS = 16 / G;        // states per lane and channel
  static constexpr int NP = NS / 2;        // float2 pairs per lane and channel
  static constexpr int CPW = 64 / G;       // channels per warp
  static constexpr int ACOLS = 2 * NS;     // TMEM columns per expert (both channels of a lane)
  static constexpr int MAXW = 4 * G;       // warps per CTA
};

// Byte offsets inside one ring stage of one warp.
template <int CPW>
struct Stage {
  static constexpr int X = 0;                      // bf16 [LC][CPW]
  static constexpr int Z = X + LC * CPW * 2;       // bf16 [LC][CPW]
  static constexpr int DL = Z + LC * CPW * 2;      // f32  [LC][CPW]
  static constexpr int B = DL + LC * CPW * 4;      // f32  [LC][16]
  static constexpr int C = B + LC * 16 * 4;        // f32  [LC][16]
  static constexpr int META = C + LC * 16 * 4;     // int4 [LC] {e0, e1, g0, g1}
  static constexpr int BYTES = META + LC * 16;
  static_assert(X % 128 == 0 && Z % 128 == 0 && DL % 128 == 0 && B % 128 == 0 && C % 128 == 0 && META % 128 == 0,
                "TMA destinations must be 128-byte aligned");
  static_assert(BYTES % 128 == 0, "stage size");
};

// TMEM columns one warp needs (ACOLS per expert, rounded up to the 32-column allocation granule).
__host__ __device__ constexpr int tmem_cols_per_warp(int E, int acols) { return ((E * acols + 31) / 32) * 32; }

// n consecutive TMEM columns of this thread's lane, without waiting (n = 8 or 16).
template <int NCOL>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NCOL]) {
  if constexpr (NCOL == 16) tmem_ld16_nowait(taddr, r);
  else tmem_ld8_nowait(taddr, r);
}

// 2^x on the FMA pipe for x <= 0: x = j + f with j = round(x) (the 1.5*2^23 shifter), f in
// [-1/2, 1/2]; 2^f by a degree-5 polynomial fitted for minimax relative error on that interval
// (fit_exp2_poly.py beside this file: float32 Horner error 2.4e-7, the size of ex2.approx's);
// the exponent j is added to the result's exponent field. Inputs below -125 are clamped (result
// 2^-125 instead of a flushed 0, which no decay product here can tell apart).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 lo = make_float2(-125.f, -125.f);
  x = make_float2(fmaxf(x.x, lo.x), fmaxf(x.y, lo.y));
  const float2 shifter = make_float2(12582912.f, 12582912.f);
  const float2 t = __fadd2_rn(x, shifter);
  const float2 j = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __fadd2_rn(x, make_float2(-j.x, -j.y));
  float2 p = make_float2(0x1.5c08e6p-10f, 0x1.5c08e6p-10f);
  p = __ffma2_rn(p, f, make_float2(0x1.3d0c52p-7f, 0x1.3d0c52p-7f));
  p = __ffma2_rn(p, f, make_float2(0x1.c6b6e4p-5f, 0x1.c6b6e4p-5f));
  p = __ffma2_rn(p, f, make_float2(0x1.ebf918p-3f, 0x1.ebf918p-3f));
  p = __ffma2_rn(p, f, make_float2(0x1.62e428p-1f, 0x1.62e428p-1f));
  p = __ffma2_rn(p, f, make_float2(0x1.000002p+0f, 0x1.000002p+0f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct FastParams {
  const int32_t* idx;
  const float* gates;
  const float* A;       // [E, D, 16]
  const float* D_skip;  // [D]
  const float* h0;      // [B, D, 16] or null (start state of segment 0)
  const float* h_seg;   // [B, S, D, 16] start state of every segment (segmented main pass) or null
  __nv_bfloat16* out;   // [B, L, D]
  float* y_pre;         // [B, L, D] or null
  float* h_final;       // [B, D, 16] or null
  float* agg_h;         // pass 1: [B, S, D, 16] end state from zero
  float* agg_logp;      // pass 1: [B, S, D, 16] log2 of the decay product
  void* status;
  int64_t L, Lseg;
  int B, D, E, k, S;
  int seg_count;        // segments this pass visits (S, or S - 1 for pass 1)
  int units;            // B * seg_count * (D / CPW)
};

// AGG = true: pass 1 (segments 0 .. S-2 only; no readout, no output).
template <int K, int NPOLY, bool AGG, int G>
__global__ void __launch_bounds__(Geo<G>::MAXW * 32, 1)
    scan_fast_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                     const __grid_constant__ CUtensorMap tm_dl, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c, const FastParams p) {
  constexpr int NS = Geo<G>::NS, NP = Geo<G>::NP, CPW = Geo<G>::CPW, ACOLS = Geo<G>::ACOLS;
  using St = Stage<CPW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  uint8_t* ring = smem + (size_t)warp * kStages * St::BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nwarps * kStages * St::BYTES);
  uint64_t* full = bars + warp * kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + nwarps * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + nwarps * kStages) + 1;

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
      }
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  // this warp's TMEM window: its lane quarter, tmem_cols_per_warp(E, ACOLS) columns
  const uint32_t tbase = *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) +
                         (uint32_t)(warp >> 2) * (uint32_t)tmem_cols_per_warp(p.E, ACOLS);

  const int cp = lane / G;    // channel pair: channels 2cp, 2cp+1 of the warp's CPW
  const int gi = lane % G;    // state group: states NS*gi .. NS*gi+NS-1
  const int n0 = gi * NS;
  // the output this lane finishes: G = 2, channel gi of both tokens of a pair; G = 4, channel
  // gi & 1 of token gi >> 1 of the pair
  const int och = G == 2 ? gi : (gi & 1);
  const int ou = G == 2 ? 0 : (gi >> 1);
  const int ntiles = p.D / CPW;
  const int u_begin = (int)((int64_t)p.units * blockIdx.x / gridDim.x);
  const int u_end = (int)((int64_t)p.units * (blockIdx.x + 1) / gridDim.x);
  uint32_t phase_bits = 0;  // one parity bit per stage
  constexpr uint32_t tx_bytes = AGG ? (LC * CPW * 2 + LC * CPW * 4 + LC * 16 * 4)
                                    : (2 * LC * CPW * 2 + LC * CPW * 4 + 2 * LC * 16 * 4);

  for (int u = u_begin + warp; u < u_end; u += nwarps) {
    const int tile = u % ntiles;
    const int bs = u / ntiles;  // b * seg_count + seg
    const int seg = bs % p.seg_count;
    const int b = bs / p.seg_count;
    const int dA = tile * CPW + 2 * cp;  // this lane's channels dA, dA + 1
    const int64_t t_begin = (int64_t)seg * p.Lseg;
    const int64_t t_end = std::min<int64_t>(p.L, t_begin + p.Lseg);
    const int nchunks = (int)((t_end - t_begin + LC - 1) / LC);

    // per-expert transition rows of this lane's 2 x NS states, times log2(e), into TMEM
    // columns ACOLS*e + NS*ch + s
    for (int e = 0; e < p.E; ++e) {
      uint32_t r[ACOLS];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const float4* src = reinterpret_cast<const float4*>(p.A + ((size_t)e * p.D + dA + ch) * 16 + n0);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
          const float4 a4 = __ldg(src + q);
          r[ch * NS + 4 * q + 0] = __float_as_uint(a4.x * kLog2e);
          r[ch * NS + 4 * q + 1] = __float_as_uint(a4.y * kLog2e);
          r[ch * NS + 4 * q + 2] = __float_as_uint(a4.z * kLog2e);
          r[ch * NS + 4 * q + 3] = __float_as_uint(a4.w * kLog2e);
        }
      }
#pragma unroll
      for (int q = 0; q < ACOLS / 8; ++q) {
        const uint32_t (&r8)[8] = *reinterpret_cast<const uint32_t(*)[8]>(r + 8 * q);
        tmem_st8(tbase + (uint32_t)(e * ACOLS + 8 * q), r8);
      }
    }
    tmem_wait_st();

    float2 h[2][NP];  // [channel][state pair]
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      const float* hs = AGG ? nullptr
                            : (p.h_seg != nullptr ? p.h_seg + (((size_t)b * p.S + seg) * p.D + dA + ch) * 16
                                                  : (p.h0 != nullptr && seg == 0 ? p.h0 + ((size_t)b * p.D + dA + ch) * 16
                                                                                 : nullptr));
#pragma unroll
      for (int s = 0; s < NP; ++s)
        h[ch][s] = hs ? *reinterpret_cast<const float2*>(hs + n0 + 2 * s) : make_float2(0.f, 0.f);
    }
    float2 lsum[2][NP];
#pragma unroll
    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
      for (int s = 0; s < NP; ++s) lsum[ch][s] = make_float2(0.f, 0.f);
    const int dmine = dA + och;  // the channel whose outputs this lane writes
    const float dsk = AGG ? 0.f : p.D_skip[dmine];

    // meta of one chunk: lane t (< LC) holds token t's {e0, e1, g0, g1}
    auto load_meta = [&](int c) -> int4 {
      int4 m = make_int4(0, 0, 0, 0);
      const int64_t t = t_begin + (int64_t)c * LC + lane;
      if (lane < LC && c < nchunks && t < t_end) {
        const size_t tok = (size_t)b * p.L + t;
        m.x = min(max(p.idx[tok * K], 0), p.E - 1);
        m.z = __float_as_int(p.gates[tok * K]);
        if (K == 2) {
          m.y = min(max(p.idx[tok * K + 1], 0), p.E - 1);
          m.w = __float_as_int(p.gates[tok * K + 1]);
        }
      }
      return m;
    };
    // fill stage (c % kStages) with chunk c: meta from registers, the rest by TMA
    auto issue = [&](int c, int4 meta) {
      uint8_t* st = ring + (c % kStages) * St::BYTES;
      if (lane < LC) reinterpret_cast<int4*>(st + St::META)[lane] = meta;
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_smem();
        uint64_t* bar = &full[c % kStages];
        mbar_arrive_expect_tx(bar, tx_bytes);
        const int t0 = (int)(t_begin + (int64_t)c * LC);
        tma_load_3d(st + St::X, &tm_x, bar, tile * CPW, t0, b);
        tma_load_3d(st + St::DL, &tm_dl, bar, tile * CPW, t0, b);
        tma_load_3d(st + St::B, &tm_b, bar, 0, t0, b);
        if (!AGG) {
          tma_load_3d(st + St::Z, &tm_z, bar, tile * CPW, t0, b);
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
    for (int c = 0; c < nchunks; ++c) {
      const int sidx = c % kStages;
      if (!mbar_wait(&full[sidx], (phase_bits >> sidx) & 1u, abort_flag)) {
        ok = false;
        break;
      }
      phase_bits ^= 1u << sidx;
      const uint8_t* st = ring + sidx * St::BYTES;
      const int4* meta = reinterpret_cast<const int4*>(st + St::META);
      const __nv_bfloat162* xs2 = reinterpret_cast<const __nv_bfloat162*>(st + St::X);
      const __nv_bfloat16* zs = reinterpret_cast<const __nv_bfloat16*>(st + St::Z);
      const float2* ds2 = reinterpret_cast<const float2*>(st + St::DL);
      const float4* bsm = reinterpret_cast<const float4*>(st + St::B);
      const float4* csm = reinterpret_cast<const float4*>(st + St::C);
      const int64_t t0 = t_begin + (int64_t)c * LC;
      const bool full_chunk = t0 + LC <= t_end;
      __nv_bfloat16* outp = AGG ? nullptr : p.out + ((size_t)b * p.L + t0) * p.D + dmine;
      float* ypp = (AGG || p.y_pre == nullptr) ? nullptr : p.y_pre + ((size_t)b * p.L + t0) * p.D + dmine;
      // pass over the chunk's tokens: the recurrence only; readout partials are kept in registers
      // and the reduction, skip term, gate and stores follow for the whole chunk, off the
      // recurrence's dependency chain
      float ypart[LC][2];  // [token][channel]
#pragma unroll
      for (int t = 0; t < LC; t += 2) {
        // loads of both tokens first: the selected experts' A rows (TMEM), Δ, x, B, C (smem)
        int4 m[2];
        uint32_t ar[2][2][ACOLS];  // [token][expert slot][columns]
        float2 dl[2], xv[2];
        float2 bv[2][NP], cv[2][NP];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          m[u] = meta[t + u];
          tmem_ld_cols<ACOLS>(tbase + (uint32_t)(m[u].x * ACOLS), ar[u][0]);
          if (K == 2) tmem_ld_cols<ACOLS>(tbase + (uint32_t)(m[u].y * ACOLS), ar[u][1]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          dl[u] = ds2[(t + u) * (CPW / 2) + cp];
          xv[u] = __bfloat1622float2(xs2[(t + u) * (CPW / 2) + cp]);
#pragma unroll
          for (int q = 0; q < NS / 4; ++q) {
            const float4 bq = bsm[(t + u) * 4 + gi * (NS / 4) + q];
            bv[u][2 * q] = make_float2(bq.x, bq.y);
            bv[u][2 * q + 1] = make_float2(bq.z, bq.w);
            if (!AGG) {
              const float4 cq = csm[(t + u) * 4 + gi * (NS / 4) + q];
              cv[u][2 * q] = make_float2(cq.x, cq.y);
              cv[u][2 * q + 1] = make_float2(cq.z, cq.w);
            }
          }
        }
        tmem_wait_ld();
        // decay factors of both tokens (independent of the state)
        float2 a[2][2][NP];  // [token][channel][state pair]
        float2 arg[2][2][NP];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const float dlt = ch == 0 ? dl[u].x : dl[u].y;
            const float c0 = dlt * __int_as_float(m[u].z);
            const float c1 = dlt * __int_as_float(m[u].w);
#pragma unroll
            for (int s = 0; s < NP; ++s) {
              const float2 a0 = make_float2(__uint_as_float(ar[u][0][ch * NS + 2 * s]), __uint_as_float(ar[u][0][ch * NS + 2 * s + 1]));
              arg[u][ch][s] = __fmul2_rn(make_float2(c0, c0), a0);
              if (K == 2) {
                const float2 a1 =
                    make_float2(__uint_as_float(ar[u][1][ch * NS + 2 * s]), __uint_as_float(ar[u][1][ch * NS + 2 * s + 1]));
                arg[u][ch][s] = __ffma2_rn(make_float2(c1, c1), a1, arg[u][ch][s]);
              }
              if (s >= NP - NPOLY / 2) {
                a[u][ch][s] = exp2_poly2(arg[u][ch][s]);
              } else {
                a[u][ch][s] = make_float2(ex2_approx(arg[u][ch][s].x), ex2_approx(arg[u][ch][s].y));
              }
            }
          }
        // the recurrence, token t then t+1; this lane's partial readouts go to ypart
#pragma unroll
        for (int u = 0; u < 2; ++u) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const float dx = (ch == 0 ? dl[u].x : dl[u].y) * (ch == 0 ? xv[u].x : xv[u].y);
            const float2 dxx = make_float2(dx, dx);
#pragma unroll
            for (int s = 0; s < NP; ++s) h[ch][s] = __ffma2_rn(a[u][ch][s], h[ch][s], __fmul2_rn(dxx, bv[u][s]));
            if (AGG) {
#pragma unroll
              for (int s = 0; s < NP; ++s) lsum[ch][s] = __fadd2_rn(lsum[ch][s], arg[u][ch][s]);
            } else {
              // two independent accumulation chains (even and odd state pairs)
              float2 ya = __fmul2_rn(cv[u][0], h[ch][0]);
              float2 yb = __fmul2_rn(cv[u][1], h[ch][1]);
#pragma unroll
              for (int s = 2; s < NP; s += 2) {
                ya = __ffma2_rn(cv[u][s], h[ch][s], ya);
                yb = __ffma2_rn(cv[u][s + 1], h[ch][s + 1], yb);
              }
              ypart[t + u][ch] = (ya.x + yb.x) + (ya.y + yb.y);
            }
          }
        }
      }
      if (!AGG) {
        const __nv_bfloat16* xs = reinterpret_cast<const __nv_bfloat16*>(st + St::X);
#pragma unroll
        for (int t = 0; t < LC; t += 2) {
          // reduce the partial readouts over the G lanes of the channel pair, scattering them so
          // that each lane finishes its own (token, channel) outputs
          float ysum[2];
          if (G == 2) {
            // lanes 2cp (states 0-7) and 2cp+1 (states 8-15) swap one partial per token
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float send = gi == 0 ? ypart[t + u][1] : ypart[t + u][0];
              const float keep = gi == 0 ? ypart[t + u][0] : ypart[t + u][1];
              ysum[u] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
            }
          } else {
            // step 1 (lanes gi, gi ^ 2): keep token ou, send the other token's two channels
            float r2[2];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              const float send = ou == 0 ? ypart[t + 1][ch] : ypart[t][ch];
              const float keep = ou == 0 ? ypart[t][ch] : ypart[t + 1][ch];
              r2[ch] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            }
            // step 2 (lanes gi, gi ^ 1): keep channel och, send the other
            const float send = och == 0 ? r2[1] : r2[0];
            const float keep = och == 0 ? r2[0] : r2[1];
            ysum[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
            ysum[1] = 0.f;
          }
#pragma unroll
          for (int o = 0; o < (G == 2 ? 2 : 1); ++o) {
            const int uu = G == 2 ? o : ou;
            if (full_chunk || t0 + t + uu < t_end) {
              const float xm = __bfloat162float(xs[(t + uu) * CPW + 2 * cp + och]);
              const float zv = __bfloat162float(zs[(t + uu) * CPW + 2 * cp + och]);
              const float y = fmaf(dsk, xm, ysum[o]);
              if (ypp != nullptr) ypp[(size_t)(t + uu) * p.D] = y;
              const float sig = fmaf(0.5f, tanh_approx(0.5f * zv), 0.5f);
              outp[(size_t)(t + uu) * p.D] = __float2bfloat16_rn(y * zv * sig);
            }
          }
        }
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
      // let this warp's copies in flight land before the CTA exits (bounded, ignores the flag)
      for (int c = issued - kStages; c < issued; ++c) {
        if (c < 0) continue;
        const int sidx = c % kStages;
        const uint64_t w0 = globaltimer_ns();
        while (!mbar_try_wait(&full[sidx], (phase_bits >> sidx) & 1u) && globaltimer_ns() - w0 < kWaitLimitNs) {
        }
        phase_bits ^= 1u << sidx;
      }
      break;
    }
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      if (AGG) {
        const size_t o = (((size_t)b * p.S + seg) * p.D + dA + ch) * 16 + n0;
#pragma unroll
        for (int s = 0; s < NP; ++s) {
          *reinterpret_cast<float2*>(p.agg_h + o + 2 * s) = h[ch][s];
          *reinterpret_cast<float2*>(p.agg_logp + o + 2 * s) = lsum[ch][s];
        }
      } else if (p.h_final != nullptr && seg == p.S - 1) {
        const size_t o = ((size_t)b * p.D + dA + ch) * 16 + n0;
#pragma unroll
        for (int s = 0; s < NP; ++s) *reinterpret_cast<float2*>(p.h_final + o + 2 * s) = h[ch][s];
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, 512);
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

constexpr int kNPoly = 0;  // states per lane and channel whose exp2 runs on the FMA pipe (even, <= NS)
#ifndef SWIMBA_SCAN_G
#define SWIMBA_SCAN_G 2
#endif
constexpr int kLanesPerPair = SWIMBA_SCAN_G;  // lanes per channel pair of the launched kernels

}  // namespace

// ---- segment plan and workspace ---------------------------------------------------------------------
ScanPlan scan_fast_plan(int64_t B, int64_t L, int D, int N, int E, int k, bool io_bf16) {
  ScanPlan pl{};
  pl.fast = io_bf16 && N == 16 && (k == 1 || k == 2) && E >= 1 && E <= 16;
  if (!pl.fast) return pl;
  pl.g = kLanesPerPair;
  const int CPW = 64 / pl.g;
  if (D % CPW != 0 || B * L > (int64_t(1) << 31)) {
    pl.fast = false;
    return pl;
  }
  const int64_t base_units = B * (D / CPW);
  const int64_t target = (int64_t)device_sms() * 3 * pl.g;  // warps per SM: 6 (G = 2) or 12 (G = 4)
  int64_t S = 1;
  if (base_units < target) S = std::min<int64_t>((target + base_units - 1) / base_units, (L + LC - 1) / LC);
  int64_t Lseg = (L + S - 1) / S;
  Lseg = (Lseg + LC - 1) / LC * LC;
  S = (L + Lseg - 1) / Lseg;
  pl.S = (int)S;
  pl.Lseg = Lseg;
  pl.ws_bytes = S > 1 ? (size_t)3 * B * S * D * 16 * sizeof(float) : 0;
  return pl;
}

template <int K, int G>
static cudaError_t launch_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, cudaStream_t s) {
  constexpr int CPW = Geo<G>::CPW, MAXW = Geo<G>::MAXW;
  using St = Stage<CPW>;
  CUtensorMap tx, tz, td, tb, tc;
  if (!map3(&tx, sp.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, CPW) ||
      !map3(&tz, sp.z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, CPW) ||
      !map3(&td, sp.delta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, sp.D, sp.L, sp.B, CPW) ||
      !map3(&tb, sp.B_mix, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 16, sp.L, sp.B, 16) ||
      !map3(&tc, sp.C_mix, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 16, sp.L, sp.B, 16))
    return cudaErrorInvalidValue;
  FastParams p{};
  p.idx = sp.idx;
  p.gates = sp.gates;
  p.A = sp.A;
  p.D_skip = sp.D_skip;
  p.h0 = sp.h0;
  p.out = reinterpret_cast<__nv_bfloat16*>(sp.out);
  p.y_pre = sp.y_pre;
  p.h_final = sp.h_final;
  p.status = status;
  p.L = sp.L;
  p.Lseg = pl.Lseg;
  p.B = sp.B;
  p.D = sp.D;
  p.E = sp.E;
  p.k = sp.k;
  p.S = pl.S;
  p.seg_count = pl.S;
  p.units = sp.B * pl.S * (sp.D / CPW);
  const int sms = device_sms();
  // block size: the kernel's register use decides how many warps a CTA may hold
  auto shape = [&](const void* fn, int units, int& ctas, int& warps) -> cudaError_t {
    cudaFuncAttributes fa;
    cudaError_t err = cudaFuncGetAttributes(&fa, fn);
    if (err != cudaSuccess) return err;
    // warps that fit one lane quarter's 512 TMEM columns
    const int per_quarter = 512 / tmem_cols_per_warp(sp.E, Geo<G>::ACOLS);
    const int wmax = std::max(1, std::min({MAXW, fa.maxThreadsPerBlock / 32, 4 * per_quarter}));
    ctas = std::max(1, std::min(sms, units));
    warps = std::min(wmax, (units + ctas - 1) / ctas);
    if ((int64_t)ctas * warps < units) ctas = std::min<int64_t>((units + warps - 1) / warps, 65535);
    return cudaSuccess;
  };
  int ctas, warps;
  const size_t smem_per_warp = (size_t)kStages * St::BYTES + (size_t)kStages * 8;
  const size_t smem = 128 + (size_t)MAXW * smem_per_warp + 32;
  cudaError_t e;
  if (pl.S > 1) {
    float* agg_h = reinterpret_cast<float*>(seg_ws);
    float* agg_logp = agg_h + (size_t)sp.B * pl.S * sp.D * 16;
    float* h_seg = agg_logp + (size_t)sp.B * pl.S * sp.D * 16;
    FastParams a = p;
    a.agg_h = agg_h;
    a.agg_logp = agg_logp;
    a.h0 = nullptr;
    a.seg_count = pl.S - 1;  // the last segment needs no aggregate
    a.units = sp.B * (pl.S - 1) * (sp.D / CPW);
    auto kagg = scan_fast_kernel<K, kNPoly, true, G>;
    if ((e = cudaFuncSetAttribute(kagg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    if ((e = shape((const void*)kagg, a.units, ctas, warps)) != cudaSuccess) return e;
    kagg<<<ctas, warps * 32, 128 + warps * smem_per_warp + 32, s>>>(tx, tz, td, tb, tc, a);
    const int64_t n = (int64_t)sp.B * sp.D * 16;
    scan_carry_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(sp.h0, agg_h, agg_logp, h_seg, sp.B, pl.S, sp.D);
    note_launch(2);
    p.h_seg = h_seg;
  }
  auto kmain = scan_fast_kernel<K, kNPoly, false, G>;
  if ((e = cudaFuncSetAttribute(kmain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
    return e;
  if ((e = shape((const void*)kmain, p.units, ctas, warps)) != cudaSuccess) return e;
  kmain<<<ctas, warps * 32, 128 + warps * smem_per_warp + 32, s>>>(tx, tz, td, tb, tc, p);
  note_launch();
  return cudaGetLastError();
}

cudaError_t run_scan_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, cudaStream_t s) {
  if (pl.g == 2) return sp.k == 1 ? launch_fast<1, 2>(sp, pl, seg_ws, status, s) : launch_fast<2, 2>(sp, pl, seg_ws, status, s);
  return sp.k == 1 ? launch_fast<1, 4>(sp, pl, seg_ws, status, s) : launch_fast<2, 4>(sp, pl, seg_ws, status, s);
}

// ---- scratch for callers that cannot allocate device memory ----------------------------------------
// Some callers of the scan have no way to hand the library a workspace: a plugin inside a host
// framework that owns every byte of device memory and exposes no allocator to it, or a latency-
// critical loop where a cudaMalloc (which can synchronise the device) is not acceptable. For them
// swimba_scan_fwd_noalloc uses this fixed array instead of a caller workspace. It lives in the
// library's module, so every GPU that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_scan_noalloc_scratch[kScanNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_addr[256] = {};
}  // namespace

// Device address of the fixed scratch on the current device. In host code the array's name is only
// a host-side stand-in, so the address comes from cudaGetSymbolAddress, once per device, with that
// device current, and is cached.
cudaError_t scan_noalloc_scratch(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_scan_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = ptr;
  }
  *addr = g_noalloc_addr[dev];
  return cudaSuccess;
}

}  // namespace swimba
