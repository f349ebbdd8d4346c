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
// B_mix / C_mix value a lane loads serves two channels.
// The per-expert transition rows (pre-multiplied by log2 e) live in tensor memory: each warp owns
// E*16 TMEM columns of its lane quarter and keeps expert e's 16 values of every lane at columns
// 16e..16e+15. Every lane of a warp reads the same token, so the selected expert is warp-uniform
// and one tcgen05.ld.32x32b.x16 at column 16e fetches it: a dynamically indexed, branch-free lookup
// that costs no registers and no shared-memory bandwidth.
// Per token and state:  arg = Σ_j (Δ g_j) A^{e_j};  ā = 2^arg;  h = ā h + (Δ x) B;  y += C h.
//
// A chunk of 16 tokens runs in two passes. The recurrence pass keeps only the state chain: each
// lane leaves its two partial readouts per token in shared memory. The readout pass then works on
// the whole chunk at once, with a different lane layout: lane l takes token l/2 and 16 channels,
// adds the two state halves' partials, the skip term D_skip x and the gate z σ(z) (σ via
// tanh.approx) with packed f32x2 arithmetic and 16-byte shared-memory loads, and writes 16 bf16
// outputs; one TMA store per chunk moves the [16 x 32] output tile to HBM (it clips rows past L).
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
constexpr int kCPW = 32;        // channels per warp
constexpr int kNS = 8;          // states per lane and channel
constexpr int kNP = kNS / 2;    // float2 state pairs per lane and channel
constexpr int kACols = 16;      // TMEM columns per expert (both channels of a lane)
constexpr int kMaxWarps = 8;    // warps per CTA (registers: up to 255 per thread)
constexpr int kPRow = kCPW + 4; // floats per row of the partial-readout buffer (padded)

// Byte offsets inside one ring stage of one warp.
struct Stage {
  static constexpr int X = 0;                      // bf16 [LC][32]
  static constexpr int Z = X + LC * kCPW * 2;      // bf16 [LC][32]
  static constexpr int DL = Z + LC * kCPW * 2;     // f32  [LC][32]
  static constexpr int B = DL + LC * kCPW * 4;     // f32  [LC][16]
  static constexpr int C = B + LC * 16 * 4;        // f32  [LC][16]
  static constexpr int META = C + LC * 16 * 4;     // int4 [LC] {e0, e1, g0, g1}
  static constexpr int BYTES = META + LC * 16;
  static_assert(X % 128 == 0 && Z % 128 == 0 && DL % 128 == 0 && B % 128 == 0 && C % 128 == 0 && META % 128 == 0,
                "TMA destinations must be 128-byte aligned");
  static_assert(BYTES % 128 == 0, "stage size");
};

// Per-warp readout area (after the ring): partial readouts, two output tiles (the TMA store of
// one may still be reading while the next is written), the warp's D_skip values.
struct Epi {
  static constexpr int P = 0;                              // f32 [LC][2 state halves][kPRow]
  static constexpr int O = P + LC * 2 * kPRow * 4;         // bf16 [2][LC][32]
  static constexpr int DS = O + 2 * LC * kCPW * 2;         // f32 [32]
  static constexpr int BYTES = DS + kCPW * 4;
  static_assert(O % 128 == 0 && DS % 16 == 0 && BYTES % 128 == 0, "readout area layout");
};

// TMEM columns one warp needs (16 per expert, rounded up to the 32-column allocation granule).
__host__ __device__ constexpr int tmem_cols_per_warp(int E) { return ((E * kACols + 31) / 32) * 32; }

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

// 8 bf16 (one 16-byte word) as 4 float2 pairs.
__device__ __forceinline__ void bf16x8_to_float2(const uint4 q, float2 (&f)[4]) {
  f[0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
  f[1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
  f[2] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.z));
  f[3] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.w));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float2 v) {
  const __nv_bfloat162 b = __float22bfloat162_rn(v);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// One token's scan inputs as the recurrence pass holds them (lane view: channels 2cp, 2cp+1,
// states 8gi .. 8gi+7).
struct TokIn {
  int4 m;              // {e0, e1, g0, g1}
  uint32_t ar[2][16];  // A rows of the selected experts (x log2 e), from TMEM
  float2 dl, xv;       // Δ and x of the two channels
  float2 bv[4], cv[4]; // B_mix, C_mix of the lane's 8 states
  float dx[2];         // Δ x per channel
  float2 arg[2][4];    // Σ_j (Δ g_j) A^{e_j}  [channel][state pair]
  float2 a[2][4];      // 2^arg
};

struct FastParams {
  const int32_t* idx;
  const float* gates;
  const float* A;       // [E, D, 16]
  const float* D_skip;  // [D]
  const float* h0;      // [B, D, 16] or null (start state of segment 0)
  const float* h_seg;   // [B, S, D, 16] start state of every segment (segmented main pass) or null
  float* y_pre;         // [B, L, D] or null
  float* h_final;       // [B, D, 16] or null
  float* agg_h;         // pass 1: [B, S, D, 16] end state from zero
  float* agg_logp;      // pass 1: [B, S, D, 16] log2 of the decay product
  void* status;
  int64_t L, Lseg;
  int B, D, E, k, S;
  int seg_count;        // segments this pass visits (S, or S - 1 for pass 1)
  int units;            // B * seg_count * (D / 32)
};

// AGG = true: pass 1 (segments 0 .. S-2 only; no readout, no output).
template <int K, int NPOLY, bool AGG>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
    scan_fast_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_z,
                     const __grid_constant__ CUtensorMap tm_dl, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_o,
                     const FastParams p) {
  constexpr int NS = kNS, NP = kNP, CPW = kCPW, ACOLS = kACols;
  using St = Stage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  uint8_t* ring = smem + (size_t)warp * kStages * St::BYTES;
  uint8_t* epi = smem + (size_t)nwarps * kStages * St::BYTES + (size_t)warp * Epi::BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nwarps * (kStages * St::BYTES + Epi::BYTES));
  uint64_t* full = bars + warp * kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + nwarps * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + nwarps * kStages) + 1;
  float* psm = reinterpret_cast<float*>(epi + Epi::P);
  const float* dsm = reinterpret_cast<const float*>(epi + Epi::DS);

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
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  // this warp's TMEM window: its lane quarter, tmem_cols_per_warp(E) columns
  const uint32_t tbase = *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) +
                         (uint32_t)(warp >> 2) * (uint32_t)tmem_cols_per_warp(p.E);

  const int cp = lane >> 1;   // recurrence pass: channel pair 2cp, 2cp+1 of the warp's 32
  const int gi = lane & 1;    //                  state group: states 8gi .. 8gi+7
  const int n0 = gi * NS;
  const int tl = lane >> 1;   // readout pass: token tl of the chunk,
  const int c0 = (lane & 1) * 16;  //           channels c0 .. c0+15 of the warp's 32
  const int ntiles = p.D / CPW;
  const int u_begin = (int)((int64_t)p.units * blockIdx.x / gridDim.x);
  const int u_end = (int)((int64_t)p.units * (blockIdx.x + 1) / gridDim.x);
  uint32_t phase_bits = 0;  // one parity bit per stage
  int ochunk = 0;           // output tiles written by this warp (selects the double buffer)
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

    // per-expert transition rows of this lane's 2 x 8 states, times log2(e), into TMEM
    // columns 16e + 8ch + s
    for (int e = 0; e < p.E; ++e) {
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const float4* src = reinterpret_cast<const float4*>(p.A + ((size_t)e * p.D + dA + ch) * 16 + n0);
        const float4 a0 = __ldg(src), a1 = __ldg(src + 1);
        const uint32_t r[8] = {__float_as_uint(a0.x * kLog2e), __float_as_uint(a0.y * kLog2e),
                               __float_as_uint(a0.z * kLog2e), __float_as_uint(a0.w * kLog2e),
                               __float_as_uint(a1.x * kLog2e), __float_as_uint(a1.y * kLog2e),
                               __float_as_uint(a1.z * kLog2e), __float_as_uint(a1.w * kLog2e)};
        tmem_st8(tbase + (uint32_t)(e * ACOLS + 8 * ch), r);
      }
    }
    tmem_wait_st();
    if (!AGG) reinterpret_cast<float*>(epi + Epi::DS)[lane] = p.D_skip[tile * CPW + lane];

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
      const float2* ds2 = reinterpret_cast<const float2*>(st + St::DL);
      const float4* bsm = reinterpret_cast<const float4*>(st + St::B);
      const float4* csm = reinterpret_cast<const float4*>(st + St::C);
      const int64_t t0 = t_begin + (int64_t)c * LC;
      // issue token t's loads (TMEM loads are waited for by the caller)
      auto load_tok = [&](TokIn& q, int t) {
        q.m = meta[t];
        tmem_ld16_nowait(tbase + (uint32_t)(q.m.x * ACOLS), q.ar[0]);
        if (K == 2) tmem_ld16_nowait(tbase + (uint32_t)(q.m.y * ACOLS), q.ar[1]);
        q.dl = ds2[t * (CPW / 2) + cp];
        q.xv = __bfloat1622float2(xs2[t * (CPW / 2) + cp]);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float4 bq = bsm[t * 4 + gi * 2 + i];
          q.bv[2 * i] = make_float2(bq.x, bq.y);
          q.bv[2 * i + 1] = make_float2(bq.z, bq.w);
          if (!AGG) {
            const float4 cq = csm[t * 4 + gi * 2 + i];
            q.cv[2 * i] = make_float2(cq.x, cq.y);
            q.cv[2 * i + 1] = make_float2(cq.z, cq.w);
          }
        }
      };
      // decay factors of a loaded token (independent of the state)
      auto decay = [&](TokIn& q) {
        q.dx[0] = q.dl.x * q.xv.x;
        q.dx[1] = q.dl.y * q.xv.y;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const float dlt = ch == 0 ? q.dl.x : q.dl.y;
          const float g0 = dlt * __int_as_float(q.m.z);
          const float g1 = dlt * __int_as_float(q.m.w);
#pragma unroll
          for (int s = 0; s < NP; ++s) {
            const float2 a0 = make_float2(__uint_as_float(q.ar[0][ch * NS + 2 * s]), __uint_as_float(q.ar[0][ch * NS + 2 * s + 1]));
            q.arg[ch][s] = __fmul2_rn(make_float2(g0, g0), a0);
            if (K == 2) {
              const float2 a1 = make_float2(__uint_as_float(q.ar[1][ch * NS + 2 * s]), __uint_as_float(q.ar[1][ch * NS + 2 * s + 1]));
              q.arg[ch][s] = __ffma2_rn(make_float2(g1, g1), a1, q.arg[ch][s]);
            }
            if (AGG) lsum[ch][s] = __fadd2_rn(lsum[ch][s], q.arg[ch][s]);  // Σ_t log2 ā_t
            if (s >= NP - NPOLY / 2) {
              q.a[ch][s] = exp2_poly2(q.arg[ch][s]);
            } else {
              q.a[ch][s] = make_float2(ex2_approx(q.arg[ch][s].x), ex2_approx(q.arg[ch][s].y));
            }
          }
        }
      };

      // ---- recurrence pass: the state chain only; partial readouts go to shared memory ----
      // Software-pipelined by one token: while token t updates the state, token t+1's inputs are
      // loaded (its A rows from TMEM, Δ, x, B, C from the ring) and its decay factors computed,
      // so the TMEM and shared-memory latencies and the exponentials of t+1 overlap t's FMAs.
      TokIn cur, nxt;
      load_tok(cur, 0);
      tmem_wait_ld();
      decay(cur);
      auto token = [&](int t) {
        if (t + 1 < LC) load_tok(nxt, t + 1);
        float yc[2];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const float2 dxx = make_float2(cur.dx[ch], cur.dx[ch]);
#pragma unroll
          for (int s = 0; s < NP; ++s) h[ch][s] = __ffma2_rn(cur.a[ch][s], h[ch][s], __fmul2_rn(dxx, cur.bv[s]));
          if (!AGG) {
            // two independent accumulation chains (even and odd state pairs)
            float2 ya = __fmul2_rn(cur.cv[0], h[ch][0]);
            float2 yb = __fmul2_rn(cur.cv[1], h[ch][1]);
#pragma unroll
            for (int s = 2; s < NP; s += 2) {
              ya = __ffma2_rn(cur.cv[s], h[ch][s], ya);
              yb = __ffma2_rn(cur.cv[s + 1], h[ch][s + 1], yb);
            }
            yc[ch] = (ya.x + yb.x) + (ya.y + yb.y);
          }
        }
        if (!AGG) *reinterpret_cast<float2*>(psm + (t * 2 + gi) * kPRow + 2 * cp) = make_float2(yc[0], yc[1]);
        if (t + 1 < LC) {
          tmem_wait_ld();
          decay(nxt);
          cur = nxt;
        }
      };
#pragma unroll
      for (int t = 0; t < LC; ++t) token(t);

      // ---- readout pass: lane = (token tl, channels c0..c0+15) ----
      if (!AGG) {
        __syncwarp();
        const float4* p0 = reinterpret_cast<const float4*>(psm + (tl * 2 + 0) * kPRow + c0);
        const float4* p1 = reinterpret_cast<const float4*>(psm + (tl * 2 + 1) * kPRow + c0);
        const uint4* xq = reinterpret_cast<const uint4*>(st + St::X + (tl * CPW + c0) * 2);
        const uint4* zq = reinterpret_cast<const uint4*>(st + St::Z + (tl * CPW + c0) * 2);
        const float4* dq = reinterpret_cast<const float4*>(dsm + c0);
        uint32_t packed[8];
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {  // 8 channels at a time
          float2 xf[4], zf[4];
          bf16x8_to_float2(xq[hq], xf);
          bf16x8_to_float2(zq[hq], zf);
          float2 yv[4], dk[4];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const float4 a4 = p0[2 * hq + i], b4 = p1[2 * hq + i], d4 = dq[2 * hq + i];
            yv[2 * i] = __fadd2_rn(make_float2(a4.x, a4.y), make_float2(b4.x, b4.y));
            yv[2 * i + 1] = __fadd2_rn(make_float2(a4.z, a4.w), make_float2(b4.z, b4.w));
            dk[2 * i] = make_float2(d4.x, d4.y);
            dk[2 * i + 1] = make_float2(d4.z, d4.w);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 y = __ffma2_rn(dk[i], xf[i], yv[i]);  // y + D_skip x
            yv[i] = y;
            const float2 hz = __fmul2_rn(zf[i], make_float2(0.5f, 0.5f));
            const float2 th = make_float2(tanh_approx(hz.x), tanh_approx(hz.y));
            const float2 sig = __ffma2_rn(th, make_float2(0.5f, 0.5f), make_float2(0.5f, 0.5f));
            packed[4 * hq + i] = pack_bf16x2(__fmul2_rn(__fmul2_rn(y, zf[i]), sig));
          }
          if (p.y_pre != nullptr && t0 + tl < t_end) {
            float4* yp = reinterpret_cast<float4*>(p.y_pre + ((size_t)b * p.L + t0 + tl) * p.D + tile * CPW + c0 + 8 * hq);
            yp[0] = make_float4(yv[0].x, yv[0].y, yv[1].x, yv[1].y);
            yp[1] = make_float4(yv[2].x, yv[2].y, yv[3].x, yv[3].y);
          }
        }
        // the previous TMA store from this output buffer must have finished reading it
        uint8_t* obuf = epi + Epi::O + (ochunk & 1) * (LC * CPW * 2);
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        uint4* od = reinterpret_cast<uint4*>(obuf + (tl * CPW + c0) * 2);
        od[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        od[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_o, obuf, tile * CPW, (int)t0, b);
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
    __syncwarp();
  }
  // the output stores must have read their shared-memory tiles before the CTA's memory goes away
  if (!AGG && lane == 0) bulk_wait<0>();
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

constexpr int kNPoly = 0;  // states per lane and channel whose exp2 runs on the FMA pipe (even, <= 8)

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
  const int64_t base_units = B * (D / kCPW);
  const int64_t target = (int64_t)device_sms() * 6;  // at least 6 warps (192 channels) per SM
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

template <int K>
static cudaError_t launch_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, cudaStream_t s) {
  constexpr int CPW = kCPW;
  CUtensorMap tx, tz, td, tb, tc, to;
  if (!map3(&tx, sp.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, CPW) ||
      !map3(&tz, sp.z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, CPW) ||
      !map3(&td, sp.delta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, sp.D, sp.L, sp.B, CPW) ||
      !map3(&tb, sp.B_mix, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 16, sp.L, sp.B, 16) ||
      !map3(&tc, sp.C_mix, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 16, sp.L, sp.B, 16) ||
      !map3(&to, sp.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sp.D, sp.L, sp.B, CPW))
    return cudaErrorInvalidValue;
  FastParams p{};
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
    const int per_quarter = 512 / tmem_cols_per_warp(sp.E);  // warps that fit one lane quarter's TMEM
    const int wmax = std::max(1, std::min({kMaxWarps, fa.maxThreadsPerBlock / 32, 4 * per_quarter}));
    ctas = std::max(1, std::min(sms, units));
    warps = std::min(wmax, (units + ctas - 1) / ctas);
    if ((int64_t)ctas * warps < units) ctas = std::min<int64_t>((units + warps - 1) / warps, 65535);
    return cudaSuccess;
  };
  int ctas, warps;
  const size_t smem_per_warp = (size_t)kStages * Stage::BYTES + Epi::BYTES + (size_t)kStages * 8;
  const size_t smem = 128 + (size_t)kMaxWarps * smem_per_warp + 32;
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
    auto kagg = scan_fast_kernel<K, kNPoly, true>;
    if ((e = cudaFuncSetAttribute(kagg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    if ((e = shape((const void*)kagg, a.units, ctas, warps)) != cudaSuccess) return e;
    kagg<<<ctas, warps * 32, 128 + warps * smem_per_warp + 32, s>>>(tx, tz, td, tb, tc, to, a);
    const int64_t n = (int64_t)sp.B * sp.D * 16;
    scan_carry_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(sp.h0, agg_h, agg_logp, h_seg, sp.B, pl.S, sp.D);
    note_launch(2);
    p.h_seg = h_seg;
  }
  auto kmain = scan_fast_kernel<K, kNPoly, false>;
  if ((e = cudaFuncSetAttribute(kmain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
    return e;
  if ((e = shape((const void*)kmain, p.units, ctas, warps)) != cudaSuccess) return e;
  kmain<<<ctas, warps * 32, 128 + warps * smem_per_warp + 32, s>>>(tx, tz, td, tb, tc, to, p);
  note_launch();
  return cudaGetLastError();
}

cudaError_t run_scan_fast(const ScanParams& sp, const ScanPlan& pl, void* seg_ws, void* status, cudaStream_t s) {
  return sp.k == 1 ? launch_fast<1>(sp, pl, seg_ws, status, s) : launch_fast<2>(sp, pl, seg_ws, status, s);
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
