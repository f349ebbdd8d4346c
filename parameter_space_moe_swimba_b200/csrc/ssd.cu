// Swimba on the Mamba-2 state-space-dual (SSD) form, chunked, on the tcgen05 tensor cores.
//
// Sources: "Swimba: Switch Mamba Model Scales State Space Models", Spanish summary §2 "Arquitectura
// de Swimba" (Swimba is built on Mamba-2 and its state space duality; every expert makes its own
// token-dependent streams B^(e), C^(e), X^(e); the transition A is shared by the experts and over
// time; the state input mixes Σ_e π_e B^(e) X^(e), the readout uses (Σ_e π_e C^(e))ᵀ h; one state
// update per token) and the Dutch summary §2 "Architectuur Implementatie" (the SSD computation
// and the chunked processing of Mamba-2 carry over); "Mamba y las SSMs", "Mamba" (Ā = exp(Δ A)).
//
// Per head h of P channels (scalar transition A_h < 0, one step Δ_t[h] per token), with the
// active expert's streams X_t [H, P] and B_t [N], gate g_t and the mixed readout C_mix,t [N]:
//   S_t[h] = exp(Δ_t A_h) S_{t-1}[h] + Δ_t g_t X_t[h] ⊗ B_t;   y_t[h] = S_t[h] C_mix,t + D_h g_t X_t[h].
// Chunked over Q = 128 tokens with cum[i] = Σ_{r<=i} Δ_r A_h (from the chunk start):
//   G[i, s]  = C_mix,i · B_s                                    (tensor cores, [Q x Q], K = N)
//   W[i, s]  = exp(cum[i] - cum[s]) Δ_s g_s G[i, s] for s <= i, else 0
//   y        = W X + exp(cum) ⊙ (C_mix S_inᵀ) + D g X           (tensor cores, K = Q and K = N)
//   S_outᵀ   = exp(cum[Q-1]) S_inᵀ + Bᵀ X_w,  X_w[s] = exp(cum[Q-1] - cum[s]) Δ_s g_s X[s]
//                                                               (tensor cores, K = Q)
//
// One CTA of 8 warps per (sequence, head) walks the chunks in order, so the carried state never
// leaves the SM: Sᵀ [N x P] is an fp32 accumulator in tensor memory, scaled by the chunk's decay
// and accumulated by the state MMA. The three operands the kernel makes itself -- the state's copy
// for the readout, W and X_w -- enter the MMAs as two bf16 parts, hi = bf16(v) and
// lo = bf16(v - hi) (about 16 significant bits, one more MMA each), so the state read out stays
// fp32-accurate; a single bf16 copy of each moved y by up to 2e-2 (1 + |y|) on the test shapes.
// W goes to tensor memory (tcgen05.st), where the Y1 product reads it as its A operand, which
// leaves shared memory for two sets of the chunk tiles: the copies for chunk c + 1 are issued when
// chunk c starts.
// Two threads own row i of every [Q x *] accumulator (TMEM lane i; warps w and w + 4 share lane
// quarter w), each half of the row's columns: they build row i of W, scale row i of X, write row i
// of y and row i of Sᵀ; two warps per scheduler hide the exponentials' and the TMEM loads' latency.
// The next chunk's Δ and gates are loaded while the current chunk's outputs are written. One
// thread issues the TMA loads (C_mix, B, X tiles, 128-byte swizzled) and the MMAs. Shapes: P = 64,
// N = 128, one active expert per token (the pages' Swimba-14B routes every token to one of 4
// experts).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace swimba {

using namespace sm100;

namespace {

constexpr int SQ = 128;  // tokens per chunk
constexpr int SP = 64;   // channels per head
constexpr int SN = 128;  // state size
constexpr int kBox = SQ * 128;  // one 128-row x 128-byte swizzled box: 16 KB

// Shared memory (1024-byte aligned boxes for the 128-byte swizzle). A chunk's tiles (C_mix, B, X)
// are double-buffered: the copies for chunk c + 1 are issued when chunk c starts.
struct SsdSmem {
  static constexpr int TILE = 5 * kBox;       // one chunk: C_mix [128 tok][128 n] (2 boxes, K-major A),
                                              // B [128 tok][128 n] (2 boxes, K-major B / MN-major A),
                                              // X [128 tok][64 p] (1 box, MN-major B)
  static constexpr int TC = 0, TB = 2 * kBox, TX = 4 * kBox;  // offsets inside a tile buffer
  static constexpr int XW = 2 * TILE;         // X_w    [128 tok][64 p]:  hi, lo: 1 box each (MN-major B)
  static constexpr int S = XW + 2 * kBox;     // S_inᵀ  [128 n][64 p]:    hi, lo: 1 box each (MN-major B)
  static constexpr int CUM = S + 2 * kBox;    // f32 [128] cum
  static constexpr int DG = CUM + SQ * 4;     // f32 [128] Δ g
  static constexpr int WSUM = DG + SQ * 4;    // f32 [4] warp totals of the scan
  static constexpr int BAR = WSUM + 64;       // 3 mbarriers: copies into buffer 0, 1; MMAs
  static constexpr int MISC = BAR + 32;       // abort flag, TMEM base
  static constexpr int BYTES = MISC + 16;
};

// TMEM columns: fp32 accumulators G, Y1, Y2, Sᵀ; then W (the Y1 product's A operand, bf16 pairs):
// hi in [kColW, kColW + 64), lo in [kColW + 64, kColW + 128).
constexpr uint32_t kColG = 0, kColY1 = 128, kColY2 = 192, kColS = 256, kColW = 320;

struct SsdParams {
  const float* gates;  // [B, L, 1]
  const float* delta;  // [B, L, H]
  const float* A;      // [H]
  const float* D_skip; // [H]
  const float* S0;     // [B, H, P, N] or null
  float* y;            // [B, L, H, P]
  float* S_final;      // [B, H, P, N] or null
  void* status;
  int64_t L;
  int B, H;
};

// Byte offset of the 16-byte chunk `c` of row `r` inside a 128-byte-swizzled box.
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Two values as bf16 pairs hi = bf16(v), lo = bf16(v - hi).
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack2(a, b);
  lo = pack2(a - bf16lo(hi), b - bf16hi(hi));
}

}  // namespace

__global__ void __launch_bounds__(256, 1)
    ssd_chunk_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_x, const SsdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* cum = reinterpret_cast<float*>(sm + SsdSmem::CUM);
  float* dg = reinterpret_cast<float*>(sm + SsdSmem::DG);
  float* wsum = reinterpret_cast<float*>(sm + SsdSmem::WSUM);
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + SsdSmem::BAR);  // [2]: copies into buffer 0, 1
  uint64_t* bar_mma = bar_tma + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SsdSmem::MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SsdSmem::MISC + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // two threads per row i = TMEM lane i: warps w and w + 4 share a lane quarter and split the
  // row's columns (half 0: the first half of every row's columns, half 1: the second)
  const int row = 32 * (warp & 3) + lane, half = warp >> 2;
  const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const float Ah = p.A[h], Dh = p.D_skip[h];
  const int nchunks = (int)((p.L + SQ - 1) / SQ);

  if (tid == 0) {
    mbar_init(&bar_tma[0], 1);
    mbar_init(&bar_tma[1], 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *abort_flag = 0;
    prefetch_tmap(&tm_c);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_x);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tlane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // this warp's lane quarter

  constexpr uint32_t tx_bytes = 2 * kBox + 2 * kBox + kBox;
  auto issue_loads = [&](int c) {  // chunk c into buffer c & 1
    uint64_t* bar = &bar_tma[c & 1];
    uint8_t* tile = sm + (c & 1) * SsdSmem::TILE;
    mbar_arrive_expect_tx(bar, tx_bytes);
    const int t0 = c * SQ;
    tma_load_3d(tile + SsdSmem::TC, &tm_c, bar, 0, t0, b);
    tma_load_3d(tile + SsdSmem::TC + kBox, &tm_c, bar, 64, t0, b);
    tma_load_3d(tile + SsdSmem::TB, &tm_b, bar, 0, t0, b);
    tma_load_3d(tile + SsdSmem::TB + kBox, &tm_b, bar, 64, t0, b);
    tma_load_3d(tile + SsdSmem::TX, &tm_x, bar, h * SP, t0, b);
  };

  // the carried state: Sᵀ[n][p] (row n = TMEM lane n; this thread's 32 columns p) into TMEM (fp32)
  // and its hi/lo copy
  {
    uint32_t r[32], hi[16], lo[16];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int pp = half * 32 + j;
      const float v = p.S0 != nullptr ? p.S0[(((size_t)b * p.H + h) * SP + pp) * SN + row] : 0.f;
      r[j] = __float_as_uint(v);
      if (j & 1) split2(__uint_as_float(r[j - 1]), v, hi[j >> 1], lo[j >> 1]);
    }
    tmem_st32(tlane + kColS + half * 32, r);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      *reinterpret_cast<uint4*>(sm + SsdSmem::S + swz(row, half * 4 + c)) =
          make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
      *reinterpret_cast<uint4*>(sm + SsdSmem::S + kBox + swz(row, half * 4 + c)) =
          make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
    }
    tmem_wait_st();
    fence_proxy_async_smem();
  }
  if (tid == 0) issue_loads(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  uint32_t ph_tma[2] = {0, 0}, ph_mma = 0;
  bool tma_pending[2] = {true, false}, mma_pending = false;  // copies / MMAs issued and not yet waited for
  const uint32_t id_qq = idesc_bf16(SQ, SQ, /*b_mn_major=*/false);        // G = C Bᵀ
  const uint32_t id_qp = idesc_bf16(SQ, SP, /*b_mn_major=*/true);         // Y1 = W X, Y2 = C Sᵀ
  const uint32_t id_st = idesc_bf16(SN, SP, /*b_mn_major=*/true, true);   // Sᵀ += Bᵀ X_w
  const uint32_t sXW = smem_u32(sm + SsdSmem::XW), sS = smem_u32(sm + SsdSmem::S);
  // every wait ends in a CTA-wide vote, so that all threads leave the loop together
  auto vote_abort = [&](bool ok_here) -> bool {
    if (!ok_here) *abort_flag = 1;
    __syncthreads();
    return *abort_flag != 0;
  };
  // the first chunk's Δ and gate of token `row` (warps 0-3); later chunks' are loaded a chunk ahead
  float dl_next = 0.f, gt_next = 0.f;
  if (half == 0 && row < p.L) {
    dl_next = p.delta[((size_t)b * p.L + row) * p.H + h];
    gt_next = p.gates[(size_t)b * p.L + row];
  }

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t = (int64_t)c * SQ + row;
    const float gt = gt_next;
    const int buf = c & 1;
    uint8_t* tile = sm + buf * SsdSmem::TILE;
    const uint32_t sC = smem_u32(tile + SsdSmem::TC), sB = smem_u32(tile + SsdSmem::TB),
                   sX = smem_u32(tile + SsdSmem::TX);
    // the next chunk's tiles into the other buffer (chunk c - 1, its last reader, is finished)
    if (c + 1 < nchunks) {
      if (tid == 0) issue_loads(c + 1);
      tma_pending[buf ^ 1] = true;
    }
    // the chunk's log decays: cum = inclusive prefix sum of Δ A_h over the 128 tokens (warps 0-3)
    if (half == 0) {
      float v = dl_next * Ah;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (lane == 31) wsum[warp] = v;
      dg[row] = dl_next * gt;
      cum[row] = v;  // finished below with the earlier warps' totals
    }
    __syncthreads();
    if (half == 0) {
      float add = 0.f;
      for (int w = 0; w < warp; ++w) add += wsum[w];
      cum[row] += add;
    }

    // the chunk's tiles have landed: G = C Bᵀ and Y2 = C S_inᵀ (K = n)
    const bool got = mbar_wait(&bar_tma[buf], ph_tma[buf], abort_flag);
    ph_tma[buf] ^= 1u;
    if (vote_abort(got)) break;  // (its barrier also publishes cum)
    tma_pending[buf] = false;
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < SN / 16; ++ks) {
        const uint32_t koff = (uint32_t)((ks >> 2) * kBox + (ks & 3) * 32);
        mma_bf16(tmem + kColG, smem_desc(sC + koff, 16, 1024, kLayoutSW128),
                 smem_desc(sB + koff, 16, 1024, kLayoutSW128), id_qq, ks > 0 ? 1u : 0u);
        mma_bf16(tmem + kColY2, smem_desc(sC + koff, 16, 1024, kLayoutSW128),
                 smem_desc(sS + ks * 16 * 128, 8192, 1024, kLayoutSW128), id_qp, ks > 0 ? 1u : 0u);
        mma_bf16(tmem + kColY2, smem_desc(sC + koff, 16, 1024, kLayoutSW128),
                 smem_desc(sS + kBox + ks * 16 * 128, 8192, 1024, kLayoutSW128), id_qp, 1u);
      }
      mma_commit(bar_mma);
    }
    mma_pending = true;
    // X_w rows (row s, this thread's 4 of the 8 16-byte chunks): exp(cum[Q-1] - cum[s]) Δ_s g_s X[s]
    {
      const float ws = __expf(cum[SQ - 1] - cum[row]) * dg[row];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const int cc = half * 4 + c4;
        const uint4 q = *reinterpret_cast<const uint4*>(tile + SsdSmem::TX + swz(row, cc));
        const uint32_t in[4] = {q.x, q.y, q.z, q.w};
        uint32_t o[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split2(bf16lo(in[e]) * ws, bf16hi(in[e]) * ws, o[e], l[e]);
        *reinterpret_cast<uint4*>(sm + SsdSmem::XW + swz(row, cc)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(sm + SsdSmem::XW + kBox + swz(row, cc)) = make_uint4(l[0], l[1], l[2], l[3]);
      }
    }
    // Sᵀ (row n, this thread's 32 columns) decays by the chunk's total before the state MMA adds to it
    {
      const float tot = __expf(cum[SQ - 1]);
      float f[32];
      tmem_ld32(tlane + kColS + half * 32, f);
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(f[j] * tot);
      tmem_st32(tlane + kColS + half * 32, r);
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    const bool done1 = mbar_wait(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1u;
    if (vote_abort(done1)) break;
    mma_pending = false;
    tc_fence_after();
    // W rows (row i, this thread's 64 columns s): exp(cum[i] - cum[s]) Δ_s g_s G[i, s] for s <= i, else 0
    {
      const float ci = cum[row];
      for (int bb = 0; bb < 2; ++bb) {  // 32 columns s at a time
        const int blk = half * 2 + bb;
        float gr[32];
        tmem_ld32(tlane + kColG + blk * 32, gr);
        uint32_t w16[16], l16[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const int s0 = blk * 32 + j;
          const float w0 = s0 <= row ? __expf(ci - cum[s0]) * dg[s0] * gr[j] : 0.f;
          const float w1 = s0 + 1 <= row ? __expf(ci - cum[s0 + 1]) * dg[s0 + 1] * gr[j + 1] : 0.f;
          split2(w0, w1, w16[j >> 1], l16[j >> 1]);
        }
        // columns s = blk*32 .. +31 of row i: 16 packed bf16 pairs of hi and of lo
        tmem_st16(tlane + kColW + blk * 16, w16);
        tmem_st16(tlane + kColW + 64 + blk * 16, l16);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    // Y1 = W X (W from tensor memory) and Sᵀ += Bᵀ X_w (K = s)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < SQ / 16; ++ks) {
        mma_bf16_ts(tmem + kColY1, tmem + kColW + ks * 8, smem_desc(sX + ks * 16 * 128, 8192, 1024, kLayoutSW128),
                    id_qp, ks > 0 ? 1u : 0u);
        mma_bf16_ts(tmem + kColY1, tmem + kColW + 64 + ks * 8,
                    smem_desc(sX + ks * 16 * 128, 8192, 1024, kLayoutSW128), id_qp, 1u);
        mma_bf16(tmem + kColS, smem_desc(sB + ks * 16 * 128, kBox, 1024, kLayoutSW128),
                 smem_desc(sXW + ks * 16 * 128, 8192, 1024, kLayoutSW128), id_st, 1u);
        mma_bf16(tmem + kColS, smem_desc(sB + ks * 16 * 128, kBox, 1024, kLayoutSW128),
                 smem_desc(sXW + kBox + ks * 16 * 128, 8192, 1024, kLayoutSW128), id_st, 1u);
      }
      mma_commit(bar_mma);
    }
    mma_pending = true;
    const bool done2 = mbar_wait(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1u;
    tc_fence_after();
    // this token's X row (the skip term; this thread's 4 chunks) leaves the tile before the next
    // chunk's copies refill it
    uint4 xr[4];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) xr[c4] = *reinterpret_cast<const uint4*>(tile + SsdSmem::TX + swz(row, half * 4 + c4));
    if (vote_abort(done2)) break;
    mma_pending = false;
    // the next chunk's Δ and gate, in flight while this chunk's outputs are written
    if (half == 0) {
      const int64_t tn = (int64_t)(c + 1) * SQ + row;
      dl_next = tn < p.L ? p.delta[((size_t)b * p.L + tn) * p.H + h] : 0.f;
      gt_next = tn < p.L ? p.gates[(size_t)b * p.L + tn] : 0.f;
    }
    // outputs (row i, this thread's 32 channels p): y = Y1 + exp(cum[i]) Y2 + D_h g_i X[i]
    {
      const float e_i = __expf(cum[row]);
      const float dgx = Dh * p.gates[(size_t)b * p.L + (t < p.L ? t : 0)];
      float* yrow = p.y + (((size_t)b * p.L + t) * p.H + h) * SP + half * 32;
      float y1[32], y2[32];
      tmem_ld32(tlane + kColY1 + half * 32, y1);
      tmem_ld32(tlane + kColY2 + half * 32, y2);
      if (t < p.L) {
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          const uint4 q = xr[j / 8];
          const float xv[8] = {bf16lo(q.x), bf16hi(q.x), bf16lo(q.y), bf16hi(q.y),
                               bf16lo(q.z), bf16hi(q.z), bf16lo(q.w), bf16hi(q.w)};
          float o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = fmaf(e_i, y2[j + e], y1[j + e]) + dgx * xv[e];
          *reinterpret_cast<float4*>(yrow + j) = make_float4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<float4*>(yrow + j + 4) = make_float4(o[4], o[5], o[6], o[7]);
        }
      }
      (void)gt;
    }
    // the new state's hi/lo copy Sᵀ[n][p] (row n, this thread's 32 columns), the next chunk's Y2 operand
    {
      float f[32];
      tmem_ld32(tlane + kColS + half * 32, f);
      uint32_t w16[16], l16[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) split2(f[j], f[j + 1], w16[j >> 1], l16[j >> 1]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        *reinterpret_cast<uint4*>(sm + SsdSmem::S + swz(row, half * 4 + cc)) =
            make_uint4(w16[4 * cc], w16[4 * cc + 1], w16[4 * cc + 2], w16[4 * cc + 3]);
        *reinterpret_cast<uint4*>(sm + SsdSmem::S + kBox + swz(row, half * 4 + cc)) =
            make_uint4(l16[4 * cc], l16[4 * cc + 1], l16[4 * cc + 2], l16[4 * cc + 3]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  const bool aborted = *abort_flag != 0;
  if (aborted) {
    if (tid == 0) {
      record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 51, blockIdx.x, 0);
      // let the copies and MMAs still in flight finish before TMEM and shared memory go away
      // (bounded; the flag is ignored here)
      for (int bb = 0; bb < 2; ++bb) {
        const uint64_t w0 = globaltimer_ns();
        if (tma_pending[bb])
          while (!mbar_try_wait(&bar_tma[bb], ph_tma[bb]) && globaltimer_ns() - w0 < kWaitLimitNs) {
          }
      }
      const uint64_t w1 = globaltimer_ns();
      if (mma_pending)
        while (!mbar_try_wait(bar_mma, ph_mma) && globaltimer_ns() - w1 < kWaitLimitNs) {
        }
    }
  } else if (p.S_final != nullptr) {
    // the final state Sᵀ[n][p] -> S_final[b, h, p, n] (row n, this thread's 32 columns)
    float f[32];
    tmem_ld32(tlane + kColS + half * 32, f);
#pragma unroll
    for (int j = 0; j < 32; ++j) p.S_final[(((size_t)b * p.H + h) * SP + half * 32 + j) * SN + row] = f[j];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- host -----------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 ssd_encode_fn() {
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

// [B, L, inner] bf16 rows viewed as 3-D, box {64, 128 tokens, 1}, 128-byte swizzle; rows past L
// read as zeros.
bool ssd_map(CUtensorMap* m, const void* base, int64_t inner, int64_t L, int64_t B) {
  auto fn = ssd_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t str[2] = {(cuuint64_t)(inner * 2), (cuuint64_t)(inner * L * 2)};
  cuuint32_t box[3] = {64, (cuuint32_t)SQ, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, str, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool ssd_supported(int P, int N, int k) { return P == SP && N == SN && k == 1; }

cudaError_t run_ssd(const void* X, const void* Bm, const void* Cmix, const float* gates, const float* delta,
                    const float* A, const float* D_skip, const float* S0, float* y, float* S_final, void* status,
                    int64_t L, int B, int H, cudaStream_t s) {
  CUtensorMap tc, tb, tx;
  if (!ssd_map(&tc, Cmix, SN, L, B) || !ssd_map(&tb, Bm, SN, L, B) || !ssd_map(&tx, X, (int64_t)H * SP, L, B))
    return cudaErrorInvalidValue;
  SsdParams p{gates, delta, A, D_skip, S0, y, S_final, status, L, B, H};
  const size_t smem = 1024 + SsdSmem::BYTES;
  cudaError_t e = cudaFuncSetAttribute(ssd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ssd_chunk_kernel<<<(unsigned)(B * H), 256, smem, s>>>(tc, tb, tx, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace swimba
