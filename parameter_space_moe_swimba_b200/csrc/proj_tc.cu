// Mixed expert projection on the tcgen05 tensor cores (bf16 x and tables, fp32 accumulation).
//
// Source: "Swimba: Switch Mamba Model Scales State Space Models", §2 "Generación de Parámetros" /
// "Mezcla en el Espacio de Parámetros" (es), "Kernmechanisme van Swimba" (nl): every expert has
// its own linear projections producing token-dependent streams, and the streams of the active
// experts are mixed with the router weights before the single recurrence. The pages attribute
// Swimba's serving overhead to routing and to this "dispersion" of tokens over experts.
//
// Design. Tokens are bucketed by the SET of experts they selected (k <= 2: an expert, or an
// unordered expert pair), so every 128-row tile shares its k weight tables and x is read once:
//   bucket kernels  a stable counting sort of the tokens by group: per-block histograms, group
//                   offsets + tile list, scatter of token ids (ascending inside every group).
//   stage 1         per tile: acc_j = X_tile · W_x^{e_j}  (j < k; TMEM, M=128, N=R+2N, K=D).
//                   x rows are gathered with cp.async 16-byte copies into the 128-byte-swizzled
//                   layout (a deep ring of its own); W_x boxes (TMA) are
//                   MN-major 128-byte-swizzled tiles of the [E, D, R+2N] table as stored.
//                   Epilogue: B_mix, C_mix = Σ_j g_j (B^j, C^j) -> global; the gated low-rank
//                   rows g_j dt_low^j, split into bf16 hi + lo parts (hi = bf16(v), lo =
//                   bf16(v - hi)), -> workspace as A'[row] = [hi_0 | hi_1 | lo_0 | lo_1].
//   stage 2         per (tile, 256-column chunk): acc = Σ_j (hi_j + lo_j) · W_dt^{e_j}
//                   (each W_dt box feeds two MMAs), i.e. Σ_j g_j dt_low^j W_dt^{e_j} with the
//                   low-rank operand carried to about 16 significant bits. Epilogue:
//                   + Σ_j g_j b_dt^{e_j}, softplus, store delta rows of the tile's tokens.
// Both GEMM kernels are persistent and warp specialised: warp 0 issues TMA, warp 1 owns TMEM and
// issues the MMAs, the remaining warps drain TMEM. Every mbarrier wait is bounded (1 s); on a
// timeout the CTA records SWIMBA_ERR_TIMEOUT in the workspace status block, lets its copies in
// flight land, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "proj.cuh"
#include "sm100.cuh"

namespace swimba {

using namespace sm100;

namespace {

constexpr int BM = 128;        // rows (token slots) per tile
constexpr int BK1 = 64;        // stage-1 K slice per ring stage (128 bytes of bf16 per row)
// Stage 1 keeps two rings: the gathered x rows (A, 16 KB a slot) are the slow, latency-bound
// loads, so their ring is deeper than the W_x ring (up to 6 TMA boxes of 8 KB a slot, L2-resident).
constexpr int kStagesA = 5;
constexpr int kSlotA = 16384;
constexpr int kStagesW = 3;
constexpr int kSlotW = 49152;
constexpr int NC = 256;        // stage-2 output columns per chunk
constexpr int kStages2 = 4;
constexpr int kSlot2 = 16384;  // 4 W_dt boxes of up to 32 rows x 128 B
constexpr int kBiasW = 2 * 64 * 4;  // per epilogue warp: the k experts' biases of its 64 columns
constexpr int kApBox = BM * 128;  // one 64-column box of A' (16 KB)

struct TileInfo {
  int row_begin, rows, e0, e1;
};

constexpr int kBucketBlock = 256;  // tokens per counting block of the bucketing sort
constexpr int kMaxGroups = 160;    // E <= 16: at most 120 groups for k = 2

struct TcLayout {
  size_t group_of, blockhist, blockbase, offsets, num_tiles, tiles, slot_tok, slot_gate, aprime, partial, total;
  int G, nb, max_tiles, K2, R_pad;
  int split, kper;  // stage-1 K split (1: none) and K slices per split
};

// Stage-1 K split for few tiles (decode steps, short prompts): each tile's K range is divided
// among `split` CTAs so that the tiles x splits work items reach about one per SM of a B200;
// the partial accumulators are summed by stage1_finish_kernel. 1 when the tiles alone fill it.
inline void stage1_split(int max_tiles, int ksteps, int& split, int& kper) {
  split = 1;
  if (max_tiles * 2 <= 148) split = std::min(std::min(8, 148 / std::max(1, max_tiles)), ksteps);
  split = std::max(split, 1);
  kper = (ksteps + split - 1) / split;
  split = (ksteps + kper - 1) / kper;  // no empty split
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

TcLayout tc_layout(int64_t T, int E, int K, int R, int D) {
  TcLayout L{};
  L.G = K == 1 ? E : E * (E - 1) / 2;
  L.max_tiles = (int)((T + BM - 1) / BM) + L.G;
  L.R_pad = (R + 63) / 64 * 64;
  L.K2 = 2 * K * L.R_pad;  // [hi_0 .. hi_{k-1} | lo_0 .. lo_{k-1}], each R_pad wide
  size_t o = kStatusBytes;
  L.nb = (int)((T + kBucketBlock - 1) / kBucketBlock);
  L.group_of = o; o = align_up(o + 4 * (size_t)T, 256);
  L.blockhist = o; o = align_up(o + 4 * (size_t)L.nb * L.G, 256);
  L.blockbase = o; o = align_up(o + 4 * (size_t)L.nb * L.G, 256);
  L.offsets = o; o = align_up(o + 4 * (size_t)(L.G + 1), 256);
  L.num_tiles = o; o += 256;
  L.tiles = o; o = align_up(o + sizeof(TileInfo) * (size_t)L.max_tiles, 256);
  L.slot_tok = o; o = align_up(o + 4 * (size_t)T, 256);
  L.slot_gate = o; o = align_up(o + 4 * (size_t)T * K, 1024);
  L.aprime = o; o = align_up(o + 2 * (size_t)L.max_tiles * BM * L.K2, 256);
  stage1_split(L.max_tiles, D / BK1, L.split, L.kper);
  const int W = R + 2 * 16;
  L.partial = o;
  if (L.split > 1) o += 4 * (size_t)L.split * L.max_tiles * K * W * BM;
  L.total = align_up(o, 256);
  return L;
}

__device__ __forceinline__ int clamp_e(int e, int E) { return min(max(e, 0), E - 1); }

// ---- bucketing -----------------------------------------------------------------------------------
// Tokens are bucketed by their expert set with a stable counting sort: inside a group, slots keep
// ascending token order, so a tile's rows are nearby tokens (the stage-2 Δ stores of a tile stay
// within a narrow address range) and the slot order does not depend on scheduling.
// Group id of a sorted expert set: k = 1 -> e; k = 2 (a < b) -> a + b(b-1)/2.

template <int K>
__device__ __forceinline__ int group_id(const int32_t* idx, int64_t t, int E) {
  if (K == 1) return clamp_e(idx[t], E);
  const int e0 = clamp_e(idx[2 * t], E), e1 = clamp_e(idx[2 * t + 1], E);
  const int a = min(e0, e1), b = max(e0, e1);
  return a + b * (b - 1) / 2;
}

// Per block of kBucketBlock tokens: the count of every group -> blockhist[block][G].
template <int K>
__global__ void __launch_bounds__(kBucketBlock) group_count_kernel(const int32_t* idx, int64_t T, int E, int G,
                                                                   int* group_of, int* blockhist) {
  __shared__ int hist[kMaxGroups];
  for (int g = threadIdx.x; g < G; g += blockDim.x) hist[g] = 0;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    const int g = group_id<K>(idx, t, E);
    group_of[t] = g;
    atomicAdd(&hist[g], 1);
  }
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += blockDim.x) blockhist[(size_t)blockIdx.x * G + g] = hist[g];
}

// One CTA: group sizes and offsets, every block's first slot per group (blockbase, in block
// order), and the tile list (tiles of up to BM rows, never crossing a group). A warp per group
// sums and prefix-sums the group's per-block counts 32 blocks at a time.
template <int K>
__global__ void __launch_bounds__(256) group_scan_kernel(const int* blockhist, int nb, int G, int* offsets,
                                                         int* blockbase, int* num_tiles, TileInfo* tiles) {
  __shared__ int s_cnt[kMaxGroups];
  __shared__ int s_off[kMaxGroups + 1];
  __shared__ int s_tstart[kMaxGroups + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int g = warp; g < G; g += nwarps) {
    int c = 0;
    for (int bb = lane; bb < nb; bb += 32) c += blockhist[(size_t)bb * G + g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) s_cnt[g] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = 0, nt = 0;
    for (int g = 0; g < G; ++g) {
      s_off[g] = off;
      s_tstart[g] = nt;
      offsets[g] = off;
      off += s_cnt[g];
      nt += (s_cnt[g] + BM - 1) / BM;
    }
    s_off[G] = off;
    s_tstart[G] = nt;
    offsets[G] = off;
    *num_tiles = nt;
  }
  __syncthreads();
  for (int g = warp; g < G; g += nwarps) {
    int carry = s_off[g];
    for (int b0 = 0; b0 < nb; b0 += 32) {
      const int bb = b0 + lane;
      const int v = bb < nb ? blockhist[(size_t)bb * G + g] : 0;
      int incl = v;  // inclusive warp scan
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (bb < nb) blockbase[(size_t)bb * G + g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  const int nt = s_tstart[G];
  for (int tile = threadIdx.x; tile < nt; tile += blockDim.x) {
    int lo = 0, hi = G - 1;  // last g with s_tstart[g] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int i = tile - s_tstart[g];
    TileInfo ti;
    ti.row_begin = s_off[g] + i * BM;
    ti.rows = min(BM, s_cnt[g] - i * BM);
    if (K == 1) {
      ti.e0 = g;
      ti.e1 = g;
    } else {
      int b = 1;
      while ((b + 1) * b / 2 <= g) ++b;
      ti.e1 = b;
      ti.e0 = g - b * (b - 1) / 2;
    }
    tiles[tile] = ti;
  }
}

// Slot of every token: its block's first slot for its group plus its rank among the block's
// earlier tokens of the same group (warp match + per-warp counts), i.e. a stable order.
template <int K>
__global__ void __launch_bounds__(kBucketBlock) group_scatter_kernel(const int32_t* idx, const float* gates, int64_t T,
                                                                     int E, int G, const int* group_of,
                                                                     const int* blockbase, int* slot_tok,
                                                                     float* slot_gate) {
  __shared__ int warpcnt[kBucketBlock / 32][kMaxGroups];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kBucketBlock / 32) * kMaxGroups; i += blockDim.x) (&warpcnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const bool valid = t < T;
  const int g = valid ? group_of[t] : -1;
  const unsigned same = __match_any_sync(0xffffffffu, g);
  const int lane_rank = __popc(same & ((1u << lane) - 1u));
  if (valid && lane_rank == 0) warpcnt[warp][g] = __popc(same);
  __syncthreads();
  if (!valid) return;
  int pos = blockbase[(size_t)blockIdx.x * G + g] + lane_rank;
  for (int w = 0; w < warp; ++w) pos += warpcnt[w][g];
  slot_tok[pos] = (int)t;
  if (K == 1) {
    slot_gate[pos] = gates[t];
  } else {
    const int e0 = clamp_e(idx[2 * t], E), e1 = clamp_e(idx[2 * t + 1], E);
    const float g0 = gates[2 * t], g1 = gates[2 * t + 1];
    // gates in the group's expert order (ascending expert index)
    slot_gate[2 * pos] = e0 <= e1 ? g0 : g1;
    slot_gate[2 * pos + 1] = e0 <= e1 ? g1 : g0;
  }
}

// The three bucketing kernels above in one CTA, for few tokens (decode steps, short prompts), where
// their work is a few microseconds of launch and latency each. Same result: group sizes and offsets,
// the tile list, and the stable slot order (tokens ascending inside every group), taken over
// chunks of kSmallBucketThreads tokens in order, each chunk ranked with warp matches and per-warp
// counts and placed after the slots of the earlier chunks.
constexpr int kSmallBucketThreads = 1024;
constexpr int kSmallBucketT = 4096;  // tokens up to which the one-CTA kernel is used

template <int K>
__global__ void __launch_bounds__(kSmallBucketThreads) group_bucket_small_kernel(const int32_t* idx, const float* gates,
                                                                                 int T, int E, int G, int* offsets,
                                                                                 int* num_tiles, TileInfo* tiles,
                                                                                 int* slot_tok, float* slot_gate) {
  constexpr int kChunks = kSmallBucketT / kSmallBucketThreads;
  constexpr int kWarps = kSmallBucketThreads / 32;
  __shared__ int s_cnt[kMaxGroups];
  __shared__ int s_off[kMaxGroups + 1];
  __shared__ int s_tstart[kMaxGroups + 1];
  __shared__ int s_run[kMaxGroups];
  __shared__ int warpcnt[kWarps][kMaxGroups];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();
  pdl_wait();  // the router has completed
  for (int g = tid; g < G; g += kSmallBucketThreads) s_cnt[g] = 0;
  __syncthreads();
  int gs[kChunks];
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int t = c * kSmallBucketThreads + tid;
    gs[c] = t < T ? group_id<K>(idx, t, E) : -1;
    if (gs[c] >= 0) atomicAdd(&s_cnt[gs[c]], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0, nt = 0;
    for (int g = 0; g < G; ++g) {
      s_off[g] = off;
      s_run[g] = off;
      s_tstart[g] = nt;
      offsets[g] = off;
      off += s_cnt[g];
      nt += (s_cnt[g] + BM - 1) / BM;
    }
    s_off[G] = off;
    s_tstart[G] = nt;
    offsets[G] = off;
    *num_tiles = nt;
  }
  __syncthreads();
  const int nt = s_tstart[G];
  for (int tile = tid; tile < nt; tile += kSmallBucketThreads) {
    int lo = 0, hi = G - 1;  // last g with s_tstart[g] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int i = tile - s_tstart[g];
    TileInfo ti;
    ti.row_begin = s_off[g] + i * BM;
    ti.rows = min(BM, s_cnt[g] - i * BM);
    if (K == 1) {
      ti.e0 = g;
      ti.e1 = g;
    } else {
      int b = 1;
      while ((b + 1) * b / 2 <= g) ++b;
      ti.e1 = b;
      ti.e0 = g - b * (b - 1) / 2;
    }
    tiles[tile] = ti;
  }
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    if (c * kSmallBucketThreads >= T) break;  // uniform over the CTA
    for (int g = lane; g < G; g += 32) warpcnt[warp][g] = 0;
    __syncthreads();
    const int g = gs[c];
    const unsigned same = __match_any_sync(0xffffffffu, g);
    const int lane_rank = __popc(same & ((1u << lane) - 1u));
    if (g >= 0 && lane_rank == 0) warpcnt[warp][g] = __popc(same);
    __syncthreads();
    if (g >= 0) {
      int pos = s_run[g] + lane_rank;
      for (int w = 0; w < warp; ++w) pos += warpcnt[w][g];
      const int t = c * kSmallBucketThreads + tid;
      slot_tok[pos] = t;
      if (K == 1) {
        slot_gate[pos] = gates[t];
      } else {
        const int e0 = clamp_e(idx[2 * t], E), e1 = clamp_e(idx[2 * t + 1], E);
        const float g0 = gates[2 * t], g1 = gates[2 * t + 1];
        slot_gate[2 * pos] = e0 <= e1 ? g0 : g1;
        slot_gate[2 * pos + 1] = e0 <= e1 ? g1 : g0;
      }
    }
    __syncthreads();
    for (int gg = tid; gg < G; gg += kSmallBucketThreads) {
      int add = 0;
      for (int w = 0; w < kWarps; ++w) add += warpcnt[w][gg];
      s_run[gg] += add;
    }
    __syncthreads();
  }
}

// ---- stage 1 ---------------------------------------------------------------------------------------
struct Stage1Params {
  int D, W, R, N, R_pad, K2, nbw;  // nbw: 64-column W_x boxes per expert
  int split, kper;                 // K split (1: the epilogue finishes the tile) and slices per split
  int xshift;                      // x row of slot token v: v >> xshift (1: slots are (token, slot) pairs)
  const __nv_bfloat16* x;          // [T, D]
  float* partial;                  // split > 1: [tile * split + s][k * W + c][128 rows] fp32
  const int* num_tiles;
  const TileInfo* tiles;
  const int* slot_tok;
  const float* slot_gate;
  __nv_bfloat16* aprime;
  float* B_mix;
  float* C_mix;
  void* status;
};

// Two floats a, b as packed bf16 pairs: hi = (bf16(a), bf16(b)), lo = the bf16 of the remainders.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 ha = __float2bfloat16_rn(a), hb = __float2bfloat16_rn(b);
  const __nv_bfloat16 la = __float2bfloat16_rn(a - __bfloat162float(ha));
  const __nv_bfloat16 lb = __float2bfloat16_rn(b - __bfloat162float(hb));
  hi = (uint32_t)__bfloat16_as_ushort(ha) | ((uint32_t)__bfloat16_as_ushort(hb) << 16);
  lo = (uint32_t)__bfloat16_as_ushort(la) | ((uint32_t)__bfloat16_as_ushort(lb) << 16);
}

// After a failed wait: let the producer's copies in flight land (bounded, ignoring the abort flag).
__device__ void drain_ring(uint64_t* full, int stages, int stage, uint32_t phase, int issued) {
  for (int i = 0; i < min(issued, stages); ++i) {
    int s = stage - 1 - i;
    uint32_t ph = phase;
    if (s < 0) {
      s += stages;
      ph ^= 1u;
    }
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&full[s], ph) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
  }
}

// Commit to a fresh barrier and wait (bounded) until every MMA this thread issued has completed,
// so that TMEM can be released.
__device__ __forceinline__ void wait_all_mma(uint64_t* done) {
  mma_commit(done);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(done, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
  }
}

template <int K>
__global__ void __launch_bounds__(224, 1)
    proj_stage1_kernel(const __grid_constant__ CUtensorMap tm_wx, const Stage1Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring_a = smem;
  uint8_t* ring_w = smem + kStagesA * kSlotA;
  uint64_t* full_a = reinterpret_cast<uint64_t*>(ring_w + kStagesW * kSlotW);
  uint64_t* empty_a = full_a + kStagesA;
  uint64_t* full_w = empty_a + kStagesA;
  uint64_t* empty_w = full_w + kStagesW;
  uint64_t* acc_full = empty_w + kStagesW;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* done = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // warp 0: x-row gathers (cp.async); warp 1: MMA; warps 2-5: epilogue; warp 6: W_x boxes (TMA)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&full_a[s], 1);
      mbar_init(&empty_a[s], 1);
    }
    for (int s = 0; s < kStagesW; ++s) {
      mbar_init(&full_w[s], 1);
      mbar_init(&empty_w[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_wx);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // the bucketing (or the previous stage) has completed
  const int num_tiles = *p.num_tiles;
  const int ksteps = p.D / BK1;
  const uint32_t w_bytes = (uint32_t)(K * p.nbw) * 8192u;

  if (warp == 0) {
    // ---------------- producer of A: 128 gathered x rows per K slice ----------------
    // cp.async 16-byte copies (lanes 8i..8i+7 fetch one 128-byte row slice, 4 rows per
    // instruction) written straight into the 128-byte-swizzled layout the MMA reads. The slot is
    // handed to the MMA LAG slots later, once this thread's copies into it have landed (wait_group)
    // and been made visible to the tensor-core proxy (fence). Plain copies keep more rows in flight
    // than the TMA row gathers did (stage 1: 171 -> ~115 µs on the Mamba-1.4B-like shape).
    constexpr int LAG = 3;  // < kStagesA
    int stage = 0, n = 0, retired = 0;
    uint32_t phase = 0;
    bool ok = true;
    const int ch = lane & 7;
    for (int it = blockIdx.x; it < num_tiles * p.split && ok; it += gridDim.x) {
      const int tile = it / p.split, sp = it - tile * p.split;
      const int kb = sp * p.kper, ke = min(ksteps, kb + p.kper);
      const TileInfo ti = p.tiles[tile];
      int tokrow[32];  // token of tile row 4i + lane/8
#pragma unroll
      for (int i = 0; i < 32; ++i)
        tokrow[i] = p.slot_tok[ti.row_begin + min(4 * i + (lane >> 3), ti.rows - 1)] >> p.xshift;
      for (int ks = kb; ks < ke; ++ks) {
        if (!mbar_wait(&empty_a[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t sbase = smem_u32(ring_a + stage * kSlotA);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = 4 * i + (lane >> 3);
          const __nv_bfloat16* src = p.x + (size_t)tokrow[i] * p.D + ks * BK1 + ch * 8;
          cp_async16(sbase + r * 128 + ((ch ^ (r & 7)) << 4), src);
        }
        cp_async_commit();
        ++n;
        if (n - retired > LAG) {
          cp_async_wait<LAG>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full_a[retired % kStagesA]);
          ++retired;
        }
        if (++stage == kStagesA) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    for (; retired < n; ++retired)
      if (lane == 0) mbar_arrive(&full_a[retired % kStagesA]);
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 11, blockIdx.x, 0);
    }
  } else if (warp == 6) {
    // ---------------- producer of B: the tile's k W_x tables, K slice by K slice ----------------
    int stage = 0, issued = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < num_tiles * p.split && ok; it += gridDim.x) {
      const int tile = it / p.split, sp = it - tile * p.split;
      const int kb = sp * p.kper, ke = min(ksteps, kb + p.kper);
      const TileInfo ti = p.tiles[tile];
      const int ej[2] = {ti.e0, ti.e1};
      for (int ks = kb; ks < ke; ++ks) {
        if (!mbar_wait(&empty_w[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* slot = ring_w + stage * kSlotW;
        if (lane == 0) mbar_arrive_expect_tx(&full_w[stage], w_bytes);
        __syncwarp();
        if (lane < K * p.nbw) {
          const int j = lane / p.nbw, nb = lane - j * p.nbw;
          tma_load_3d(slot + lane * 8192, &tm_wx, &full_w[stage], nb * 64, ks * BK1, ej[j]);
        }
        ++issued;
        if (++stage == kStagesW) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 14, blockIdx.x, 0);
      drain_ring(full_w, kStagesW, stage, phase, issued);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BM, p.W, /*b_mn_major=*/true);
      int sa = 0, sw = 0;
      uint32_t pa = 0, pw = 0, acc_phase = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < num_tiles * p.split && ok; it += gridDim.x) {
        const int sp = it % p.split;
        const int kb = sp * p.kper, ke = min(ksteps, kb + p.kper);
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int ks = kb; ks < ke; ++ks) {
          if (!mbar_wait(&full_a[sa], pa, abort_flag) || !mbar_wait(&full_w[sw], pw, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t abase = smem_u32(ring_a + sa * kSlotA);
          const uint32_t wbase = smem_u32(ring_w + sw * kSlotW);
#pragma unroll
          for (int kk = 0; kk < BK1 / 16; ++kk) {
            const uint64_t adesc = smem_desc(abase + kk * 32, 16, 1024, kLayoutSW128);
#pragma unroll
            for (int j = 0; j < K; ++j) {
              const uint64_t bdesc = smem_desc(wbase + j * p.nbw * 8192 + kk * 16 * 128, 8192, 1024, kLayoutSW128);
              mma_bf16(tmem + j * 256, adesc, bdesc, idesc, (ks != kb || kk != 0) ? 1u : 0u);
            }
          }
          mma_commit(&empty_a[sa]);
          mma_commit(&empty_w[sw]);
          if (++sa == kStagesA) {
            sa = 0;
            pa ^= 1u;
          }
          if (++sw == kStagesW) {
            sw = 0;
            pw ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(acc_full);
        acc_phase ^= 1u;
      }
      if (!ok) {
        *abort_flag = 1;
        record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 12, blockIdx.x, 0);
      }
      wait_all_mma(done);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: one TMEM lane (= tile row) per thread ----------------
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
    uint32_t acc_phase = 0;
    for (int it = blockIdx.x; it < num_tiles * p.split; it += gridDim.x) {
      const int tile = it / p.split;
      const TileInfo ti = p.tiles[tile];
      if (!mbar_wait(acc_full, acc_phase, abort_flag)) {
        *abort_flag = 1;
        if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 13, blockIdx.x, tile);
        break;
      }
      acc_phase ^= 1u;
      tc_fence_after();
      if (p.split > 1) {
        // K split: this item's raw accumulators, column-major (lanes = rows write 128 bytes)
        float* pp = p.partial + (size_t)it * K * p.W * BM + row;
        float v[16];
#pragma unroll
        for (int j = 0; j < K; ++j)
          for (int c = 0; c < p.W; c += 16) {
            tmem_ld16(tl + j * 256 + c, v);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c + i < p.W) pp[(size_t)(j * p.W + c + i) * BM] = v[i];
          }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        continue;
      }
      const bool valid = row < ti.rows;
      const int pos = ti.row_begin + min(row, ti.rows - 1);
      const int t = p.slot_tok[pos];
      float g[K];
#pragma unroll
      for (int j = 0; j < K; ++j) g[j] = p.slot_gate[pos * K + j];
      uint4* arow = reinterpret_cast<uint4*>(p.aprime + ((size_t)tile * BM + row) * p.K2);
      float v[16];
#pragma unroll
      for (int j = 0; j < K; ++j) {
        for (int c = 0; c < p.R; c += 16) {
          tmem_ld16(tl + j * 256 + c, v);
          uint32_t hw[8], lw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) split_bf16x2(g[j] * v[2 * i], g[j] * v[2 * i + 1], hw[i], lw[i]);
          const int ohi = (j * p.R_pad + c) / 8, olo = ((K + j) * p.R_pad + c) / 8;
          arow[ohi] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          arow[ohi + 1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
          arow[olo] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          arow[olo + 1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
        }
        for (int c = p.R; c < p.R_pad; c += 8) {
          arow[(j * p.R_pad + c) / 8] = make_uint4(0, 0, 0, 0);
          arow[((K + j) * p.R_pad + c) / 8] = make_uint4(0, 0, 0, 0);
        }
      }
      float bs[16], cs[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) bs[i] = cs[i] = 0.f;
#pragma unroll
      for (int j = 0; j < K; ++j) {
        tmem_ld16(tl + j * 256 + p.R, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) bs[i] = fmaf(g[j], v[i], bs[i]);
        tmem_ld16(tl + j * 256 + p.R + 16, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) cs[i] = fmaf(g[j], v[i], cs[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      if (valid) {
        float4* bo = reinterpret_cast<float4*>(p.B_mix + (size_t)t * 16);
        float4* co = reinterpret_cast<float4*>(p.C_mix + (size_t)t * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          bo[i] = make_float4(bs[4 * i], bs[4 * i + 1], bs[4 * i + 2], bs[4 * i + 3]);
          co[i] = make_float4(cs[4 * i], cs[4 * i + 1], cs[4 * i + 2], cs[4 * i + 3]);
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- stage 2 ---------------------------------------------------------------------------------------
struct Stage2Params {
  int D, R, R_pad, K2, RS;  // RS: W_dt rows per ring stage (32, or 16 when R is not a multiple of 32)
  const int* num_tiles;
  const TileInfo* tiles;
  const int* slot_tok;
  const float* slot_gate;
  const float* b_dt;  // [E, D]
  float* delta;       // softplus of the tile rows' sums; raw != 0: the sums themselves
  int raw;
  void* status;
};

// Finishes a K-split stage 1: sums the splits' partial accumulators (in split order, so the
// result does not depend on scheduling) and applies the same epilogue as the unsplit kernel:
// gated dt_low rows as bf16 hi + lo into A', B_mix and C_mix. Block (tile, group), thread = tile
// row; groups 0 .. k R/8 - 1 are 8 dt_low columns of one expert, the last four are 8 values of
// B_mix or C_mix. The partial buffer is column-major, so each load instruction of a warp reads
// 128 consecutive bytes.
template <int K>
__global__ void __launch_bounds__(128) stage1_finish_kernel(const Stage1Params p) {
  const int tile = blockIdx.x;
  pdl_trigger();
  pdl_wait();
  if (tile >= *p.num_tiles) return;
  const int row = threadIdx.x;
  const TileInfo ti = p.tiles[tile];
  const int pos = ti.row_begin + min(row, ti.rows - 1);
  float g[K];
#pragma unroll
  for (int j = 0; j < K; ++j) g[j] = p.slot_gate[pos * K + j];
  const size_t item_stride = (size_t)K * p.W * BM;
  const float* base = p.partial + (size_t)tile * p.split * item_stride + row;
  // Σ over splits of 8 consecutive accumulator columns of expert j starting at c
  auto sum8 = [&](int j, int c, float (&v)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
#pragma unroll 8  // the splits' loads in flight together (split <= 8)
    for (int sp = 0; sp < p.split; ++sp) {
      const float* q = base + sp * item_stride + (size_t)(j * p.W + c) * BM;
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += q[(size_t)i * BM];
    }
  };
  const int ng = p.R / 8;  // dt_low groups per expert
  const int grp = blockIdx.y;
  const bool live = row < ti.rows;  // rows past the tile's tokens: A' zeros, no B/C output
  if (grp < K * ng) {
    const int j = grp / ng, c = (grp - j * ng) * 8;
    float v[8];
    if (live) {
      sum8(j, c, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_bf16x2(g[j] * v[2 * i], g[j] * v[2 * i + 1], hw[i], lw[i]);
    uint4* arow = reinterpret_cast<uint4*>(p.aprime + ((size_t)tile * BM + row) * p.K2);
    arow[(j * p.R_pad + c) / 8] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    arow[((K + j) * p.R_pad + c) / 8] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    if (c + 8 == p.R) {  // the expert's last group also clears the padding columns
      for (int cz = p.R; cz < p.R_pad; cz += 8) {
        arow[(j * p.R_pad + cz) / 8] = make_uint4(0, 0, 0, 0);
        arow[((K + j) * p.R_pad + cz) / 8] = make_uint4(0, 0, 0, 0);
      }
    }
  } else if (live) {
    const int q = grp - K * ng;      // 0, 1: B_mix n = 0..7, 8..15; 2, 3: C_mix
    const int which = q >> 1, n0 = (q & 1) * 8;
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      float v[8];
      sum8(j, p.R + 16 * which + n0, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = fmaf(g[j], v[i], o[i]);
    }
    float4* dst = reinterpret_cast<float4*>((which == 0 ? p.B_mix : p.C_mix) + (size_t)p.slot_tok[pos] * 16 + n0);
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
}

// softplus(v) = max(v, 0) + ln 2 * log2(1 + e) with e = 2^{-|v| log2 e} in (0, 1]: two
// special-function instructions (ex2, lg2) and four others, no branch, so the 32 values of one TMEM
// load interleave freely. 1 + e rounds e to 2^-24 absolute, so softplus of a very negative v (the
// small-Δ end, Δ ~ e) carries ~1e-7 absolute error: 1e-4 relative at Δ = 1e-3, far inside what
// the scan's tolerance admits (the recurrence sees Δ through exp(Δ A) and Δ B x).
constexpr float kLn2 = 0.69314718055994531f;
__device__ __forceinline__ float softplus_fast(float v) {
  const float e = ex2_approx(-fabsf(v) * kLog2e);
  float l;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(1.0f + e));
  return fmaf(l, kLn2, fmaxf(v, 0.f));
}

template <int K>
__global__ void __launch_bounds__(576, 1)
    proj_stage2_kernel(const __grid_constant__ CUtensorMap tm_ap, const __grid_constant__ CUtensorMap tm_wdt,
                       const Stage2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nbox_ap = p.K2 / 64;
  uint8_t* ap = smem;                                // [K2/64][128 rows][128 B]
  uint8_t* ring = smem + nbox_ap * kApBox;           // [kStages2][kSlot2]
  uint8_t* bias_area = ring + kStages2 * kSlot2;     // [16 epilogue warps][kBiasW]
  uint64_t* full = reinterpret_cast<uint64_t*>(bias_area + 16 * kBiasW);
  uint64_t* empty = full + kStages2;
  uint64_t* ap_full = empty + kStages2;
  uint64_t* ap_empty = ap_full + 1;
  uint64_t* acc_full = ap_empty + 1;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(ap_full, 1);
    mbar_init(ap_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 16);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_ap);
    prefetch_tmap(&tm_wdt);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // the bucketing (or the previous stage) has completed
  const int num_tiles = *p.num_tiles;
  const int nchunks = (p.D + NC - 1) / NC;
  const long long total = (long long)num_tiles * nchunks;
  const long long item_begin = total * blockIdx.x / gridDim.x;
  const long long item_end = total * (blockIdx.x + 1) / gridDim.x;
  const int rs_steps = p.R / p.RS;

  if (warp == 0) {
    // ---------------- producer ----------------
    int stage = 0, issued = 0, cur_tile = -1;
    uint32_t phase = 0, ap_phase = 0;
    int ej[2] = {0, 0};
    bool ok = true;
    for (long long item = item_begin; item < item_end && ok; ++item) {
      const int tile = (int)(item / nchunks);
      const int c = (int)(item - (long long)tile * nchunks);
      if (tile != cur_tile) {
        if (!mbar_wait(ap_empty, ap_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(ap_full, (uint32_t)(nbox_ap * kApBox));
          for (int kb = 0; kb < nbox_ap; ++kb) tma_load_2d(ap + kb * kApBox, &tm_ap, ap_full, kb * 64, tile * BM);
        }
        ap_phase ^= 1u;
        cur_tile = tile;
        const TileInfo ti = p.tiles[tile];
        ej[0] = ti.e0;
        ej[1] = ti.e1;
      }
      for (int j = 0; j < K && ok; ++j) {
        for (int rs = 0; rs < rs_steps; ++rs) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* slot = ring + stage * kSlot2;
          if (lane == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)(4 * p.RS * 128));
          __syncwarp();
          if (lane < 4) tma_load_3d(slot + lane * p.RS * 128, &tm_wdt, &full[stage], c * NC + lane * 64, rs * p.RS, ej[j]);
          ++issued;
          if (++stage == kStages2) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 21, blockIdx.x, 0);
      drain_ring(full, kStages2, stage, phase, issued);
      if (cur_tile >= 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(ap_full, ap_phase ^ 1u) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BM, NC, /*b_mn_major=*/true);
      const uint32_t ap_base = smem_u32(ap);
      int stage = 0, cur_tile = -1, buf = 0;
      uint32_t phase = 0, ap_phase = 0;
      uint32_t acc_phase[2] = {0, 0};
      bool ok = true;
      for (long long item = item_begin; item < item_end && ok; ++item) {
        const int tile = (int)(item / nchunks);
        if (tile != cur_tile) {
          if (cur_tile >= 0) mma_commit(ap_empty);
          if (!mbar_wait(ap_full, ap_phase, abort_flag)) {
            ok = false;
            break;
          }
          ap_phase ^= 1u;
          cur_tile = tile;
        }
        if (!mbar_wait(&acc_empty[buf], acc_phase[buf] ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        acc_phase[buf] ^= 1u;
        tc_fence_after();
        bool first = true;
        for (int j = 0; j < K && ok; ++j) {
          for (int rs = 0; rs < rs_steps; ++rs) {
            if (!mbar_wait(&full[stage], phase, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sbase = smem_u32(ring + stage * kSlot2);
            for (int kk = 0; kk < p.RS / 16; ++kk) {
              const uint64_t bdesc = smem_desc(sbase + kk * 16 * 128, p.RS * 128, 1024, kLayoutSW128);
#pragma unroll
              for (int part = 0; part < 2; ++part) {  // hi, then lo
                const int kg = (part * K + j) * p.R_pad + rs * p.RS + kk * 16;  // K offset inside A'
                const uint64_t adesc =
                    smem_desc(ap_base + (kg >> 6) * kApBox + (kg & 63) * 2, 16, 1024, kLayoutSW128);
                mma_bf16(tmem + buf * NC, adesc, bdesc, idesc, first ? 0u : 1u);
                first = false;
              }
            }
            mma_commit(&empty[stage]);
            if (++stage == kStages2) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        buf ^= 1;
      }
      if (!ok) {
        *abort_flag = 1;
        record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 22, blockIdx.x, 0);
      }
      wait_all_mma(done);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: 16 warps, four per TMEM lane quarter ----------------
    // Each warp drains 64 of the chunk's 256 columns for the 32 rows of its lane quarter, as two
    // 16-row halves read with the 16x256b shape: four consecutive threads hold eight consecutive
    // columns of one row, so every warp-wide store writes whole 32-byte sectors of 8 rows. Four
    // warps per scheduler hide the latency of the softplus chains.
    const int q = warp & 3;
    const int cq = (warp - 2) >> 2;  // chunk columns [64 cq, 64 cq + 64)
    const int t0 = lane & 3, t1 = lane >> 2;
    int cur_tile = -1, buf = 0;
    uint32_t acc_phase[2] = {0, 0};
    // the 4 rows of this thread: 32q + 16dh + t1 + 8r  (dh, r in {0, 1})
    bool valid[2][2] = {{false, false}, {false, false}};
    int tok[2][2] = {{0, 0}, {0, 0}};
    float g[2][2][K];
    int e[2] = {0, 0};
    // The k experts' biases of this warp's 64 columns go through a warp-private shared-memory
    // buffer, one 16-byte load per lane per item, issued one item ahead.
    float* bias_w = reinterpret_cast<float*>(bias_area + (warp - 2) * kBiasW);
    const int bj = lane >> 4, bc4 = (lane & 15) * 4;  // lane's expert slot and first column
    // the experts of item `it` come from `known` (the current tile's) unless it starts a new tile
    auto load_bias = [&](long long it, int known_tile, const int (&known_e)[2]) -> float4 {
      const int tl = (int)(it / nchunks);
      const int cl = (int)(it - (long long)tl * nchunks);
      const int col = cl * NC + cq * 64 + bc4;
      if (bj >= K || col >= p.D) return make_float4(0.f, 0.f, 0.f, 0.f);
      int ee;
      if (tl == known_tile) {
        ee = known_e[bj];
      } else {
        const TileInfo tn = p.tiles[tl];
        ee = bj == 0 ? tn.e0 : tn.e1;
      }
      return __ldg(reinterpret_cast<const float4*>(p.b_dt + (size_t)ee * p.D + col));
    };
    float4 bq_next = item_begin < item_end ? load_bias(item_begin, -1, e) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long item = item_begin; item < item_end; ++item) {
      const int tile = (int)(item / nchunks);
      const int c = (int)(item - (long long)tile * nchunks);
      if (tile != cur_tile) {
        const TileInfo ti = p.tiles[tile];
#pragma unroll
        for (int dh = 0; dh < 2; ++dh)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int row = 32 * q + 16 * dh + t1 + 8 * r;
            valid[dh][r] = row < ti.rows;
            const int pos = ti.row_begin + min(row, ti.rows - 1);
            tok[dh][r] = p.slot_tok[pos];
#pragma unroll
            for (int j = 0; j < K; ++j) g[dh][r][j] = p.slot_gate[pos * K + j];
          }
        e[0] = ti.e0;
        e[1] = ti.e1;
        cur_tile = tile;
      }
      const int dcol = c * NC + cq * 64 + 2 * t0;  // column of r[0]; r[4k] is at dcol + 8k
      {
        const float4 bq = bq_next;
        if (item + 1 < item_end) bq_next = load_bias(item + 1, cur_tile, e);
        __syncwarp();  // the previous item's reads of bias_w are done
        if (bj < K) *reinterpret_cast<float4*>(bias_w + bj * 64 + bc4) = bq;
        __syncwarp();
      }
      if (!mbar_wait(&acc_full[buf], acc_phase[buf], abort_flag)) {
        *abort_flag = 1;
        if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 23, blockIdx.x, (int)item);
        break;
      }
      acc_phase[buf] ^= 1u;
      tc_fence_after();
#pragma unroll
      for (int dh = 0; dh < 2; ++dh) {
        uint32_t v[32];
        tmem_ld_16x256b_x8_nowait(tmem + ((uint32_t)(32 * q + 16 * dh) << 16) + buf * NC + cq * 64, v);
        tmem_wait_ld();
        if (dh == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int d = dcol + 8 * k;
          if (d < p.D) {
            // the k experts' biases of columns d, d+1
            float2 bias[K];
#pragma unroll
            for (int j = 0; j < K; ++j) bias[j] = *reinterpret_cast<const float2*>(bias_w + j * 64 + 2 * t0 + 8 * k);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              float2 bmix = make_float2(0.f, 0.f);
#pragma unroll
              for (int j = 0; j < K; ++j) {
                bmix.x = fmaf(g[dh][r][j], bias[j].x, bmix.x);
                bmix.y = fmaf(g[dh][r][j], bias[j].y, bmix.y);
              }
              if (valid[dh][r]) {
                const float a0 = __uint_as_float(v[4 * k + 2 * r]) + bmix.x;
                const float a1 = __uint_as_float(v[4 * k + 2 * r + 1]) + bmix.y;
                const float2 o = p.raw ? make_float2(a0, a1) : make_float2(softplus_fast(a0), softplus_fast(a1));
                *reinterpret_cast<float2*>(p.delta + (size_t)tok[dh][r] * p.D + d) = o;
              }
            }
          }
        }
      }
      buf ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- host side -------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
            const cuuint32_t* box, CUtensorMapSwizzle swz) {
  auto fn = get_encode();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims, strides_bytes, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// The projection over "slots" p.T x k: tokens (xshift 0), or (token, slot) pairs run with k = 1
// (xshift 1, raw 1: per-pair sums out, no softplus; see run_proj_pairs).
template <int K>
cudaError_t run_tc(const ProjParams& p, uint8_t* ws, cudaStream_t s, int xshift = 0, int raw = 0) {
  const TcLayout L = tc_layout(p.T, p.E, K, p.R, p.D);
  int* group_of = reinterpret_cast<int*>(ws + L.group_of);
  int* blockhist = reinterpret_cast<int*>(ws + L.blockhist);
  int* blockbase = reinterpret_cast<int*>(ws + L.blockbase);
  int* offsets = reinterpret_cast<int*>(ws + L.offsets);
  int* num_tiles = reinterpret_cast<int*>(ws + L.num_tiles);
  TileInfo* tiles = reinterpret_cast<TileInfo*>(ws + L.tiles);
  int* slot_tok = reinterpret_cast<int*>(ws + L.slot_tok);
  float* slot_gate = reinterpret_cast<float*>(ws + L.slot_gate);
  __nv_bfloat16* aprime = reinterpret_cast<__nv_bfloat16*>(ws + L.aprime);

  cudaError_t e;
  if (p.T <= kSmallBucketT) {
    if ((e = launch_pdl(group_bucket_small_kernel<K>, dim3(1), dim3(kSmallBucketThreads), 0, s, p.idx, p.gates, (int)p.T,
                        p.E, L.G, offsets, num_tiles, tiles, slot_tok, slot_gate)) != cudaSuccess)
      return e;
    note_launch();
  } else {
    group_count_kernel<K><<<(unsigned)L.nb, kBucketBlock, 0, s>>>(p.idx, p.T, p.E, L.G, group_of, blockhist);
    group_scan_kernel<K><<<1, 256, 0, s>>>(blockhist, L.nb, L.G, offsets, blockbase, num_tiles, tiles);
    group_scatter_kernel<K><<<(unsigned)L.nb, kBucketBlock, 0, s>>>(p.idx, p.gates, p.T, p.E, L.G, group_of,
                                                                     blockbase, slot_tok, slot_gate);
    note_launch(3);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const int W = p.R + 2 * p.N;
  const int nbw = (W + 63) / 64;
  CUtensorMap tm_wx, tm_ap, tm_wdt;
  {
    cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)p.D, (cuuint64_t)p.E};
    cuuint64_t str[2] = {(cuuint64_t)W * 2, (cuuint64_t)W * p.D * 2};
    cuuint32_t box[3] = {64, BK1, 1};
    if (!encode(&tm_wx, p.W_x, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)L.K2, (cuuint64_t)L.max_tiles * BM};
    cuuint64_t str[1] = {(cuuint64_t)L.K2 * 2};
    cuuint32_t box[2] = {64, BM};
    if (!encode(&tm_ap, aprime, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  }
  const int RS = p.R % 32 == 0 ? 32 : 16;
  {
    cuuint64_t dims[3] = {(cuuint64_t)p.D, (cuuint64_t)p.R, (cuuint64_t)p.E};
    cuuint64_t str[2] = {(cuuint64_t)p.D * 2, (cuuint64_t)p.R * p.D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)RS, 1};
    if (!encode(&tm_wdt, p.W_dt, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  }

  const int sms = num_sms();
  Stage1Params s1{p.D,     W,       p.R,    p.N,      L.R_pad, L.K2,      nbw,       L.split,
                  L.kper,  xshift,  reinterpret_cast<const __nv_bfloat16*>(p.x), reinterpret_cast<float*>(ws + L.partial),
                  num_tiles, tiles, slot_tok, slot_gate, aprime, p.B_mix, p.C_mix, ws};
  const size_t smem1 = 1024 + (size_t)kStagesA * kSlotA + (size_t)kStagesW * kSlotW + 256;
  e = cudaFuncSetAttribute(proj_stage1_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  if ((e = launch_pdl(proj_stage1_kernel<K>, dim3((unsigned)std::min(L.max_tiles * L.split, sms)), dim3(224), smem1, s,
                      tm_wx, s1)) != cudaSuccess)
    return e;
  note_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (L.split > 1) {
    if ((e = launch_pdl(stage1_finish_kernel<K>, dim3((unsigned)L.max_tiles, (unsigned)(K * p.R / 8 + 4)), dim3(128), 0,
                        s, s1)) != cudaSuccess)
      return e;
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  Stage2Params s2{p.D, p.R, L.R_pad, L.K2, RS, num_tiles, tiles, slot_tok, slot_gate, p.b_dt, p.delta, raw, ws};
  const size_t smem2 = 1024 + (size_t)(L.K2 / 64) * kApBox + (size_t)kStages2 * kSlot2 + 16 * kBiasW + 256;
  e = cudaFuncSetAttribute(proj_stage2_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
  if (e != cudaSuccess) return e;
  if ((e = launch_pdl(proj_stage2_kernel<K>, dim3((unsigned)sms), dim3(576), smem2, s, tm_ap, tm_wdt, s2)) != cudaSuccess)
    return e;
  note_launch();
  return cudaGetLastError();
}

// ---- few tokens, k = 2: the (token, slot) pairs bucketed by single expert ----------------------------
// Bucketing tokens by expert PAIR leaves a decode step's 256 tokens spread over up to E(E-1)/2
// groups of a few rows, each tile reading two experts' tables. For few tokens the projection runs
// instead on the T k (token, slot) pairs v = k t + j as k = 1 slots (their expert idx[t][j], gate
// g[t][j], x row t): every expert's tables are read by about (T k / 128 + 1) tiles, and the tiles
// are fuller. The per-pair results -- g_j (dt_low_j W_dt^{e_j} + b_dt^{e_j}), g_j B^j, g_j C^j --
// are summed per token in slot order by pair_combine_kernel, which also takes the softplus.
constexpr int64_t kPairMaxT = 1024;  // tokens up to which k = 2 runs on expanded pairs

struct PairLayout {
  TcLayout inner;
  size_t raw, bv, cv, total;
};

PairLayout pair_layout(int64_t T, int E, int R, int D) {
  PairLayout L{};
  L.inner = tc_layout(2 * T, E, 1, R, D);
  size_t o = L.inner.total;
  L.raw = o; o = align_up(o + 4 * (size_t)2 * T * D, 256);
  L.bv = o; o = align_up(o + 4 * (size_t)2 * T * 16, 256);
  L.cv = o; o = align_up(o + 4 * (size_t)2 * T * 16, 256);
  L.total = o;
  return L;
}

__global__ void __launch_bounds__(256) pair_combine_kernel(const float* raw, const float* bv, const float* cv,
                                                           int64_t T, int D, float* delta, float* B_mix,
                                                           float* C_mix) {
  pdl_trigger();
  pdl_wait();
  const int64_t nd = T * (D / 4), total = nd + T * 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    if (i < nd) {
      const int64_t t = i / (D / 4);
      const int c4 = (int)(i - t * (D / 4));
      const float4 a = reinterpret_cast<const float4*>(raw + (size_t)(2 * t) * D)[c4];
      const float4 b = reinterpret_cast<const float4*>(raw + (size_t)(2 * t + 1) * D)[c4];
      reinterpret_cast<float4*>(delta + (size_t)t * D)[c4] =
          make_float4(softplus_fast(a.x + b.x), softplus_fast(a.y + b.y), softplus_fast(a.z + b.z),
                      softplus_fast(a.w + b.w));
    } else {
      const int64_t r = i - nd, t = r / 8;
      const int q = (int)(r - t * 8);  // 0..3: B_mix float4 q; 4..7: C_mix float4 q - 4
      const float* src = q < 4 ? bv : cv;
      const float4 a = reinterpret_cast<const float4*>(src + (size_t)(2 * t) * 16)[q & 3];
      const float4 b = reinterpret_cast<const float4*>(src + (size_t)(2 * t + 1) * 16)[q & 3];
      reinterpret_cast<float4*>((q < 4 ? B_mix : C_mix) + (size_t)t * 16)[q & 3] =
          make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
    }
  }
}

cudaError_t run_proj_pairs(const ProjParams& p, uint8_t* ws, cudaStream_t s) {
  const PairLayout L = pair_layout(p.T, p.E, p.R, p.D);
  ProjParams q = p;
  q.T = 2 * p.T;  // idx and gates [T, 2] are the pairs' [2T, 1]
  q.k = 1;
  q.delta = reinterpret_cast<float*>(ws + L.raw);
  q.B_mix = reinterpret_cast<float*>(ws + L.bv);
  q.C_mix = reinterpret_cast<float*>(ws + L.cv);
  cudaError_t e = run_tc<1>(q, ws, s, 1, 1);
  if (e != cudaSuccess) return e;
  const int64_t total = p.T * (p.D / 4 + 8);  // one item per thread: a single round of loads
  const unsigned grid = (unsigned)std::min<int64_t>((total + 255) / 256, 1 << 20);
  if ((e = launch_pdl(pair_combine_kernel, dim3(grid), dim3(256), 0, s, q.delta, q.B_mix, q.C_mix, p.T, p.D, p.delta,
                      p.B_mix, p.C_mix)) != cudaSuccess)
    return e;
  note_launch();
  return cudaGetLastError();
}

bool use_pairs(int64_t T, int k) { return k == 2 && T <= kPairMaxT; }

}  // namespace

// The tensor-core path covers bf16 activations and tables, k <= 2, N = 16, R a multiple of 16 with
// R <= 64 or R in {128}, R + 2N <= 192 (<= 256 for k = 1), and D a multiple of 64.
bool proj_tc_supported(const ProjParams& p, bool io_bf16, bool w_bf16) {
  const int W = p.R + 2 * p.N;
  if (!io_bf16 || !w_bf16) return false;
  if (p.k < 1 || p.k > 2 || p.N != 16) return false;
  if (p.R % 16 != 0 || !(p.R <= 64 || p.R == 128)) return false;
  if (W % 16 != 0 || W > (p.k == 2 ? 192 : 256)) return false;
  if (p.D % 64 != 0 || p.T < 1 || p.T > (int64_t(1) << 30)) return false;
  return true;
}

size_t proj_tc_workspace(int64_t T, int E, int k, int R, int D) {
  return use_pairs(T, k) ? pair_layout(T, E, R, D).total : tc_layout(T, E, k, R, D).total;
}

cudaError_t run_proj_tc(const ProjParams& p, void* ws, cudaStream_t s) {
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  if (use_pairs(p.T, p.k)) return run_proj_pairs(p, w, s);
  return p.k == 1 ? run_tc<1>(p, w, s) : run_tc<2>(p, w, s);
}

}  // namespace swimba
