// The surrounding block's two dense projections on the tcgen05 tensor cores.
//
// Source: "Mamba y las SSMs: el retorno del estado persistente", section "Mamba" (Figura 3: a linear
// projection makes the SSM branch and the gate branch, a linear projection maps the gated output
// back) and "Estado interno puramente lineal" (the output projection is followed by a residual
// connection).
//
//   in-projection:   [x_pre | z] = u W_in        (the epilogue splits the columns into the x_pre
//                                                 and z buffers)
//   out-projection:  o = y W_out + u             (the residual is added in the epilogue)
//
// C[M, N] = A[M, K] B[K, N] (+ R[M, N]), bf16 operands as stored, fp32 accumulation in tensor
// memory, bf16 or fp32 out. A is stored either [M, K] (K contiguous, "K-major") or [K, M] (M
// contiguous: the transpose of a stored matrix, as the weight gradients x^T dV need); B is stored
// either [K, N] (N contiguous) or [N, K] (K contiguous: a stored weight used transposed, as the
// input gradients dV W^T need). Persistent, warp-specialised: warp 0 streams the A tile [128 x 64]
// and the B tile [64 x 256] of each k-step by TMA (128-byte swizzle; MN-major operands as 64-wide
// boxes) through a 4-stage ring; warp 1 issues tcgen05.mma M=128, N=256, K=16 into one of two
// 256-column TMEM accumulators; warps 2-5 drain the other accumulator (one TMEM lane = one output
// row) while the next tile accumulates. Tiles go in groups of 16 row tiles (see tile_origin), so
// the CTAs working at one time share both their A rows and their B columns in L2. Every wait is bounded: a wait that runs out records
// SWIMBA_ERR_TIMEOUT in the status block, the CTA lets its copies land, frees TMEM and exits. fp32
// operands take a SIMT kernel (tiles of 64 x 64 in shared memory).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace swimba {

using namespace sm100;

namespace {

constexpr int GBM = 128, GBN = 256, GBK = 64;
constexpr int kGStages = 4;
constexpr int kGA = GBM * GBK * 2;   // 16 KB
constexpr int kGB = GBK * GBN * 2;   // 32 KB: four 64-column boxes of 8 KB
constexpr int kGStage = kGA + kGB;

__device__ __forceinline__ uint32_t bf16pair(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct GemmParams {
  void* C0;           // columns [0, split) of the output
  void* C1;           // columns [split, N) (split == N: unused)
  const void* R;      // residual [M, N] or null
  void* status;
  int M, N, K, split, ldc0, ldc1, ldr;
  const int* rows;    // fp32 output only: output (and residual) row of row m = rows[m] / rows_div, or null
  int rows_div;
};

}  // namespace

// Tile order: groups of kGroupM row tiles; inside a group the column tiles advance while the
// row tiles cycle fastest. The CTAs working at one time then cover ~16 row blocks of A and ~9
// column blocks of B, both of which stay in L2 while the group sweeps the columns, so A is read
// from HBM about once (a plain row-fastest order re-read all of A for every column tile: 3.1 GB
// of DRAM reads for the Mamba-1.4B-like block's in-projection, whose operands are 168 MB).
constexpr int kGroupM = 16;
__device__ __forceinline__ void tile_origin(int tile, int mt, int nt, int& m0, int& n0) {
  const int group = tile / (kGroupM * nt);
  const int first = group * kGroupM;
  const int gm = min(mt - first, kGroupM);
  const int r = tile - group * kGroupM * nt;
  m0 = (first + r % gm) * GBM;
  n0 = (r / gm) * GBN;
}

template <bool A_MN, bool B_K, bool F32OUT>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStage);
  uint64_t* empty = full + kGStages;
  uint64_t* acc_full = empty + kGStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* done = acc_empty + 2;          // every MMA of the CTA has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int mt = (p.M + GBM - 1) / GBM, nt = (p.N + GBN - 1) / GBN, kt = (p.K + GBK - 1) / GBK;
  const int tiles = mt * nt;

  if (warp == 0) {
    // ---------------- producer ----------------
    int stage = 0, issued = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
      int m0, n0;
      tile_origin(tile, mt, nt, m0, n0);
      for (int k = 0; k < kt; ++k) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + stage * kGStage;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], (uint32_t)kGStage);
          if (A_MN) {  // two 64-column boxes of the stored [K, M]
            tma_load_2d(st, &tm_a, &full[stage], m0, k * GBK);
            tma_load_2d(st + 8192, &tm_a, &full[stage], m0 + 64, k * GBK);
          } else {
            tma_load_2d(st, &tm_a, &full[stage], k * GBK, m0);
          }
          if (B_K) {  // one box of 256 rows of the stored [N, K]
            tma_load_2d(st + kGA, &tm_b, &full[stage], k * GBK, n0);
          } else {
            for (int i = 0; i < 4; ++i) tma_load_2d(st + kGA + i * 8192, &tm_b, &full[stage], n0 + 64 * i, k * GBK);
          }
        }
        __syncwarp();
        ++issued;
        if (++stage == kGStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 61, blockIdx.x, 0);
      // the copies of the last min(issued, stages) stages may still be landing
      for (int i = 0; i < (issued < kGStages ? issued : kGStages); ++i) {
        if (--stage < 0) {
          stage = kGStages - 1;
          phase ^= 1u;
        }
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[stage], phase) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(GBM, GBN, /*b_mn_major=*/!B_K, /*a_mn_major=*/A_MN);
      const uint32_t base = smem_u32(smem);
      int stage = 0, buf = 0;
      uint32_t phase = 0;
      uint32_t acc_phase[2] = {0, 0};
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&acc_empty[buf], acc_phase[buf] ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        acc_phase[buf] ^= 1u;
        tc_fence_after();
        for (int k = 0; k < kt; ++k) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + stage * kGStage, sb = sa + kGA;
#pragma unroll
          for (int kk = 0; kk < GBK / 16; ++kk) {
            const uint64_t adesc = A_MN ? smem_desc(sa + kk * 16 * 128, 8192, 1024, kLayoutSW128)
                                        : smem_desc(sa + kk * 32, 16, 1024, kLayoutSW128);
            const uint64_t bdesc = B_K ? smem_desc(sb + kk * 32, 16, 1024, kLayoutSW128)
                                       : smem_desc(sb + kk * 16 * 128, 8192, 1024, kLayoutSW128);
            mma_bf16(tmem + buf * GBN, adesc, bdesc, idesc, (k | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == kGStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        buf ^= 1;
      }
      if (!ok) {
        *abort_flag = 1;
        record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 62, blockIdx.x, 0);
      }
      // every MMA this thread issued has completed when `done` completes its first phase
      mma_commit(done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(done, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lane quarter = warp % 4 ----------------
    const int q = warp & 3;
    int buf = 0;
    uint32_t acc_phase[2] = {0, 0};
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
      int m0, n0;
      tile_origin(tile, mt, nt, m0, n0);
      if (!mbar_wait(&acc_full[buf], acc_phase[buf], abort_flag)) {
        *abort_flag = 1;
        if (lane == 0) record_device_error(p.status, SWIMBA_ERR_TIMEOUT, 63, blockIdx.x, tile);
        break;
      }
      acc_phase[buf] ^= 1u;
      tc_fence_after();
      // One TMEM lane = one output row: each thread writes its row's 32-column slices as 16-byte
      // (bf16) or 2 x 16-byte (fp32) stores. (Staging the 32 x 32 blocks through shared memory so
      // that a warp instruction covers one row was timed slower: 987 against 500 µs for the
      // out-projection with its residual, 9.8 against 2.8 ms for the projection backward.)
      const int m = m0 + 32 * q + lane;
      const int mo = (F32OUT && p.rows != nullptr && m < p.M) ? p.rows[m] / p.rows_div : m;
      // The residual's 32 values of a slice are loaded one slice ahead, before the current slice is
      // stored: the residual may be the output itself (an in-place accumulation), so the compiler
      // may not move a load above an earlier store, and loads interleaved with the stores made one
      // memory round trip per 8 columns.
      auto load_r = [&](int cb, float (&r)[32]) {
        const int n = n0 + cb * 32;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          const int col = n + j;
          if (p.R != nullptr && m < p.M && col < p.N) {
            if (F32OUT) {
              const float4* r4 =
                  reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.R) + (size_t)mo * p.ldr + col);
              const float4 r0 = r4[0], r1 = r4[1];
              r[j] = r0.x;
              r[j + 1] = r0.y;
              r[j + 2] = r0.z;
              r[j + 3] = r0.w;
              r[j + 4] = r1.x;
              r[j + 5] = r1.y;
              r[j + 6] = r1.z;
              r[j + 7] = r1.w;
            } else {
              const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.R) +
                                                              (size_t)m * p.ldr + col);
              r[j] = bf16lo(w.x);
              r[j + 1] = bf16hi(w.x);
              r[j + 2] = bf16lo(w.y);
              r[j + 3] = bf16hi(w.y);
              r[j + 4] = bf16lo(w.z);
              r[j + 5] = bf16hi(w.z);
              r[j + 6] = bf16lo(w.w);
              r[j + 7] = bf16hi(w.w);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) r[j + e] = 0.f;
          }
        }
      };
      float rr[32], rn[32];
      load_r(0, rr);
#pragma unroll
      for (int cb = 0; cb < GBN / 32; ++cb) {
        if (cb + 1 < GBN / 32) load_r(cb + 1, rn);
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + buf * GBN + cb * 32, v);
        const int n = n0 + cb * 32;
        if (m < p.M && n < p.N) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {  // groups of 8 columns (N and split are multiples of 8)
            const int col = n + j;
            if (col < p.N && F32OUT) {
              float o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = p.R != nullptr ? v[j + e] + rr[j + e] : v[j + e];
              float* out = col < p.split ? reinterpret_cast<float*>(p.C0) + (size_t)mo * p.ldc0 + col
                                         : reinterpret_cast<float*>(p.C1) + (size_t)mo * p.ldc1 + (col - p.split);
              reinterpret_cast<float4*>(out)[0] = make_float4(o[0], o[1], o[2], o[3]);
              reinterpret_cast<float4*>(out)[1] = make_float4(o[4], o[5], o[6], o[7]);
            } else if (col < p.N) {
              float o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = p.R != nullptr ? v[j + e] + rr[j + e] : v[j + e];
              __nv_bfloat16* out = col < p.split
                                       ? reinterpret_cast<__nv_bfloat16*>(p.C0) + (size_t)m * p.ldc0 + col
                                       : reinterpret_cast<__nv_bfloat16*>(p.C1) + (size_t)m * p.ldc1 + (col - p.split);
              *reinterpret_cast<uint4*>(out) = make_uint4(bf16pair(o[0], o[1]), bf16pair(o[2], o[3]),
                                                          bf16pair(o[4], o[5]), bf16pair(o[6], o[7]));
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) rr[e] = rn[e];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      buf ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// fp32 operands: C[M, N] = A B (+ R), 64 x 64 tiles, 256 threads with 4 x 4 outputs each.
__global__ void __launch_bounds__(256) gemm_simt_f32_kernel(const float* A, int lda, const float* B, int ldb,
                                                            float* C0, int ldc0, float* C1, int ldc1, int split,
                                                            const float* R, int ldr, int M, int N, int K) {
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64 + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i / 64, c = i % 64;
      As[kk][c] = (m0 + c < M && k0 + kk < K) ? A[(size_t)(m0 + c) * lda + k0 + kk] : 0.f;
      Bs[kk][c] = (n0 + c < N && k0 + kk < K) ? B[(size_t)(k0 + kk) * ldb + n0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(As[kk][ty + 16 * i], Bs[kk][tx + 16 * j], acc[i][j]);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < M && n < N) {
        const float v = acc[i][j] + (R != nullptr ? R[(size_t)m * ldr + n] : 0.f);
        if (n < split) C0[(size_t)m * ldc0 + n] = v;
        else C1[(size_t)m * ldc1 + n - split] = v;
      }
    }
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn() {
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

// 2-D bf16 map over a row-major [rows, cols] matrix with row stride ld (elements), box {64, box_rows}.
bool gemm_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  auto fn = gemm_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t str[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, str, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

template <bool A_MN, bool B_K, bool F32OUT>
cudaError_t launch_gemm_tc(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = ((p.M + GBM - 1) / GBM) * ((p.N + GBN - 1) / GBN);
  const size_t smem = 1024 + (size_t)kGStages * kGStage + 256;  // ring, then barriers and the TMEM slot
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<A_MN, B_K, F32OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<A_MN, B_K, F32OUT><<<(unsigned)std::min(tiles, sms), 192, smem, s>>>(ta, tb, p);
  note_launch();
  return cudaGetLastError();
}

// The tensor-core GEMM in its four operand layouts: A stored [M, K] (a_t = false, row stride lda)
// or [K, M] (a_t = true); B stored [K, N] (b_t = false, row stride ldb) or [N, K] (b_t = true).
// bf16 operands; out (C0 below column `split`, C1 from it) and the optional residual R are bf16 or,
// with f32_out, fp32. Row strides must be multiples of 8 elements (bf16) and pointers 16-byte aligned.
// With `rows` (fp32 out only), output row m goes to row rows[m] / rows_div of C0/C1/R: a scatter
// (rows must be distinct within one call).
cudaError_t run_gemm_tc(bool a_t, bool b_t, bool f32_out, int M, int N, int K, const void* A, int lda, const void* B,
                        int ldb, void* C0, int ldc0, void* C1, int ldc1, int split, const void* R, int ldr,
                        void* status, cudaStream_t s, const int* rows, int rows_div) {
  CUtensorMap ta, tb;
  const bool ok_a = a_t ? gemm_map(&ta, A, K, M, lda, GBK) : gemm_map(&ta, A, M, K, lda, GBM);
  const bool ok_b = b_t ? gemm_map(&tb, B, N, K, ldb, GBN) : gemm_map(&tb, B, K, N, ldb, GBK);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;
  if (rows != nullptr && !f32_out) return cudaErrorInvalidValue;
  GemmParams p{C0, C1, R, status, M, N, K, split, ldc0, ldc1, ldr, rows, rows_div > 0 ? rows_div : 1};
  const int sel = (a_t ? 4 : 0) | (b_t ? 2 : 0) | (f32_out ? 1 : 0);
  switch (sel) {
    case 0: return launch_gemm_tc<false, false, false>(ta, tb, p, s);
    case 1: return launch_gemm_tc<false, false, true>(ta, tb, p, s);
    case 2: return launch_gemm_tc<false, true, false>(ta, tb, p, s);
    case 3: return launch_gemm_tc<false, true, true>(ta, tb, p, s);
    case 4: return launch_gemm_tc<true, false, false>(ta, tb, p, s);
    case 5: return launch_gemm_tc<true, false, true>(ta, tb, p, s);
    case 6: return launch_gemm_tc<true, true, false>(ta, tb, p, s);
    default: return launch_gemm_tc<true, true, true>(ta, tb, p, s);
  }
}

// C[M, N] = A[M, K] (row stride lda) B[K, N] (row stride ldb) (+ R, row stride ldr): columns below
// `split` go to C0 (row stride ldc0), the others to C1 (ldc1). bf16 needs every row stride and
// split a multiple of 8 elements and 16-byte aligned pointers.
cudaError_t run_block_gemm(bool bf16, int M, int N, int K, const void* A, int lda, const void* B, int ldb, void* C0,
                           int ldc0, void* C1, int ldc1, int split, const void* R, int ldr, void* status,
                           cudaStream_t s) {
  if (!bf16) {
    dim3 grid((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64));
    gemm_simt_f32_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(A), lda, static_cast<const float*>(B), ldb,
                                              static_cast<float*>(C0), ldc0, static_cast<float*>(C1), ldc1, split,
                                              static_cast<const float*>(R), ldr, M, N, K);
    note_launch();
    return cudaGetLastError();
  }
  return run_gemm_tc(false, false, false, M, N, K, A, lda, B, ldb, C0, ldc0, C1, ldc1, split, R, ldr, status, s,
                     nullptr, 1);
}

}  // namespace swimba
