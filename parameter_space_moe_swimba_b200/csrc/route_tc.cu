// Router on the tensor cores: logits = x W_r with fp32 accumulation, then top-k and softmax.
//
// Source: "Swimba: Switch Mamba Model Scales State Space Models", §2 "Arquitectura de Swimba"
// (es) / "Kernmechanisme van Swimba" (nl): a router gives each token mixing weights π_t over the
// active experts.
//
// The router is a [T x D] x [D x E] product with E <= 16: almost no arithmetic per byte of x, so
// the kernel's job is to stream x from HBM once at full bandwidth. Tiles of 128 consecutive tokens
// x 64 channels arrive by TMA (128-byte swizzle) into a 4-stage ring (two CTAs per SM); one thread
// issues tcgen05.mma (M = 128, N = 3E rounded up to 16, K = 16) into a double-buffered TMEM
// accumulator, so the dot products cost the SM's issue slots nothing.
//
// W_r stays fp32-exact: every weight is split into three bf16 parts w = w1 + w2 + w3 (each part is
// the bf16 rounding of what the previous ones leave; three 8-bit significands cover fp32's 24);
// B column 3e + q holds part q of expert e, and the epilogue adds the three fp32 partial logits.
// Products of bf16 x and a bf16 part are exact in fp32, so the logits are the fp32-accumulated
// x W_r up to summation order. The TMA brings each K slice's 64 rows of W_r (fp32) with the x tile;
// two warps split them into the B slice in shared memory (K-major, 128-byte swizzle); four
// epilogue warps (one TMEM lane = one token each) read the partial logits and run the same top-k /
// softmax as the SIMT router.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "route.cuh"
#include "sm100.cuh"

namespace swimba {

using namespace sm100;

namespace {

constexpr int RBM = 128;            // tokens per tile
constexpr int RBK = 64;             // channels per K slice (128 bytes of bf16)
constexpr int kRStages = 4;         // ring depth (two CTAs per SM: 8 stages of x per SM)
constexpr int kXSlot = RBM * RBK * 2;  // 16 KB
constexpr int kBSlot = 6144;           // 48 B rows of 128 bytes (3E <= 48)
constexpr int kWSlot = RBK * 16 * 4;   // the slice's W_r rows, fp32 [64][E <= 16]
constexpr int kAccCols = 64;           // TMEM columns per accumulator buffer

struct RouteTcParams {
  const float* W_r;  // [D, E]
  int32_t* idx;      // [T, k]
  float* gates;      // [T, k]
  int64_t T;
  int D, E, k, npad;
};

// After a failed wait: let the TMA copies in flight land before the CTA exits (bounded).
__device__ void drain_x_ring(uint64_t* full, int stage, uint32_t phase, int issued) {
  for (int i = 0; i < min(issued, kRStages); ++i) {
    int s = stage - 1 - i;
    uint32_t ph = phase;
    if (s < 0) {
      s += kRStages;
      ph ^= 1u;
    }
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&full[s], ph) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
  }
}

// Let every MMA this thread issued finish (bounded) before TMEM is released.
__device__ __forceinline__ void wait_all_mma_done(uint64_t* done) {
  mma_commit(done);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(done, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
  }
}

template <int EP>
__global__ void __launch_bounds__(256, 2) route_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                                                          const RouteTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring = smem;
  uint8_t* bring = smem + kRStages * kXSlot;
  uint8_t* wring = bring + kRStages * kBSlot;
  uint64_t* full_x = reinterpret_cast<uint64_t*>(wring + kRStages * kWSlot);
  uint64_t* full_w = full_x + kRStages;
  uint64_t* full_b = full_w + kRStages;
  uint64_t* empty = full_b + kRStages;
  uint64_t* acc_full = empty + kRStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&full_x[s], 1);
      mbar_init(&full_w[s], 1);
      mbar_init(&full_b[s], 64);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
  }
  // B rows past 3E stay zero for the whole kernel
  for (int i = threadIdx.x; i < kRStages * kBSlot / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(bring)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = (int)((p.T + RBM - 1) / RBM);
  const int ksteps = p.D / RBK;

  if (warp == 0) {
    // ---------------- producer: x tiles by TMA ----------------
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          // W_r rows first (L2-resident, they gate the B conversion), then the x tile
          mbar_arrive_expect_tx(&full_w[stage], (uint32_t)(RBK * p.E * 4));
          tma_load_2d(wring + stage * kWSlot, &tm_w, &full_w[stage], 0, ks * RBK);
          mbar_arrive_expect_tx(&full_x[stage], (uint32_t)kXSlot);
          tma_load_2d(xring + stage * kXSlot, &tm_x, &full_x[stage], ks * RBK, tile * RBM);
          ++issued;
          if (++stage == kRStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        drain_x_ring(full_w, stage, phase, issued);
        drain_x_ring(full_x, stage, phase, issued);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(RBM, p.npad, /*b_mn_major=*/false);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t uses[2] = {0u, 0u};
      int buf = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&acc_empty[buf], (uses[buf] & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < ksteps; ++ks) {
          if (!mbar_wait(&full_x[stage], phase, abort_flag) || !mbar_wait(&full_b[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(xring + stage * kXSlot);
          const uint32_t b_base = smem_u32(bring + stage * kBSlot);
#pragma unroll
          for (int kk = 0; kk < RBK / 16; ++kk) {
            const uint64_t adesc = smem_desc(a_base + kk * 32, 16, 1024, kLayoutSW128);
            const uint64_t bdesc = smem_desc(b_base + kk * 32, 16, 1024, kLayoutSW128);
            mma_bf16(tmem + (uint32_t)(buf * kAccCols), adesc, bdesc, idesc, (ks | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == kRStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
        ++uses[buf];
        buf ^= 1;
      }
      if (!ok) *abort_flag = 1;
      wait_all_mma_done(done);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ---------------- B slices: W_r rows split into three bf16 parts ----------------
    // thread (rp, eh): K rows 2rp, 2rp+1 of the slice, experts eh*E/2 .. eh*E/2 + E/2 - 1; the two
    // rows' parts are packed as bf16x2, one 4-byte store per (expert, part)
    const int ct = threadIdx.x - 64;
    const int rp = ct & 31, eh = ct >> 5;
    const int eh0 = eh * (p.E / 2);
    const uint32_t cin = (uint32_t)(rp & 3) * 4u;
    const uint32_t chunk = (uint32_t)(rp >> 2);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      for (int ks = 0; ks < ksteps; ++ks) {
        // the slot is free (empty) and this slice's W_r rows have landed (full_w)
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag) || !mbar_wait(&full_w[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        const float* w0 = reinterpret_cast<const float*>(wring + stage * kWSlot) + (2 * rp) * p.E + eh0;
        const float* w1 = w0 + p.E;
        uint8_t* bt = bring + stage * kBSlot;
#pragma unroll
        for (int i = 0; i < EP / 2; i += 2) {
          if (i < p.E / 2) {
            const float2 a = *reinterpret_cast<const float2*>(w0 + i);  // row 2rp: experts eh0+i, +1
            const float2 b = *reinterpret_cast<const float2*>(w1 + i);  // row 2rp+1
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float2 w = u == 0 ? make_float2(a.x, b.x) : make_float2(a.y, b.y);  // (row 2rp, 2rp+1)
              const __nv_bfloat162 h1 = __float22bfloat162_rn(w);
              const float2 h1f = __bfloat1622float2(h1);
              const float2 r1 = __fadd2_rn(w, make_float2(-h1f.x, -h1f.y));
              const __nv_bfloat162 h2 = __float22bfloat162_rn(r1);
              const float2 h2f = __bfloat1622float2(h2);
              const __nv_bfloat162 h3 = __float22bfloat162_rn(__fadd2_rn(r1, make_float2(-h2f.x, -h2f.y)));
              const __nv_bfloat162 part[3] = {h1, h2, h3};
              const int e = eh0 + i + u;
#pragma unroll
              for (int q = 0; q < 3; ++q) {
                const uint32_t n = (uint32_t)(3 * e + q);
                *reinterpret_cast<__nv_bfloat162*>(bt + n * 128u + ((chunk ^ (n & 7u)) << 4) + cin) = part[q];
              }
            }
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&full_b[stage]);
        if (++stage == kRStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) *abort_flag = 1;
  } else {
    // ---------------- epilogue: one TMEM lane (= token) per thread ----------------
    const int q = warp & 3;
    const int row = 32 * q + lane;
    uint32_t uses[2] = {0u, 0u};
    int buf = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      const int64_t t = (int64_t)tile * RBM + row;
      if (ok && !mbar_wait(&acc_full[buf], uses[buf] & 1u, abort_flag)) {
        ok = false;
        *abort_flag = 1;
      }
      if (!ok) {
        // gave up: mark this CTA's remaining tokens as unrouted (idx -1, gate 0)
        if (t < p.T)
          for (int j = 0; j < p.k; ++j) {
            p.idx[t * p.k + j] = -1;
            p.gates[t * p.k + j] = 0.f;
          }
        continue;
      }
      tc_fence_after();
      float v[48];
#pragma unroll
      for (int i = 0; i < 48; ++i) v[i] = 0.f;
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * kAccCols);
      tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(v));
      if (p.npad > 16) tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(v + 16));
      if (p.npad > 32) tmem_ld16(ta + 32, *reinterpret_cast<float(*)[16]>(v + 32));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      ++uses[buf];
      buf ^= 1;
      if (t < p.T) {
        float l[EP];
#pragma unroll
        for (int e = 0; e < EP; ++e) l[e] = (v[3 * e] + v[3 * e + 1]) + v[3 * e + 2];
        select_topk<EP>(l, p.E, p.k, p.idx + t * p.k, p.gates + t * p.k);
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 route_encode_fn() {
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

template <int EP>
cudaError_t launch_route_tc(const RouteParams& rp, const CUtensorMap& tm, const CUtensorMap& tw, cudaStream_t s) {
  RouteTcParams p{rp.W_r, rp.idx, rp.gates, rp.T, rp.D, rp.E, rp.k, ((3 * rp.E + 15) / 16) * 16};
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = (int)((rp.T + RBM - 1) / RBM);
  const size_t smem = 1024 + (size_t)kRStages * (kXSlot + kBSlot + kWSlot) + 512;  // + barriers
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel<EP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // two CTAs per SM: two independent tile streams per SM (and every tile in the first wave when
  // T <= 296 x 128)
  route_tc_kernel<EP><<<(unsigned)std::min(ntiles, 2 * sms), 256, smem, s>>>(tm, tw, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

// E a multiple of 4: a TMA row of W_r (E fp32) must be a multiple of 16 bytes.
bool route_tc_supported(bool io_bf16, int D, int E, int k) {
  return io_bf16 && D >= RBK && D % RBK == 0 && E >= 4 && E <= 16 && E % 4 == 0 && k >= 1 && k <= E;
}

cudaError_t run_route_tc(const RouteParams& p, cudaStream_t s) {
  if (p.T <= 0) return cudaSuccess;
  auto fn = route_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)p.D, (cuuint64_t)p.T};
  cuuint64_t str[1] = {(cuuint64_t)p.D * 2};
  cuuint32_t box[2] = {(cuuint32_t)RBK, (cuuint32_t)RBM};
  cuuint32_t es[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p.x), dims, str, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // W_r [D, E] fp32 as a 2-D map of E-wide rows; one box = the K slice's 64 rows
  CUtensorMap tw;
  cuuint64_t wdims[2] = {(cuuint64_t)p.E, (cuuint64_t)p.D};
  cuuint64_t wstr[1] = {(cuuint64_t)p.E * 4};
  cuuint32_t wbox[2] = {(cuuint32_t)p.E, (cuuint32_t)RBK};
  if (fn(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p.W_r), wdims, wstr, wbox, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (p.E <= 4) return launch_route_tc<4>(p, tm, tw, s);
  if (p.E <= 8) return launch_route_tc<8>(p, tm, tw, s);
  return launch_route_tc<16>(p, tm, tw, s);
}

}  // namespace swimba
