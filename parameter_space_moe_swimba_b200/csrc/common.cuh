// Shared device helpers of libswimba (sm_100a). No step of the layer lives here: only dtype
// conversion, the exp2 instruction wrapper and the device status block.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "swimba.h"

namespace swimba {

// The first bytes of every workspace: device-side error reporting (bounded waits that gave up).
constexpr size_t kStatusBytes = 256;
struct DeviceStatus {
  int code;   // 0 or a swimba_status
  int where;  // kernel-specific location code of the first error
  int info0;  // kernel-specific detail (e.g. CTA index)
  int info1;
};

__device__ __forceinline__ void record_device_error(void* ws, int code, int where, int info0, int info1) {
  if (ws == nullptr) return;
  DeviceStatus* s = reinterpret_cast<DeviceStatus*>(ws);
  if (atomicCAS(&s->code, 0, code) == 0) {
    s->where = where;
    s->info0 = info0;
    s->info1 = info1;
  }
}

// Counts every kernel launch of the library (read through swimba_kernel_launches).
void note_launch(int n = 1);

// ---- programmatic dependent launch ---------------------------------------------------------------
// The kernels of a chain (a decode step: router, bucketing, the projection's stages, the state
// step) are launched with programmatic stream serialisation: a kernel may be scheduled while its
// predecessor in the stream still runs, does its set-up (barriers, tensor memory, weight rows) and
// then waits in pdl_wait() -- a hardware dependency, not a spin -- until the predecessor grid has
// completed and its writes are visible. Nothing before pdl_wait() reads what an earlier kernel of
// the stream writes or writes what it reads. pdl_trigger() lets the successor be scheduled early.
// Launched without the attribute (or after a host-side dependency) both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr float kLog2e = 1.4426950408889634f;  // log2(e)

// 2^x with the MUFU ex2 instruction (flush-to-zero; relative error about 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The zero-order-hold injection relative to the Euler one ("Mamba y las SSMs", "Mamba":
// B-bar = A^-1 (exp(Δ A) - I) B): with w = Δ A_t (natural units; arg2 = w log2 e as the scan
// kernels hold it) and a = 2^arg2 = e^w, the injection is φ Δ B x with φ = (a - 1) / w. Near w = 0
// the quotient cancels, so there φ = 1 + w/2 + w²/6 (truncation error below 2e-8 for |w| < 1e-2).
__device__ __forceinline__ float zoh_phi(float arg2, float a) {
  const float w = arg2 * 0.6931471805599453f;
  if (fabsf(w) < 1e-2f) return fmaf(fmaf(w, 1.f / 6.f, 0.5f), w, 1.f);
  return __fdividef(a - 1.f, w);
}

// ---- io dtype access -----------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f32(float& dst, float v) { dst = v; }
__device__ __forceinline__ void from_f32(__nv_bfloat16& dst, float v) { dst = __float2bfloat16_rn(v); }

// Low / high bf16 of a packed 32-bit word, widened exactly.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Unpack 16 bytes of io values into floats: 8 bf16 or 4 fp32.
template <typename IO>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
  }
};
template <>
struct Vec16<float> {
  static constexpr int n = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
};

}  // namespace swimba
