// Shared device helpers: storage-type conversion, 16-byte vector access,
// warp/block reductions, RoPE angles and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

namespace csahca {

// Error codes ORed into g_device_error by a bounded wait that gave up.
enum : int32_t {
  DEVERR_MBAR_TIMEOUT = 1,     // an mbarrier wait exceeded its iteration limit
  DEVERR_BAD_INDEX = 2,        // a selection index outside [0, N) was skipped
};

__device__ int32_t g_device_error;

__device__ __forceinline__ void raise_device_error(int32_t code) {
  atomicOr(&g_device_error, code);
}

// ---- storage types --------------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Elements of T per 16-byte vector.
template <typename T> struct Vec16 { static constexpr int N = 16 / sizeof(T); };

__device__ __forceinline__ void load16(const float* p, float* o) {
  float4 v = __ldg(reinterpret_cast<const float4*>(p));
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float* o) {
  uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    o[2 * i] = f.x; o[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store16(float* p, const float* o) {
  *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float* o) {
  uint4 v;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = v;
}

// e4m3 ("fn") byte -> float, through the CUDA fp8 conversion intrinsic.
__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(__half(h));
}

// ---- reductions -------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---- RoPE -----------------------------------------------------------------------
// Pair j of the last r dims at position pos rotates by pos * theta_j,
// theta_j = base^(-2j/r).  The angle pos * theta_j is formed in double (its
// error is ~2^-53 of |angle|, about 1e-10 rad at pos = 2^20) and reduced to
// [-pi, pi] by Cody-Waite reduction with 2*pi split into a double head and
// tail, k = rint(angle / 2pi): r = (angle - k*hi) - k*lo, each step one fma.
// cos/sin of the reduced float angle then come from sincosf (|r| <= pi).
__device__ __forceinline__ double rope_theta(int j, int r, double base) {
  return pow(base, -2.0 * (double)j / (double)r);
}
__device__ __forceinline__ void rope_sincos(double pos, double theta, float* c, float* s) {
  const double kTwoPiHi = 6.283185307179586;           // 2*pi rounded to double
  const double kTwoPiLo = 2.4492935982947064e-16;      // 2*pi - kTwoPiHi
  const double x = pos * theta;
  const double k = rint(x * (1.0 / kTwoPiHi));
  const double red = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, x));
  sincosf((float)red, s, c);
}
__device__ __forceinline__ void rope_cos_sin(double pos, int j, int r, double base, float* c, float* s) {
  rope_sincos(pos, rope_theta(j, r, base), c, s);
}

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// L2 prefetch of `bytes` contiguous bytes (16-byte aligned address, multiple of 16).
// One 128-byte line into L2 (a plain load-unit prefetch, no TMA op).
__device__ __forceinline__ void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---- programmatic dependent launch --------------------------------------------
// Every kernel of the library is launched so that it may start while the
// previous kernel in the stream finishes.  Before its first read of global
// data that an earlier kernel of the library may write (compressed rows,
// scores, selections, partials) and before its first global write, a thread
// calls griddep_wait(), which returns once every prerequisite grid has
// completed and its writes are visible (at once when there is none).  A
// kernel signals its dependents only after its own wait: so when a kernel
// starts, everything queued before its predecessor (the caller's work
// included) has completed, and it may read the call's inputs before its own
// wait.  The first kernel of a call reads nothing before its wait.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel in the stream be scheduled once every CTA of this grid
// has issued it or exited.
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

}  // namespace csahca
