// Internal helpers shared by the kernels of libmoe_b200 (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------- launches
// Process-wide count of kernels this library has launched (diagnostic only).
void count_launch(int n = 1);

// Device status word layout at the start of every workspace.
constexpr size_t kStatusBytes = 256;
enum : int { kDevOk = 0, kDevTimeout = 1 };

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

#define MOE_CUDA_TRY(expr)                                  \
  do {                                                      \
    cudaError_t _e = (expr);                                \
    if (_e != cudaSuccess) return MOE_ERR_CUDA;             \
  } while (0)

#define MOE_LAUNCH_CHECK()                                  \
  do {                                                      \
    ::moe::count_launch();                                  \
    cudaError_t _e = cudaGetLastError();                    \
    if (_e != cudaSuccess) return MOE_ERR_CUDA;             \
  } while (0)

// ---------------------------------------------------------- checked builds
// Built with MOE_CHECKED (build.py --checked -> libmoe_b200_checked.so), the
// kernels check the indices they read from their inputs (row maps, slot rows,
// expert offsets) before using them: an index out of range skips the access
// and counts a violation in the compiling file's device counter, which
// moe_checked_violations() reads; nothing traps.  Other builds trust their
// inputs and compile the checks away.
#ifdef MOE_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// One counter per source file (device variables are not shared between files
// without relocatable device code); `reader` returns the count and clears it.
#define MOE_VIOLATION_COUNTER(reader)                                                 \
  namespace {                                                                         \
  __device__ unsigned int g_violations;                                               \
  __device__ __forceinline__ void note_violation() { atomicAdd(&g_violations, 1u); }  \
  }                                                                                   \
  unsigned int reader() {                                                             \
    unsigned int h = 0, z = 0;                                                        \
    if (cudaMemcpyFromSymbol(&h, g_violations, sizeof(h)) != cudaSuccess) return 0;   \
    if (cudaMemcpyToSymbol(g_violations, &z, sizeof(z)) != cudaSuccess) return h;     \
    return h;                                                                         \
  }

// ------------------------------------------------------------ element types
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// 16-byte vector of elements: 4 floats or 8 bf16.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  float4 v;
  __device__ __forceinline__ float get(int i) const { return (&v.x)[i]; }
  __device__ __forceinline__ void set(int i, float f) { (&v.x)[i] = f; }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  uint4 v;
  __device__ __forceinline__ float get(int i) const {
    uint32_t w = (&v.x)[i >> 1];
    uint32_t bits = (i & 1) ? (w & 0xFFFF0000u) : (w << 16);
    return __uint_as_float(bits);
  }
  __device__ __forceinline__ void set(int i, float f) {
    uint32_t b = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
    uint32_t &w = (&v.x)[i >> 1];
    w = (i & 1) ? ((w & 0x0000FFFFu) | (b << 16)) : ((w & 0xFFFF0000u) | b);
  }
};

template <typename T>
__device__ __forceinline__ Vec16<T> load16(const T *p) {
  Vec16<T> r;
  r.v = *reinterpret_cast<const decltype(r.v) *>(p);
  return r;
}
template <typename T>
__device__ __forceinline__ void store16(T *p, const Vec16<T> &r) {
  *reinterpret_cast<decltype(r.v) *>(p) = r.v;
}

// --------------------------------------------------------- gate functions
// softplus(s) = ln(1 + e^s) in the overflow-free form max(s,0) + ln(1 + e^-|s|).
__device__ __forceinline__ float softplus_f32(float s) {
  return fmaxf(s, 0.0f) + log1pf(expf(-fabsf(s)));
}
__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

// SwiGLU hidden value with the optional clamp (limit <= 0: off).
__device__ __forceinline__ float swiglu_h(float g, float u, float limit, int clamp_mode) {
  if (limit > 0.0f && clamp_mode == MOE_CLAMP_PREACT) {
    g = fminf(fmaxf(g, -limit), limit);
    u = fminf(fmaxf(u, -limit), limit);
  }
  float h = silu_f32(g) * u;
  if (limit > 0.0f && clamp_mode == MOE_CLAMP_OUTPUT) h = fminf(fmaxf(h, -limit), limit);
  return h;
}

}  // namespace moe
