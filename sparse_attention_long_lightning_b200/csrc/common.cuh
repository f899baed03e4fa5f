// common.cuh -- device helpers shared by the libsala kernels (single translation unit).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sala.h"

namespace sala {

// Device error word: first device-detected condition since the last read
// (0 = none, else a sala_status value).  One per device context.
__device__ int g_device_error;

__device__ __forceinline__ void raise_device_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

// SALA_IN_BOUNDS(cond): true when cond holds.  Built with SALA_DEBUG, a false cond
// records its source line (the first since the last read), raises SALA_ERR_BOUNDS and
// yields false, so the caller skips the access; otherwise the check compiles to true and
// cond is not evaluated.
#ifdef SALA_DEBUG
__device__ int g_bounds_line;
__device__ __noinline__ bool bounds_failed(int line) {
  atomicCAS(&g_bounds_line, 0, line);
  raise_device_error(SALA_ERR_BOUNDS);
  return false;
}
#define SALA_IN_BOUNDS(cond) ((cond) ? true : ::sala::bounds_failed(__LINE__))
#else
#define SALA_IN_BOUNDS(cond) true
#endif

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};
template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
  }
};

template <typename T>
__device__ __forceinline__ float ld(const T* p) { return Elem<T>::load(p); }
template <typename T>
__device__ __forceinline__ void st(T* p, float x) { Elem<T>::store(p, x); }

// Logistic sigmoid with the fast approximate divide (a few ulp; an exact IEEE
// division here costs a multi-instruction sequence per output element).
__device__ __forceinline__ float sigmoidf_(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

// Rotary angle for position `pos` and pair i of a D-dim head, reduced to
// [-pi, pi] in double precision before the fp32 sine/cosine, so that long
// positions (up to 2^31) keep the angle accurate:
//   theta = pos * base^(-2i/D)   (rotate-half RoPE, inverse frequency base^(-2i/D))
__device__ __forceinline__ void rope_cos_sin(int64_t pos, int i, int D, double log2_base,
                                             float* c, float* s) {
  const double inv_freq = exp2(-(2.0 * (double)i / (double)D) * log2_base);
  const double a = (double)pos * inv_freq;
  const double two_pi = 6.283185307179586476925286766559;
  const double r = a - rint(a * (1.0 / two_pi)) * two_pi;
  sincosf((float)r, s, c);
}

// Bounded spin budget (cycles) for mbarrier waits: about 2 s at 1.9 GHz.
constexpr long long kSpinCycleBudget = 4000000000LL;

}  // namespace sala
