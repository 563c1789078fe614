// la2_common.cuh -- small device helpers shared by the libla2 kernels.
//
// Everything in libla2 is compiled as ONE translation unit (la2_api.cu
// includes the kernel headers), so the device error word below is a single
// object without relocatable device code.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace la2 {

// Error word written by device code (bounded waits that gave up, bounds
// checks).  Bit 0: a wait timed out.  Read and cleared by
// la2_last_device_error().
__device__ unsigned int g_error_word = 0;

enum : unsigned int { ERR_TIMEOUT = 1u, ERR_BOUNDS = 2u };

// Trace buffer: when a pass is traced, CTA 0 stamps %globaltimer at fixed
// points of each block into g_trace[event * kTraceBlocks + block].
constexpr int kTraceEvents = 16, kTraceBlocks = 512;
__device__ unsigned long long g_trace[kTraceEvents * kTraceBlocks];

__device__ __forceinline__ void raise_error(unsigned int bits) {
  atomicOr(&g_error_word, bits);
}

// ---------------------------------------------------------------- dtypes
template <typename T> struct io;
template <> struct io<float> {
  static __device__ __forceinline__ float ld(const float *p) { return *p; }
  static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
};
template <> struct io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) {
    *p = __float2bfloat16_rn(x);
  }
};

// lambda^n for an integer n >= 0 by binary exponentiation (square and
// multiply) in fp64; 0^0 = 1.  Used to build the small per-CTA decay tables,
// so its cost does not matter; fp64 keeps the table entries within an ulp
// of the fp32 they are rounded to.
__device__ __forceinline__ double pow_int(double x, long long n) {
  double r = 1.0;
  while (n > 0) {
    if (n & 1) r *= x;
    x *= x;
    n >>= 1;
  }
  return r;
}

}  // namespace la2
