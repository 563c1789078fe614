// la2_fmap.cuh -- the feature map applied to q and k before the attention,
// and its chain rule for the backward pass.
//
// The Lightning Attention glossary page (section "主な特徴・仕組み") has
// linear attention replace softmax by a kernel feature map, which is what
// lets K^T V be aggregated first, but names no map.  The map built here is
// elu + 1, the positive map of "Transformers are RNNs" (one of the works the
// Luna page lists as its basis, next to the ELU paper):
//
//   phi(x)  = x + 1  (x > 0),   e^x  (x <= 0)
//   phi'(x) = 1      (x > 0),   e^x  (x <= 0)
//
// Forward:  phi_q = phi(q), phi_k = phi(k).
// Backward: dq = dphi_q * phi'(q), dk = dphi_k * phi'(k), where dphi_* are
//           the attention's gradients with respect to its (mapped) inputs.
//
// Both are one streaming pass over q and k together (one launch), HBM-bound:
// the forward moves 2 * (read + write) elements per element of q, the
// backward 2 * (2 reads + 1 write).  Each thread moves 16-byte vectors (8
// bf16 or 4 fp32 values) with the streaming cache hint, and issues U vector
// indices' loads (for both tensors, and the upstream gradients) before any
// arithmetic; CTAs are 1,024 threads, U = 1 for the map and 2 for its
// gradient.  (Measured on B200 at 2 x 268 M bf16 values: many warps with a
// short load-compute-store chain each hide the latency best -- the map at
// 86 % of the copy bandwidth against 70 % with 256 threads and U = 4, the
// gradient at 96 % against 80 %.)  The grid is the SM count times the CTAs
// an SM holds; it walks the vectors with a grid stride.  A ragged tail (n
// not a multiple of the vector width) is done element by element by CTA 0.
// Arithmetic in fp32; e^x is CUDA's expf; results rounded to the I/O type
// (bf16: round to nearest even).
#pragma once

#include "la2_common.cuh"

namespace la2 {
namespace fmap {

// threads per CTA and vector indices in flight per thread, per direction
template <bool GRAD> struct Shape {
  static constexpr int NT = 1024;
  static constexpr int U = GRAD ? 2 : 1;
};

__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float dphi(float x) { return x > 0.f ? 1.f : expf(x); }

// 16 bytes of T as fp32 values.
template <typename T> struct vec16;
template <> struct vec16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void unpack(const uint4 &r, float (&f)[N]) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
  }
  static __device__ __forceinline__ uint4 pack(const float (&f)[N]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};
template <> struct vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void unpack(const uint4 &r, float (&f)[N]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  static __device__ __forceinline__ uint4 pack(const float (&f)[N]) {
    uint4 r;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; i++) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return r;
  }
};

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  return __ldcs(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void st_stream(void *p, const uint4 &x) {
  __stcs(reinterpret_cast<uint4 *>(p), x);
}

// GRAD = false: y_t = phi(x_t).  GRAD = true: y_t = g_t * phi'(x_t).
// Tensor t = 0 is q, t = 1 is k (absent when x1 is null); each has n values.
// An output may be the very buffer of its own tensor's x (or g): every
// element is read before it is written, by the same thread.
template <typename T, bool GRAD>
__global__ void __launch_bounds__(Shape<GRAD>::NT)
map_kernel(const T *x0, const T *g0, T *y0, const T *x1, const T *g1, T *y1, int64_t n) {
  constexpr int NT = Shape<GRAD>::NT, U = Shape<GRAD>::U;
  using V = vec16<T>;
  const int64_t nv = n / V::N;
  const int64_t stride = (int64_t)gridDim.x * NT;
  const int nt = x1 ? 2 : 1;
  const T *xs[2] = {x0, x1};
  const T *gs[2] = {g0, g1};
  T *ys[2] = {y0, y1};
  for (int64_t base = (int64_t)blockIdx.x * NT + threadIdx.x; base < nv; base += stride * U) {
    uint4 xr[2][U], gr[2][U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t i = base + u * stride;
      if (i < nv) {
#pragma unroll
        for (int t = 0; t < 2; t++) {
          if (t < nt) {
            xr[t][u] = ld_stream(xs[t] + i * V::N);
            if constexpr (GRAD) gr[t][u] = ld_stream(gs[t] + i * V::N);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int64_t i = base + u * stride;
      if (i < nv) {
#pragma unroll
        for (int t = 0; t < 2; t++) {
          if (t < nt) {
            float f[V::N];
            V::unpack(xr[t][u], f);
            if constexpr (GRAD) {
              float g[V::N];
              V::unpack(gr[t][u], g);
#pragma unroll
              for (int j = 0; j < V::N; j++) f[j] = g[j] * dphi(f[j]);
            } else {
#pragma unroll
              for (int j = 0; j < V::N; j++) f[j] = phi(f[j]);
            }
            st_stream(ys[t] + i * V::N, V::pack(f));
          }
        }
      }
    }
  }
  if (blockIdx.x == 0) {
    for (int64_t j = nv * V::N + threadIdx.x; j < n; j += NT) {
      for (int t = 0; t < nt; t++) {
        const float x = io<T>::ld(xs[t] + j);
        float y;
        if constexpr (GRAD) y = io<T>::ld(gs[t] + j) * dphi(x);
        else y = phi(x);
        io<T>::st(ys[t] + j, y);
      }
    }
  }
}

// CTAs for n values per tensor: the SM count times the CTAs one SM holds,
// fewer when there is not that much work.
template <typename T, bool GRAD>
int grid_for(int64_t n, int sms) {
  constexpr int NT = Shape<GRAD>::NT, U = Shape<GRAD>::U;
  static int per_sm = [] {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, map_kernel<T, GRAD>, NT, 0) !=
            cudaSuccess ||
        b < 1)
      b = 1;
    return b;
  }();
  const int64_t nv = n / vec16<T>::N;
  const int64_t need = (nv + (int64_t)NT * U - 1) / ((int64_t)NT * U);
  const int64_t full = (int64_t)sms * per_sm;
  return (int)(need < 1 ? 1 : (need < full ? need : full));
}

// Enqueues the launch; the caller reads the launch status.
template <typename T, bool GRAD>
void enqueue(const void *x0, const void *g0, void *y0, const void *x1, const void *g1, void *y1,
             int64_t n, int grid, cudaStream_t st) {
  map_kernel<T, GRAD><<<grid, Shape<GRAD>::NT, 0, st>>>(
      static_cast<const T *>(x0), static_cast<const T *>(g0), static_cast<T *>(y0),
      static_cast<const T *>(x1), static_cast<const T *>(g1), static_cast<T *>(y1), n);
}

}  // namespace fmap
}  // namespace la2
