// la2_decode.cuh -- recurrent decode steps, HBM-bound.
//
//   kv <- lambda kv + k^T v,   o = q kv        (per (b,h), kv fp32 d x e)
//
// applied to T consecutive tokens per call (T = 1: one step).
//
// The recurrent form with a fixed-size state (Lightning Attention glossary
// page, section "主な特徴・仕組み").  Each step must read and write the whole
// fp32 state once, so the kernel is a streaming pass over 2 * d * e * 4 bytes
// per (b,h): one CTA per state, each warp owns d/8 rows, each lane a 16-byte
// (e = 128) or 8-byte (e = 64) column slice, so every warp-wide load or store
// is one contiguous 512/256-byte row.  All of a thread's row loads are issued
// before any arithmetic so ~64 KB per CTA is in flight; loads and stores use
// the streaming (evict-first) cache hint since the state is touched once per
// step.  The column sums o_j = sum_i q_i kv_ij are reduced across warps in
// shared memory.
#pragma once

#include "la2_common.cuh"

namespace la2 {
namespace dec {

constexpr int NT = 256;
constexpr int NW = NT / 32;

template <int VEC> struct vec_t;
template <> struct vec_t<4> {
  using type = float4;
  static __device__ __forceinline__ float4 ld(const float *p) {
    return __ldcs(reinterpret_cast<const float4 *>(p));
  }
  static __device__ __forceinline__ void st(float *p, float4 x) {
    __stcs(reinterpret_cast<float4 *>(p), x);
  }
  static __device__ __forceinline__ float &at(float4 &x, int i) {
    return reinterpret_cast<float *>(&x)[i];
  }
};
template <> struct vec_t<2> {
  using type = float2;
  static __device__ __forceinline__ float2 ld(const float *p) {
    return __ldcs(reinterpret_cast<const float2 *>(p));
  }
  static __device__ __forceinline__ void st(float *p, float2 x) {
    __stcs(reinterpret_cast<float2 *>(p), x);
  }
  static __device__ __forceinline__ float &at(float2 &x, int i) {
    return reinterpret_cast<float *>(&x)[i];
  }
};

// T tokens per (b,h) in order: the state is read once, updated T times in
// registers (o_t from the state after token t), and written back once.  The
// state of request b lives at pool[slot], slot = slots[b] (slots NULL: slot =
// b); a negative slot marks an inactive request (nothing read or written), a
// slot >= pool_size is recorded as a bounds error and skipped.  q, k
// [B,H,T,D], v, o [B,H,T,E]; T = 1 is the single decode step.
// G: tokens per group; the library runs it for single-token calls (G = 1,
// the plain one-token loop) and tokens_kernel for several tokens per call.
template <typename T, int D, int E, int G>
__global__ void __launch_bounds__(NT)
decode_kernel(const T *__restrict__ q, const T *__restrict__ k,
              const T *__restrict__ v, const float *__restrict__ lambda,
              float *__restrict__ pool, const int *__restrict__ slots, int pool_size,
              T *__restrict__ o, int H, int ntok) {
  constexpr int ROWS = D / NW;   // rows per warp
  constexpr int VEC = E / 32;    // columns per lane
  using V = vec_t<VEC>;
  // tokens go in groups of G: one load of their q, k, v and one cross-warp
  // reduction of their outputs per group (two block syncs per G tokens)
  __shared__ float qs[G][D], ks[G][D], vs[G][E];
  __shared__ float red[NW][G][E];

  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H;
  const int h = (int)(bh % H);
  const int tid = threadIdx.x, w = tid / 32, l = tid % 32;
  int64_t slot = b;
  if (slots) {
    slot = slots[b];
    if (slot < 0) return;  // inactive request
    if (slot >= pool_size) {
      if (tid == 0) raise_error(ERR_BOUNDS);
      return;
    }
  }
  const float lam = lambda[h];
  float *base = pool + (slot * H + h) * (int64_t)D * E + (int64_t)(w * ROWS) * E + l * VEC;
  typename V::type x[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; r++) x[r] = V::ld(base + (int64_t)r * E);

  for (int t0 = 0; t0 < ntok; t0 += G) {
    const int ng = ntok - t0 < G ? ntok - t0 : G;
    const int64_t tok0 = bh * ntok + t0;
    for (int idx = tid; idx < ng * D; idx += NT) {
      qs[idx / D][idx % D] = io<T>::ld(q + tok0 * D + idx);
      ks[idx / D][idx % D] = io<T>::ld(k + tok0 * D + idx);
    }
    for (int idx = tid; idx < ng * E; idx += NT) vs[idx / E][idx % E] = io<T>::ld(v + tok0 * E + idx);
    __syncthreads();  // this group's q, k, v in; the last group's sums read out

    float acc[G][VEC];
#pragma unroll
    for (int g = 0; g < G; g++) {
      if (g >= ng) break;
      float vv[VEC];
#pragma unroll
      for (int c = 0; c < VEC; c++) {
        vv[c] = vs[g][l * VEC + c];
        acc[g][c] = 0.f;
      }
#pragma unroll
      for (int r = 0; r < ROWS; r++) {
        const int i = w * ROWS + r;
        const float ki = ks[g][i], qi = qs[g][i];
#pragma unroll
        for (int c = 0; c < VEC; c++) {
          float sv = fmaf(lam, V::at(x[r], c), ki * vv[c]);
          V::at(x[r], c) = sv;
          acc[g][c] = fmaf(qi, sv, acc[g][c]);
        }
        // the last token's row goes out as soon as it is final
        if (t0 + g == ntok - 1) V::st(base + (int64_t)r * E, x[r]);
      }
#pragma unroll
      for (int c = 0; c < VEC; c++) red[w][g][l * VEC + c] = acc[g][c];
    }
    __syncthreads();  // every warp's partial sums of the group in
    for (int idx = tid; idx < ng * E; idx += NT) {
      const int g = idx / E, j = idx % E;
      float sum = 0.f;
#pragma unroll
      for (int ww = 0; ww < NW; ww++) sum += red[ww][g][j];
      io<T>::st(o + (tok0 + g) * E + j, sum);
    }
  }
}

// Several tokens per call (T = ntok >= 2): decode_kernel's state update
// with the tokens' q, k, v staged in shared memory up to TS = 8 at a time (one
// load of all of them, in flight together with the state's), and the
// per-group cross-warp sums double-buffered, so each group of G tokens costs
// one block barrier and no exposed global-load latency.  512 threads per
// state (16 warps of D / 16 rows): from T ~ 8 the per-state token work, not
// the state's traffic, sets the time, and this spreads it over twice
// decode_kernel's threads while two states still fit an SM (measured on
// B200: 0.50 against 0.58 ms per call at T = 8 for batch 256 x 64 heads;
// 1,024 threads, one state per SM, 0.71 ms).
constexpr int NTT = 512;           // threads per state (tokens_kernel)
constexpr int NWT = NTT / 32;
template <int E, int G> constexpr size_t tokens_smem() { return sizeof(float) * 2 * NWT * G * E; }

template <typename T, int D, int E, int G>
__global__ void __launch_bounds__(NTT)
tokens_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const float *__restrict__ lambda, float *__restrict__ pool,
              const int *__restrict__ slots, int pool_size, T *__restrict__ o, int H, int ntok) {
  constexpr int NT = NTT, NW = NWT;  // (this kernel's CTA: 16 warps of D / 16 rows)
  constexpr int ROWS = D / NW;
  constexpr int VEC = E / 32;
  constexpr int TS = 8;  // tokens staged at once
  using V = vec_t<VEC>;
  __shared__ float qs[TS][D], ks[TS][D], vs[TS][E];
  extern __shared__ float red_raw[];  // [2][NW][G][E] cross-warp sums, double-buffered
  auto red = reinterpret_cast<float(*)[NW][G][E]>(red_raw);

  const int64_t bh = blockIdx.x;
  const int64_t b = bh / H;
  const int h = (int)(bh % H);
  const int tid = threadIdx.x, w = tid / 32, l = tid % 32;
  int64_t slot = b;
  if (slots) {
    slot = slots[b];
    if (slot < 0) return;  // inactive request
    if (slot >= pool_size) {
      if (tid == 0) raise_error(ERR_BOUNDS);
      return;
    }
  }
  const float lam = lambda[h];
  float *base = pool + (slot * H + h) * (int64_t)D * E + (int64_t)(w * ROWS) * E + l * VEC;
  typename V::type x[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; r++) x[r] = V::ld(base + (int64_t)r * E);

  int gi = 0;  // groups done (the parity picks the sums buffer)
  for (int c0 = 0; c0 < ntok; c0 += TS) {
    const int nc = ntok - c0 < TS ? ntok - c0 : TS;
    const int64_t tokc = bh * ntok + c0;
    // (the previous chunk's q, k, v were last read before the barrier of
    // its last group, which every thread has passed)
    for (int idx = tid; idx < nc * D; idx += NT) {
      qs[idx / D][idx % D] = io<T>::ld(q + tokc * D + idx);
      ks[idx / D][idx % D] = io<T>::ld(k + tokc * D + idx);
    }
    for (int idx = tid; idx < nc * E; idx += NT) vs[idx / E][idx % E] = io<T>::ld(v + tokc * E + idx);
    __syncthreads();  // the chunk's q, k, v in
    for (int t0 = 0; t0 < nc; t0 += G) {
      const int ng = nc - t0 < G ? nc - t0 : G;
      // sums buffer of this group: the group before last read it before the
      // last group's barrier
      float(*rb)[G][E] = red[gi & 1];
      gi++;
#pragma unroll
      for (int g = 0; g < G; g++) {
        if (g >= ng) break;
        const int tt = t0 + g;
        float vv[VEC], acc[VEC];
#pragma unroll
        for (int c = 0; c < VEC; c++) {
          vv[c] = vs[tt][l * VEC + c];
          acc[c] = 0.f;
        }
#pragma unroll
        for (int r = 0; r < ROWS; r++) {
          const int i = w * ROWS + r;
          const float ki = ks[tt][i], qi = qs[tt][i];
#pragma unroll
          for (int c = 0; c < VEC; c++) {
            float sv = fmaf(lam, V::at(x[r], c), ki * vv[c]);
            V::at(x[r], c) = sv;
            acc[c] = fmaf(qi, sv, acc[c]);
          }
          // the last token's row goes out as soon as it is final
          if (c0 + tt == ntok - 1) V::st(base + (int64_t)r * E, x[r]);
        }
#pragma unroll
        for (int c = 0; c < VEC; c++) rb[w][g][l * VEC + c] = acc[c];
      }
      __syncthreads();  // every warp's partial sums of the group in
      for (int idx = tid; idx < ng * E; idx += NT) {
        const int g = idx / E, j = idx % E;
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ww++) sum += rb[ww][g][j];
        io<T>::st(o + (tokc + t0 + g) * E + j, sum);
      }
    }
  }
}

}  // namespace dec
}  // namespace la2
