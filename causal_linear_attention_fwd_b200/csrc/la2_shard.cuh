// la2_shard.cuh -- the state algebra of a sequence split into shards.
//
// A long sequence cut into R equal shards of Ls rows (one per GPU) needs,
// per shard, only two d x e summaries of the others: the forward state
// entering it and the reverse state flowing into it from the rows after it.
// Both are exact reassociations of the block recurrence (Lightning
// Attention-2 notes page, "Tiling." paragraph):
//   forward delta of a shard  dF = sum_t lambda^(Ls-1-t) k_t^T v_t
//   reverse delta of a shard  dR = sum_t lambda^t q_t^T dO_t
//   entry state of shard r    F_r = lambda^Ls F_{r-1} + dF_{r-1},  F_0 = kv0
//   end state of shard r      R_r = lambda^Ls R_{r+1} + dR_{r+1},  R_{R-1} = 0
// (t local to the shard).  The deltas themselves come from the chunk-state
// passes over sub-chunks of the shard, combined here.
#pragma once

#include "la2_common.cuh"

namespace la2 {
namespace shard {

constexpr int NT = 256;

// One shard's delta from its nsub sub-chunk deltas, slots [first, first +
// nsub) of each (b,h)'s workspace row of wsS slots: forward (sub-chunk
// deltas relative to their end) sum_c lambda^(L - end_c) delta_c, reverse
// (relative to their start) sum_c lambda^(start_c) delta_c; sub-chunks of
// Ls rows, the last one L - (nsub-1) Ls.  Horner's rule in both directions.
template <int D, int E>
__global__ void __launch_bounds__(NT)
combine_kernel(const float *__restrict__ ws, int wsS, int first, int nsub, int64_t Ls,
               int64_t L, const float *__restrict__ lambda, int H, int reverse,
               float *__restrict__ out) {
  const int64_t bh = blockIdx.y;
  const int idx = blockIdx.x * NT + threadIdx.x;
  if (idx >= D * E) return;
  const double lam = (double)lambda[bh % H];
  const float full = (float)pow_int(lam, Ls);
  const float last = (float)pow_int(lam, L - (int64_t)(nsub - 1) * Ls);
  const float *base = ws + (bh * wsS + first) * (int64_t)D * E + idx;
  float run = 0.f;
  if (!reverse) {
    for (int c = 0; c < nsub; c++)
      run = (c == nsub - 1 ? last : full) * run + base[(int64_t)c * D * E];
  } else {
    for (int c = nsub - 1; c >= 0; c--)
      run = (c == nsub - 1 ? last : full) * run + base[(int64_t)c * D * E];
  }
  out[bh * D * E + idx] = run;
}

// Per-shard entry (forward) or end (reverse) states from the R shards'
// deltas [R, B*H, D*E]; out [R, B*H, D*E].  Forward: out[0] = kv0 (or 0),
// out[r] = lambda^Ls out[r-1] + delta[r-1]; reverse: out[R-1] = 0, out[r] =
// lambda^Ls out[r+1] + delta[r+1].
template <int D, int E>
__global__ void __launch_bounds__(NT)
prefix_kernel(const float *__restrict__ delta, const float *__restrict__ kv0,
              const float *__restrict__ lambda, int H, int R, int64_t BH, int64_t Ls,
              int reverse, float *__restrict__ out) {
  const int64_t bh = blockIdx.y;
  const int idx = blockIdx.x * NT + threadIdx.x;
  if (idx >= D * E) return;
  const float f = (float)pow_int((double)lambda[bh % H], Ls);
  const int64_t one = (int64_t)D * E, stride = BH * one;
  const int64_t at = bh * one + idx;
  if (!reverse) {
    float run = (kv0 ? kv0[at] : 0.f);
    out[at] = run;
    for (int r = 1; r < R; r++) {
      run = f * run + delta[(int64_t)(r - 1) * stride + at];
      out[(int64_t)r * stride + at] = run;
    }
  } else {
    float run = 0.f;
    out[(int64_t)(R - 1) * stride + at] = run;
    for (int r = R - 2; r >= 0; r--) {
      run = f * run + delta[(int64_t)(r + 1) * stride + at];
      out[(int64_t)r * stride + at] = run;
    }
  }
}

}  // namespace shard
}  // namespace la2
