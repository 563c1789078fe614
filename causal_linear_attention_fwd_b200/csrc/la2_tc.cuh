// la2_tc.cuh -- tensor-core (tcgen05 / TMEM / TMA) kernels for bf16, d = e = 128.
#pragma once

#include "la2_common.cuh"
#include "la2_simt.cuh"

namespace la2 {
namespace tc {

constexpr int BLOCK = 128;

inline bool supports(int d, int e, bool bf16) { return false && bf16 && d == 128 && e == 128; }

inline int64_t auto_split(int64_t BH, int64_t nblk, int sms) {
  return BH >= sms ? 1 : (sms + BH - 1) / BH;
}

template <typename Timed>
cudaError_t forward(const void *, const void *, const void *, const float *, const float *,
                    void *, float *, float *, const Geo &, cudaStream_t, Timed &&) {
  return cudaErrorNotSupported;
}

template <typename Timed>
cudaError_t backward(const void *, const void *, const void *, const float *, const float *,
                     const void *, void *, void *, void *, float *, float *, const Geo &,
                     cudaStream_t, Timed &&) {
  return cudaErrorNotSupported;
}

}  // namespace tc
}  // namespace la2
