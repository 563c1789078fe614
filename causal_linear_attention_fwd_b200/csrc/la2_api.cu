// la2_api.cu -- the C ABI of libla2 (see include/la2.h): argument checks,
// chunk planning, workspace carving, kernel dispatch, device error word and
// per-kernel event timing.  The whole library is this one translation unit.
#include <cuda_runtime.h>

#include <atomic>
#include <initializer_list>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>
#include <vector>

#include "../../include/la2.h"
#include "la2_common.cuh"
#include "la2_decode.cuh"
#include "la2_dlam_tc.cuh"
#include "la2_fmap.cuh"
#include "la2_shard.cuh"
#include "la2_simt.cuh"
#include "la2_tc.cuh"

namespace {

using la2::Geo;

std::atomic<int> g_opt_split{0};
std::atomic<int> g_opt_path{0};
std::atomic<int> g_opt_inject{0};
std::atomic<int> g_opt_variant{0};
std::atomic<int> g_opt_trace{0};
std::atomic<int> g_opt_varlen_order{0};
std::atomic<int> g_opt_decode_block{0};
std::atomic<int> g_opt_bwd_form{0};

// ------------------------------------------------------------ profiling
enum KernelId {
  K_SIMT_FWD_STATE, K_SIMT_FWD_SCAN, K_SIMT_FWD, K_SIMT_DQ, K_SIMT_REV_STATE,
  K_SIMT_REV_SCAN, K_SIMT_DKDV, K_DECODE, K_TC_FWD_STATE, K_TC_FWD, K_TC_DQ,
  K_TC_REV_STATE, K_TC_DV, K_TC_DK, K_SCAN_FWD, K_SCAN_REV, K_SIMT_DLAMBDA,
  K_SIMT_DLAMBDA_STATE, K_SIMT_DLAMBDA_SCAN, K_TC_DECODE_UNITS, K_FMAP, K_FMAP_GRAD, K_TC_DKDV,
  K_TC_DLAMBDA, K_TC_DLAMBDA_STATE, K_STATE_PAD, K_COUNT
};
const char *kKernelName[K_COUNT] = {
    "simt_fwd_chunk_state", "simt_scan_fwd", "simt_fwd", "simt_dq",
    "simt_rev_chunk_state", "simt_scan_rev", "simt_dkdv", "decode_step",
    "tc_fwd_chunk_state", "tc_fwd", "tc_dq", "tc_rev_chunk_state", "tc_dv", "tc_dk",
    "scan_fwd", "scan_rev", "simt_dlambda", "simt_dlambda_chunk_state", "simt_dlambda_scan",
    "tc_decode_units", "feature_map", "feature_map_grad", "tc_dkdv", "tc_dlambda",
    "tc_dlambda_chunk_state", "state_pad"};

struct ProfRec {
  int kid;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::atomic<int> g_prof_on{0};
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_ev_pool;
constexpr size_t kMaxProfRecs = 1 << 16;

cudaEvent_t ev_get() {
  if (!g_ev_pool.empty()) {
    cudaEvent_t e = g_ev_pool.back();
    g_ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Runs `launch` (which enqueues one kernel on `st`) and, while profiling is
// on, brackets it with events.  Returns the launch error, if any.
// Runs a launch callable: one that returns void (the launch's error is
// then the runtime's last error) or its own cudaError_t.
template <typename F>
cudaError_t run_launch(F &&launch) {
  if constexpr (std::is_same_v<decltype(launch()), cudaError_t>) {
    const cudaError_t e = launch();
    const cudaError_t last = cudaGetLastError();
    return e != cudaSuccess ? e : last;
  } else {
    launch();
    return cudaGetLastError();
  }
}

template <typename F>
cudaError_t timed(int kid, cudaStream_t st, F &&launch) {
  if (!g_prof_on.load(std::memory_order_relaxed)) return run_launch(launch);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t a = nullptr, b = nullptr;
  if (g_prof.size() < kMaxProfRecs) {
    a = ev_get();
    b = ev_get();
  }
  if (a) cudaEventRecord(a, st);
  cudaError_t err = run_launch(launch);
  if (a && b) {
    cudaEventRecord(b, st);
    g_prof.push_back({kid, a, b});
  }
  return err;
}

// ------------------------------------------------------------- helpers
int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

int device_cc() {
  int dev = 0, ma = 0, mi = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  cudaDeviceGetAttribute(&ma, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&mi, cudaDevAttrComputeCapabilityMinor, dev);
  return ma * 10 + mi;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Span {
  const void *p;
  size_t n;
};
bool overlaps(Span x, Span y) {
  if (!x.p || !y.p || x.n == 0 || y.n == 0) return false;
  uintptr_t a0 = reinterpret_cast<uintptr_t>(x.p), a1 = a0 + x.n;
  uintptr_t b0 = reinterpret_cast<uintptr_t>(y.p), b1 = b0 + y.n;
  return a0 < b1 && b0 < a1;
}
// An output sharing any byte with an input (an exact alias included) or
// with another output.
bool any_overlap(const std::vector<Span> &outs, const std::vector<Span> &ins) {
  for (size_t i = 0; i < outs.size(); i++) {
    for (size_t j = 0; j < ins.size(); j++)
      if (overlaps(outs[i], ins[j])) return true;
    for (size_t j = i + 1; j < outs.size(); j++)
      if (overlaps(outs[i], outs[j])) return true;
  }
  return false;
}

bool shape_supported(int d, int e, la2_dtype dt) {
  return (d == 64 || d == 128) && (e == 64 || e == 128) &&
         (dt == LA2_F32 || dt == LA2_BF16);
}

size_t esize(la2_dtype dt) { return dt == LA2_F32 ? 4 : 2; }

// Which kernel family serves a call.  any_head: the entry point runs the
// tensor-core passes for head sizes 64 too (its 64-column tensors read with
// zero columns beyond their width, its states padded to 128 x 128 in
// workspace scratch); else bf16 with d = e = 128 only.
enum Path { PATH_SIMT = 0, PATH_TC = 1, PATH_NONE = 2 };
Path choose_path(int d, int e, la2_dtype dt, bool any_head = false) {
  const int opt = g_opt_path.load();
  const bool shape_ok = la2::tc::supports(d, e, dt == LA2_BF16) ||
                        (any_head && dt == LA2_BF16 && shape_supported(d, e, dt));
  const bool tc_ok = shape_ok && device_cc() == 100;
  if (opt == 1) return PATH_SIMT;
  if (opt == 2) return tc_ok ? PATH_TC : PATH_NONE;
  return tc_ok ? PATH_TC : PATH_SIMT;
}

// Chunk plan: split each (b,h) sequence into S chunks of Lc rows (Lc a
// multiple of the block size `blk`) so that B*H*S CTAs fill the GPU.
// slots: how many chunks the GPU runs at once (0: one per SM; the paired
// reverse pass runs one per two SMs).
Geo plan(int B, int H, int64_t L, int blk, Path path, int slots = 0) {
  Geo g;
  g.cu = nullptr;
  g.lpt = 0;
  g.slots = nullptr;
  g.pool = 0;
  g.inject = 0;
  g.variant = g_opt_variant.load();
  g.trace = g_opt_trace.load() - 1;
  g.B = B;
  g.H = H;
  g.L = L;
  const int64_t nblk = (L + blk - 1) / blk;
  int64_t S = g_opt_split.load();
  if (S <= 0) {
    const int64_t BH = (int64_t)B * H;
    const int sms = device_sms();
    S = path == PATH_TC ? la2::tc::auto_split(BH, nblk, slots > 0 ? slots : sms)
                        : (BH >= 2 * sms ? 1 : (2 * sms + BH - 1) / BH);
  }
  if (S > nblk) S = nblk;
  if (S < 1) S = 1;
  const int64_t per = (nblk + S - 1) / S;
  g.Lc = per * blk;
  g.S = (int)((L + g.Lc - 1) / g.Lc);
  if (g.S < 1) g.S = 1;
  // Sub-chunks for the tensor-core chunk-state pre-passes: those passes
  // have B*H*(S-1) chunks, fewer than the SMs when the split exists at all,
  // so each chunk is cut into M sub-chunks, M minimising (waves of CTAs) x
  // (blocks per CTA).  Lc becomes M * Ls with Ls a multiple of the block.
  int64_t M = 1;
  if (path == PATH_TC && g.S > 1) {
    const int sms = device_sms();
    const int64_t work = (int64_t)B * H * (g.S - 1);
    int64_t best = -1;
    for (int64_t m = 1; m <= 8 && m <= per; m++) {
      const int64_t cost = ((work * m + sms - 1) / sms) * ((per + m - 1) / m);
      if (best < 0 || cost < best) {
        best = cost;
        M = m;
      }
    }
    g.Lc = M * (((per + M - 1) / M) * blk);
    g.S = (int)((L + g.Lc - 1) / g.Lc);
    if (g.S <= 1) {
      g.S = 1;
      M = 1;
    }
  }
  g.M = (int)M;
  g.Ls = g.Lc / M;
  g.Ssub = (int)((L + g.Ls - 1) / g.Ls);
  g.wsS = g.Ssub;
  g.nst = g.S - 1;
  g.c0 = 0;
  return g;
}

int block_rows(Path p) { return p == PATH_TC ? la2::tc::BLOCK : la2::simt::C; }

// Whether the tensor-core backward runs dV and dK as one paired launch (two
// CTAs per chunk in clusters of two) rather than as two passes: yes unless
// LA2_OPT_BWD_FORM = 1 or the phase-serial kernel form is forced.
bool rev_paired(Path p) {
  return p == PATH_TC && g_opt_bwd_form.load() != 1 && g_opt_variant.load() != 1;
}

// Chunk plan of the backward's reverse passes.  Paired, each chunk occupies
// two SMs, so the automatic split aims at SMs / 2 chunks at a time: fewer
// chunks per sequence than the forward scan's plan, and so fewer chunk
// boundaries for the reverse chunk-state pre-pass to cover.  A forced split
// (LA2_OPT_SPLIT) applies to both plans alike.
Geo plan_rev(int B, int H, int64_t L, Path p) {
  if (!rev_paired(p)) return plan(B, H, L, block_rows(p), p);
  Geo g = plan(B, H, L, block_rows(p), p, device_sms() / 2);
  g.rev_pair = 1;
  return g;
}

// Chunk plan of the decay gradient (blocks of blk rows: 32 for the fp32-FMA
// kernel, one CTA per chunk; 128 for the tensor-core one, two CTAs per chunk,
// one per half of the e columns): at most one wave, S = floor(slots / (B*H))
// chunks per sequence when B*H is below the slots -- the SMs, or half of them
// for the tensor-core kernel (LA2_OPT_SPLIT overrides) -- Lc a multiple of
// the block.  (Counting a tensor-core chunk as one slot would split B*H = 64
// sequences in two on 148 SMs: 256 CTAs, two waves as long as the one wave of
// 128 unsplit, plus the pre-pass and the scan.)
// The chunk-state pre-pass covers chunks 0..S-2 only, so it runs on M
// sub-chunks of Ls rows per chunk (Lc = M Ls), M filling the slots (at most
// 8); the workspace holds (S-1) M + 1 (KV, W) pairs per (b,h).
Geo plan_dlambda(int B, int H, int64_t L, bool split_ok, int blk_rows) {
  Geo g = plan(B, H, L, blk_rows, PATH_SIMT);
  const int64_t blk = blk_rows, nblk = (L + blk - 1) / blk;
  const int64_t BH = (int64_t)B * H;
  const int slots = blk_rows == la2::tc::BLOCK ? device_sms() / 2 : device_sms();
  int64_t S = g_opt_split.load();
  if (S <= 0) S = BH >= slots ? 1 : slots / BH;
  if (!split_ok || S > nblk) S = split_ok ? nblk : 1;
  if (S < 1) S = 1;
  int64_t per = (nblk + S - 1) / S;  // blocks per chunk
  S = (nblk + per - 1) / per;
  int64_t M = 1;
  if (S > 1) {
    // the largest M <= min(8, slots / (B*H*(S-1))) whose whole sub-chunks
    // keep S chunks
    int64_t want = slots / (BH * (S - 1));
    if (want > 8) want = 8;
    for (int64_t m = want; m > 1; m--) {
      const int64_t p = ((per + m - 1) / m) * m;
      if ((nblk + p - 1) / p == S) {
        M = m;
        per = p;
        break;
      }
    }
  }
  g.S = (int)S;
  g.Lc = per * blk;
  g.M = (int)M;
  g.Ls = g.Lc / M;
  g.nst = (int)((S - 1) * M);
  g.wsS = g.nst + 1;
  g.Ssub = g.wsS;
  return g;
}

// Workspace of a backward: the forward scan's chunk states (plan g) then
// the reverse scan's (plan gr).
size_t ws_bwd_bytes(const Geo &g, const Geo &gr, int d, int e) {
  auto one = [&](const Geo &x) {
    return x.S > 1 ? (size_t)x.B * x.H * x.wsS * d * e * sizeof(float) : (size_t)0;
  };
  return one(g) + one(gr);
}

// A tensor-core call with a 64-column head size keeps its initial and final
// states padded to 128 x 128 fp32 in scratch after the chunk states: n
// states per (b,h).
bool padded(Path p, int d, int e) { return p == PATH_TC && (d != 128 || e != 128); }
size_t pad_bytes(const Geo &g, int n) { return (size_t)g.B * g.H * 128 * 128 * sizeof(float) * n; }

size_t ws_bytes(int op, const Geo &g, int d, int e) {
  if (op == LA2_OP_DLAMBDA)  // (KV, W) per sub-chunk boundary
    return g.S > 1 ? (size_t)g.B * g.H * g.wsS * 2 * d * e * sizeof(float) : 0;
  if (op == LA2_OP_SHARD_STATE)  // one delta per sub-chunk plus one spare slot
    return (size_t)g.B * g.H * (g.Ssub + 1) * d * e * sizeof(float);
  if (g.S <= 1) return 0;
  size_t one = (size_t)g.B * g.H * g.wsS * d * e * sizeof(float);
  return op == LA2_OP_BACKWARD ? 2 * one : one;
}

// ------------------------------------------------------ SIMT dispatch
// A kernel's dynamic shared memory above the default 48 KB needs an opt-in
// attribute; its failure is returned rather than left to the launch.
template <typename K>
cudaError_t opt_in_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, int D, int E>
cudaError_t simt_forward(const void *q, const void *k, const void *v,
                         const float *lam, const float *kv0, void *o,
                         float *kv_out, float *ws, const Geo &g, cudaStream_t st) {
  using namespace la2::simt;
  const T *Q = (const T *)q, *K = (const T *)k, *V = (const T *)v;
  cudaError_t err = cudaSuccess;
  const int64_t BH = (int64_t)g.B * g.H;
  if (g.S > 1) {
    auto kst = fwd_kernel<T, D, E, false>;
    if (cudaError_t e = opt_in_smem(kst, fwd_smem<D, E>())) return e;
    err = timed(K_SIMT_FWD_STATE, st, [&] {
      kst<<<(unsigned)(BH * (g.S - 1)), NT, fwd_smem<D, E>(), st>>>(
          Q, K, V, lam, nullptr, nullptr, nullptr, ws, la2::state_geo(g, false));
    });
    if (err) return err;
    err = timed(K_SIMT_FWD_SCAN, st, [&] {
      scan_fwd_kernel<D, E><<<dim3((D * E + NT - 1) / NT, (unsigned)BH), NT, 0, st>>>(
          ws, kv0, lam, la2::state_geo(g, false));
    });
    if (err) return err;
  }
  auto kf = fwd_kernel<T, D, E, true>;
  if (cudaError_t e = opt_in_smem(kf, fwd_smem<D, E>())) return e;
  return timed(K_SIMT_FWD, st, [&] {
    kf<<<(unsigned)(BH * g.S), NT, fwd_smem<D, E>(), st>>>(Q, K, V, lam, kv0, (T *)o, kv_out, ws, g);
  });
}

template <typename T, int D, int E>
cudaError_t simt_backward(const void *q, const void *k, const void *v,
                          const float *lam, const float *kv0, const void *dO,
                          void *dq, void *dk, void *dv, float *dkv0, float *ws,
                          const Geo &g, bool reuse_fwd, cudaStream_t st,
                          const float *dend = nullptr) {
  using namespace la2::simt;
  const T *Q = (const T *)q, *K = (const T *)k, *V = (const T *)v, *G = (const T *)dO;
  const int64_t BH = (int64_t)g.B * g.H;
  float *wsf = ws;
  float *wsr = ws ? ws + (size_t)BH * g.wsS * D * E : nullptr;
  cudaError_t err = cudaSuccess;
  if (g.S > 1 && !reuse_fwd) {
    auto kst = fwd_kernel<T, D, E, false>;
    if (cudaError_t e = opt_in_smem(kst, fwd_smem<D, E>())) return e;
    err = timed(K_SIMT_FWD_STATE, st, [&] {
      kst<<<(unsigned)(BH * (g.S - 1)), NT, fwd_smem<D, E>(), st>>>(
          Q, K, V, lam, nullptr, nullptr, nullptr, wsf, la2::state_geo(g, false));
    });
    if (err) return err;
    err = timed(K_SIMT_FWD_SCAN, st, [&] {
      scan_fwd_kernel<D, E><<<dim3((D * E + NT - 1) / NT, (unsigned)BH), NT, 0, st>>>(
          wsf, kv0, lam, la2::state_geo(g, false));
    });
    if (err) return err;
  }
  if (g.S > 1) {
    auto krs = rev_state_kernel<T, D, E>;
    if (cudaError_t e = opt_in_smem(krs, rev_smem<D, E>())) return e;
    err = timed(K_SIMT_REV_STATE, st, [&] {
      krs<<<(unsigned)(BH * (g.S - 1)), NT, rev_smem<D, E>(), st>>>(Q, G, lam, wsr,
                                                                    la2::state_geo(g, true));
    });
    if (err) return err;
    err = timed(K_SIMT_REV_SCAN, st, [&] {
      scan_rev_kernel<D, E><<<dim3((D * E + NT - 1) / NT, (unsigned)BH), NT, 0, st>>>(
          wsr, lam, dend, la2::state_geo(g, true));
    });
    if (err) return err;
  }
  auto kq = dq_kernel<T, D, E>;
  if (cudaError_t e = opt_in_smem(kq, dq_smem<D, E>())) return e;
  err = timed(K_SIMT_DQ, st, [&] {
    kq<<<(unsigned)(BH * g.S), NT, dq_smem<D, E>(), st>>>(K, V, G, lam, kv0, (T *)dq, wsf, g);
  });
  if (err) return err;
  auto kk = dkdv_kernel<T, D, E>;
  if (cudaError_t e = opt_in_smem(kk, dkdv_smem<D, E>())) return e;
  return timed(K_SIMT_DKDV, st, [&] {
    kk<<<(unsigned)(BH * g.S), NT, dkdv_smem<D, E>(), st>>>(Q, K, V, G, lam, (T *)dk, (T *)dv,
                                                           dkv0, wsr, dend, g);
  });
}

template <typename T, int D, int E>
cudaError_t decode(const void *q, const void *k, const void *v, const float *lam,
                   float *pool, const int *slots, int pool_size, void *o, int B, int H,
                   int ntok, cudaStream_t st) {
  if (ntok == 1)
    return timed(K_DECODE, st, [&] {
      la2::dec::decode_kernel<T, D, E, 1><<<(unsigned)((int64_t)B * H), la2::dec::NT, 0, st>>>(
          (const T *)q, (const T *)k, (const T *)v, lam, pool, slots, pool_size, (T *)o, H, ntok);
    });
  auto kern = la2::dec::tokens_kernel<T, D, E, 4>;
  constexpr size_t smem = la2::dec::tokens_smem<E, 4>();
  if (cudaError_t e = opt_in_smem(kern, smem)) return e;
  return timed(K_DECODE, st, [&] {
    kern<<<(unsigned)((int64_t)B * H), la2::dec::NTT, smem, st>>>(
        (const T *)q, (const T *)k, (const T *)v, lam, pool, slots, pool_size, (T *)o, H, ntok);
  });
}

#define LA2_DISPATCH_DE(d, e, FN, T, ...)                                   \
  ((d) == 64 && (e) == 64     ? FN<T, 64, 64>(__VA_ARGS__)                  \
   : (d) == 64 && (e) == 128  ? FN<T, 64, 128>(__VA_ARGS__)                 \
   : (d) == 128 && (e) == 64  ? FN<T, 128, 64>(__VA_ARGS__)                 \
                              : FN<T, 128, 128>(__VA_ARGS__))

la2_status to_status(cudaError_t e) { return e == cudaSuccess ? LA2_OK : LA2_ERR_CUDA; }

}  // namespace

// Tokens per request from which la2_decode_tokens runs the tensor-core
// block form (one block of the chunk schedule per request) instead of the
// token-by-token register update.  Measured on B200 at batch 256 x 64 heads:
// the decode-unit kernel takes ~0.93 ms per call for any T <= 128 (148 CTAs,
// ~110 units each, set by each unit's state round trip), the token kernel
// 0.40 ms at T = 4, 0.50 at 8, 0.89 at 16 and 1.18 at 24 (~0.05 ms a token).
constexpr int kDecodeBlockTokens = 17;

// ------------------------------------------------------- d lambda helper
// dlam = 0; split: chunk-state pre-pass over the sub-chunks of chunks
// 0..S-2, the scan of the (KV, W) pairs, then the gradient pass over every
// chunk.
template <typename T, int D, int E>
cudaError_t simt_dlambda(const void *q, const void *k, const void *v, const void *dO,
                         const float *lam, const float *kv0, float *dlam, float *ws,
                         const Geo &g, cudaStream_t st) {
  using namespace la2::simt;
  auto kd = dlambda_kernel<T, D, E, false>;
  auto ks = dlambda_kernel<T, D, E, true>;
  cudaError_t e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)dlam_smem<T, D, E>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dlam_smem<T, D, E>());
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(dlam, 0, (size_t)g.H * sizeof(float), st);
  if (e != cudaSuccess) return e;
  const int64_t BH = (int64_t)g.B * g.H;
  const T *Q = (const T *)q, *K = (const T *)k, *V = (const T *)v, *G = (const T *)dO;
  if (g.S > 1) {
    e = timed(K_SIMT_DLAMBDA_STATE, st, [&] {
      ks<<<(unsigned)(BH * g.nst), NT, dlam_smem<T, D, E>(), st>>>(Q, K, V, G, lam, nullptr, ws,
                                                                  nullptr, g);
    });
    if (e != cudaSuccess) return e;
    e = timed(K_SIMT_DLAMBDA_SCAN, st, [&] {
      dlam_scan_kernel<D, E><<<dim3(D * E / NT, (unsigned)BH), NT, 0, st>>>(ws, kv0, lam, g);
    });
    if (e != cudaSuccess) return e;
  }
  return timed(K_SIMT_DLAMBDA, st, [&] {
    kd<<<(unsigned)(BH * g.S), NT, dlam_smem<T, D, E>(), st>>>(Q, K, V, G, lam, kv0, ws, dlam, g);
  });
}

// ------------------------------------------------------- shard helpers
template <typename T, int D, int E>
cudaError_t simt_shard_state(const void *a, const void *b, const float *lam, float *ws,
                             const Geo &gs, bool reverse, cudaStream_t st) {
  using namespace la2::simt;
  const int64_t BH = (int64_t)gs.B * gs.H;
  if (!reverse) {
    auto kst = fwd_kernel<T, D, E, false>;
    if (cudaError_t e = opt_in_smem(kst, fwd_smem<D, E>())) return e;
    return timed(K_SIMT_FWD_STATE, st, [&] {
      kst<<<(unsigned)(BH * gs.nst), NT, fwd_smem<D, E>(), st>>>(
          nullptr, (const T *)a, (const T *)b, lam, nullptr, nullptr, nullptr, ws, gs);
    });
  }
  auto krs = rev_state_kernel<T, D, E>;
  if (cudaError_t e = opt_in_smem(krs, rev_smem<D, E>())) return e;
  return timed(K_SIMT_REV_STATE, st, [&] {
    krs<<<(unsigned)(BH * gs.nst), NT, rev_smem<D, E>(), st>>>((const T *)a, (const T *)b, lam,
                                                              ws + (size_t)D * E, gs);
  });
}

template <typename T, int D, int E>
cudaError_t combine(const float *ws, const Geo &gs, const float *lam, bool reverse, float *out,
                    cudaStream_t st) {
  const int64_t BH = (int64_t)gs.B * gs.H;
  la2::shard::combine_kernel<D, E>
      <<<dim3((D * E + la2::shard::NT - 1) / la2::shard::NT, (unsigned)BH), la2::shard::NT, 0, st>>>(
          ws, gs.wsS, reverse ? 0 : 1, gs.nst, gs.Lc, gs.L, lam, gs.H, reverse ? 1 : 0, out);
  return cudaGetLastError();
}

template <typename T, int D, int E>
cudaError_t prefix(const float *delta, const float *kv0, const float *lam, int R, int B, int H,
                   int64_t Ls, bool reverse, float *out, cudaStream_t st) {
  const int64_t BH = (int64_t)B * H;
  la2::shard::prefix_kernel<D, E>
      <<<dim3((D * E + la2::shard::NT - 1) / la2::shard::NT, (unsigned)BH), la2::shard::NT, 0, st>>>(
          delta, kv0, lam, H, R, BH, Ls, reverse ? 1 : 0, out);
  return cudaGetLastError();
}


// ------------------------------------------------------------ feature map
namespace {

// The elementwise calls: tensor t's output may be exactly its own `own`
// input (in place); every other pair of arguments shares no byte.
bool fmap_args_ok(const std::vector<Span> &outs, const std::vector<Span> &ins,
                  const std::vector<const void *> &own) {
  for (size_t i = 0; i < outs.size(); i++) {
    if (!outs[i].p) continue;
    for (size_t j = 0; j < ins.size(); j++)
      if (overlaps(outs[i], ins[j]) && !(ins[j].p == outs[i].p && ins[j].p == own[i]))
        return false;
    for (size_t j = i + 1; j < outs.size(); j++)
      if (overlaps(outs[i], outs[j])) return false;
  }
  return true;
}

template <bool GRAD>
la2_status fmap_call(const void *q, const void *k, const void *gq, const void *gk, void *yq,
                     void *yk, int64_t n, la2_dtype dt, cudaStream_t stream) {
  if (n < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (n == 0) return LA2_OK;
  if (!q || !yq || (GRAD && !gq)) return LA2_ERR_INVALID;
  const bool has_k = k != nullptr;
  if ((yk != nullptr) != has_k || (GRAD && (gk != nullptr) != has_k)) return LA2_ERR_INVALID;
  for (const void *p : {q, k, gq, gk, (const void *)yq, (const void *)yk})
    if (p && !aligned16(p)) return LA2_ERR_INVALID;
  const size_t bytes = (size_t)n * esize(dt);
  std::vector<Span> ins = {{q, bytes}, {k, bytes}, {gq, bytes}, {gk, bytes}};
  std::vector<Span> outs = {{yq, bytes}, {yk, bytes}};
  // in place: the map over its input, the gradient over its upstream gradient
  if (!fmap_args_ok(outs, ins, {GRAD ? gq : q, GRAD ? gk : k})) return LA2_ERR_INVALID;
  const int sms = device_sms();
  const int grid = dt == LA2_F32 ? la2::fmap::grid_for<float, GRAD>(n, sms)
                                 : la2::fmap::grid_for<__nv_bfloat16, GRAD>(n, sms);
  cudaError_t err = timed(GRAD ? K_FMAP_GRAD : K_FMAP, stream, [&] {
    if (dt == LA2_F32)
      la2::fmap::enqueue<float, GRAD>(q, gq, yq, k, gk, yk, n, grid, stream);
    else
      la2::fmap::enqueue<__nv_bfloat16, GRAD>(q, gq, yq, k, gk, yk, n, grid, stream);
  });
  return to_status(err);
}

}  // namespace

extern "C" {

const char *la2_status_string(la2_status s) {
  switch (s) {
    case LA2_OK: return "LA2_OK";
    case LA2_ERR_INVALID: return "LA2_ERR_INVALID";
    case LA2_ERR_UNSUPPORTED: return "LA2_ERR_UNSUPPORTED";
    case LA2_ERR_CUDA: return "LA2_ERR_CUDA";
    case LA2_ERR_TIMEOUT: return "LA2_ERR_TIMEOUT";
  }
  return "LA2_ERR_UNKNOWN";
}

const char *la2_version(void) { return "la2 0.1 sm_100a"; }

int la2_set_option(int option, int value) {
  if (option == LA2_OPT_SPLIT) return g_opt_split.exchange(value);
  if (option == LA2_OPT_PATH) return g_opt_path.exchange(value);
  if (option == LA2_OPT_INJECT_TIMEOUT) return g_opt_inject.exchange(value);
  if (option == LA2_OPT_VARIANT) return g_opt_variant.exchange(value);
  if (option == LA2_OPT_TRACE) return g_opt_trace.exchange(value);
  if (option == LA2_OPT_VARLEN_ORDER) return g_opt_varlen_order.exchange(value);
  if (option == LA2_OPT_DECODE_BLOCK_TOKENS) return g_opt_decode_block.exchange(value);
  if (option == LA2_OPT_BWD_FORM) return g_opt_bwd_form.exchange(value);
  return -1;
}

size_t la2_workspace_size(int op, int B, int H, int64_t L, int d, int e, la2_dtype dt) {
  if (B <= 0 || H <= 0 || L <= 0 || !shape_supported(d, e, dt)) return 0;
  if (op == LA2_OP_DLAMBDA) {
    const Path p = choose_path(d, e, dt);
    if (p == PATH_NONE) return 0;
    return ws_bytes(op, plan_dlambda(B, H, L, true, block_rows(p)), d, e);
  }
  if (op != LA2_OP_FORWARD && op != LA2_OP_BACKWARD && op != LA2_OP_SHARD_STATE) return 0;
  Path p = choose_path(d, e, dt, op != LA2_OP_SHARD_STATE);
  if (p == PATH_NONE) return 0;
  Geo g = plan(B, H, L, block_rows(p), p);
  const int sd = p == PATH_TC ? 128 : d, se = p == PATH_TC ? 128 : e;  // state slot shape
  if (op == LA2_OP_BACKWARD)
    return ws_bwd_bytes(g, plan_rev(B, H, L, p), sd, se) + (padded(p, d, e) ? pad_bytes(g, 2) : 0);
  if (op == LA2_OP_FORWARD) return ws_bytes(op, g, sd, se) + (padded(p, d, e) ? pad_bytes(g, 2) : 0);
  return ws_bytes(op, g, d, e);
}

}  // extern "C"

namespace {

// The argument checks of la2_forward (and of la2_forward_noalloc, which
// passes no workspace).  LA2_OK with *empty set: B*H == 0, nothing to do.
la2_status forward_checks(const void *q, const void *k, const void *v, const float *lambda,
                          const float *kv0, const void *o, const float *kv_out, int B, int H,
                          int64_t L, int d, int e, la2_dtype dt, const void *workspace,
                          size_t workspace_bytes, bool *empty) {
  *empty = false;
  if (B < 0 || H < 0 || L < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  const size_t es = esize(dt);
  const size_t nq = (size_t)BH * L * d * es, nv = (size_t)BH * L * e * es;
  const size_t ns = (size_t)BH * d * e * sizeof(float);
  if (BH == 0) {
    *empty = true;
    return LA2_OK;
  }
  if (!lambda || (L > 0 && (!q || !k || !v || !o))) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{(const void *)q, (const void *)k, (const void *)v, (const void *)lambda,
                        (const void *)kv0, (const void *)o, (const void *)kv_out, workspace})
    if (p && !aligned16(p)) return LA2_ERR_INVALID;
  if (kv_out && kv_out == kv0) return LA2_ERR_INVALID;
  std::vector<Span> ins = {{q, nq}, {k, nq}, {v, nv}, {lambda, (size_t)H * 4}, {kv0, kv0 ? ns : 0}};
  std::vector<Span> outs = {{o, nv}, {kv_out, kv_out ? ns : 0}, {workspace, workspace_bytes}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  return LA2_OK;
}

}  // namespace

extern "C" {

la2_status la2_forward(const void *q, const void *k, const void *v,
                       const float *lambda, const float *kv0, void *o, float *kv_out,
                       int B, int H, int64_t L, int d, int e, la2_dtype dt,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  bool empty = false;
  const la2_status chk = forward_checks(q, k, v, lambda, kv0, o, kv_out, B, H, L, d, e, dt,
                                        workspace, workspace_bytes, &empty);
  if (chk != LA2_OK || empty) return chk;
  const int64_t BH = (int64_t)B * H;
  const size_t ns = (size_t)BH * d * e * sizeof(float);

  if (L == 0) {
    if (!kv_out) return LA2_OK;
    cudaError_t err = kv0 ? cudaMemcpyAsync(kv_out, kv0, ns, cudaMemcpyDeviceToDevice, stream)
                          : cudaMemsetAsync(kv_out, 0, ns, stream);
    return to_status(err);
  }
  Path p = choose_path(d, e, dt, true);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  Geo g = plan(B, H, L, block_rows(p), p);
  const bool pad = padded(p, d, e);
  const size_t states = ws_bytes(LA2_OP_FORWARD, g, p == PATH_TC ? 128 : d, p == PATH_TC ? 128 : e);
  const size_t need = states + (pad ? pad_bytes(g, 2) : 0);
  if (need > 0 && (!workspace || workspace_bytes < need)) return LA2_ERR_INVALID;
  float *ws = (float *)workspace;
  cudaError_t err;
  if (p == PATH_TC) {
    g.inject = g_opt_inject.exchange(0);
    g.d = d;
    g.e = e;
    // 64-column heads: the states in and out padded to 128 x 128
    float *scratch = pad ? reinterpret_cast<float *>(reinterpret_cast<char *>(workspace) + states)
                         : nullptr;
    const float *kv0_t = kv0;
    float *kv_out_t = kv_out;
    if (pad) {
      kv0_t = kv0 ? scratch : nullptr;
      kv_out_t = kv_out ? scratch + (size_t)BH * 128 * 128 : nullptr;
      if (kv0) {
        err = timed(K_STATE_PAD, stream, [&] { la2::tc::pad_states(kv0, scratch, BH, d, e, stream); });
        if (err != cudaSuccess) return to_status(err);
      }
    }
    err = la2::tc::forward(q, k, v, lambda, kv0_t, o, kv_out_t, ws, g, stream,
                           [&](int which, auto &&fn) {
                             return timed(which == 0 ? K_TC_FWD_STATE : which == 1 ? K_SCAN_FWD : K_TC_FWD,
                                          stream, fn);
                           });
    if (err == cudaSuccess && pad && kv_out)
      err = timed(K_STATE_PAD, stream,
                  [&] { la2::tc::unpad_states(kv_out_t, kv_out, BH, d, e, stream); });
  } else if (dt == LA2_F32) {
    err = LA2_DISPATCH_DE(d, e, simt_forward, float, q, k, v, lambda, kv0, o, kv_out, ws, g, stream);
  } else {
    err = LA2_DISPATCH_DE(d, e, simt_forward, __nv_bfloat16, q, k, v, lambda, kv0, o, kv_out, ws, g,
                          stream);
  }
  return to_status(err);
}

la2_status la2_backward(const void *q, const void *k, const void *v,
                        const float *lambda, const float *kv0, const void *dO,
                        void *dq, void *dk, void *dv, float *dkv0,
                        int B, int H, int64_t L, int d, int e, la2_dtype dt,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  return la2_backward_ex(q, k, v, lambda, kv0, dO, dq, dk, dv, dkv0, B, H, L, d, e, dt, workspace,
                         workspace_bytes, 0u, stream);
}

la2_status la2_backward_ex(const void *q, const void *k, const void *v,
                           const float *lambda, const float *kv0, const void *dO,
                           void *dq, void *dk, void *dv, float *dkv0,
                           int B, int H, int64_t L, int d, int e, la2_dtype dt,
                           void *workspace, size_t workspace_bytes, unsigned flags,
                           cudaStream_t stream) {
  if (flags & ~(unsigned)LA2_BWD_REUSE_FORWARD_STATES) return LA2_ERR_INVALID;
  const bool reuse = (flags & LA2_BWD_REUSE_FORWARD_STATES) != 0;
  if (B < 0 || H < 0 || L < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  const size_t es = esize(dt);
  const size_t nq = (size_t)BH * L * d * es, nv = (size_t)BH * L * e * es;
  const size_t ns = (size_t)BH * d * e * sizeof(float);
  if (BH == 0) return LA2_OK;
  if (!lambda || (L > 0 && (!q || !k || !v || !dO || !dq || !dk || !dv))) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{(const void *)q, (const void *)k, (const void *)v, (const void *)lambda,
                        (const void *)kv0, (const void *)dO, (const void *)dq, (const void *)dk,
                        (const void *)dv, (const void *)dkv0, workspace})
    if (p && !aligned16(p)) return LA2_ERR_INVALID;
  std::vector<Span> ins = {{q, nq}, {k, nq}, {v, nv}, {dO, nv}, {lambda, (size_t)H * 4},
                           {kv0, kv0 ? ns : 0}};
  std::vector<Span> outs = {{dq, nq}, {dk, nq}, {dv, nv}, {dkv0, dkv0 ? ns : 0},
                            {workspace, workspace_bytes}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;

  if (L == 0) {
    if (!dkv0) return LA2_OK;
    return to_status(cudaMemsetAsync(dkv0, 0, ns, stream));
  }
  Path p = choose_path(d, e, dt, true);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  Geo g = plan(B, H, L, block_rows(p), p);
  Geo gr = plan_rev(B, H, L, p);
  const bool pad = padded(p, d, e);
  const size_t states =
      ws_bwd_bytes(g, gr, p == PATH_TC ? 128 : d, p == PATH_TC ? 128 : e);
  const size_t need = states + (pad ? pad_bytes(g, 2) : 0);
  if (need > 0 && (!workspace || workspace_bytes < need)) return LA2_ERR_INVALID;
  float *ws = (float *)workspace;
  cudaError_t err;
  if (p == PATH_TC) {
    g.d = gr.d = d;
    g.e = gr.e = e;
    // 64-column heads: kv0 in and dkv0 out padded to 128 x 128
    float *scratch = pad ? reinterpret_cast<float *>(reinterpret_cast<char *>(workspace) + states)
                         : nullptr;
    const float *kv0_t = kv0;
    float *dkv0_t = dkv0;
    if (pad) {
      kv0_t = kv0 ? scratch : nullptr;
      dkv0_t = dkv0 ? scratch + (size_t)BH * 128 * 128 : nullptr;
      if (kv0) {
        err = timed(K_STATE_PAD, stream, [&] { la2::tc::pad_states(kv0, scratch, BH, d, e, stream); });
        if (err != cudaSuccess) return to_status(err);
      }
    }
    err = la2::tc::backward(q, k, v, lambda, kv0_t, dO, dq, dk, dv, dkv0_t, ws, g, gr, reuse, stream,
                            [&](int which, auto &&fn) {
                              static const int ids[] = {K_TC_FWD_STATE, K_SCAN_FWD, K_TC_DQ,
                                                        K_TC_REV_STATE, K_SCAN_REV, K_TC_DV,
                                                        K_TC_DK, K_TC_DKDV};
                              return timed(ids[which], stream, fn);
                            });
    if (err == cudaSuccess && pad && dkv0)
      err = timed(K_STATE_PAD, stream,
                  [&] { la2::tc::unpad_states(dkv0_t, dkv0, BH, d, e, stream); });
  } else if (dt == LA2_F32) {
    err = LA2_DISPATCH_DE(d, e, simt_backward, float, q, k, v, lambda, kv0, dO, dq, dk, dv, dkv0,
                          ws, g, reuse, stream);
  } else {
    err = LA2_DISPATCH_DE(d, e, simt_backward, __nv_bfloat16, q, k, v, lambda, kv0, dO, dq, dk,
                          dv, dkv0, ws, g, reuse, stream);
  }
  return to_status(err);
}

// ------------------------------------------------------- packed varlen
namespace {

// One CTA per (sequence, head) over the sequence's rows; no chunk split.
Geo plan_varlen(int N, int H, int64_t T, const int64_t *cu) {
  Geo g;
  g.B = N;
  g.H = H;
  g.L = T;
  g.S = 1;
  g.Lc = T;
  g.M = 1;
  g.Ls = T;
  g.Ssub = 1;
  g.wsS = 1;
  g.nst = 0;
  g.c0 = 0;
  g.cu = cu;
  g.lpt = N <= 64 && g_opt_varlen_order.load() == 0;
  g.slots = nullptr;
  g.pool = 0;
  g.inject = 0;
  g.variant = 0;  // the packed form exists in the warp-specialised kernel only
  g.trace = -1;
  return g;
}

// Shared argument checks of the packed entry points: sizes, null and
// alignment rules, and no output overlapping any argument.
la2_status check_varlen(int N, int H, int64_t T, int d, int e, la2_dtype dt, const int64_t *cu,
                        const float *lambda, std::vector<Span> ins, std::vector<Span> outs,
                        bool need_tensors) {
  if (N < 0 || H < 0 || T < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  if (!lambda || !cu || need_tensors) return LA2_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(cu) % 8 != 0) return LA2_ERR_INVALID;
  for (const Span &sp : ins)
    if (sp.p && sp.p != (const void *)cu && !aligned16(sp.p)) return LA2_ERR_INVALID;
  for (const Span &sp : outs)
    if (sp.p && !aligned16(sp.p)) return LA2_ERR_INVALID;
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  return LA2_OK;
}

}  // namespace

la2_status la2_forward_varlen(const void *q, const void *k, const void *v, const float *lambda,
                              const int64_t *cu_seqlens, const float *kv0, void *o,
                              float *kv_out, int N, int H, int64_t T, int d, int e,
                              la2_dtype dt, cudaStream_t stream) {
  if (N == 0 || H == 0) return (N < 0 || H < 0 || T < 0) ? LA2_ERR_INVALID : LA2_OK;
  const size_t es = (dt == LA2_F32 || dt == LA2_BF16) ? esize(dt) : 0;
  const size_t nq = (size_t)H * T * d * es, nv = (size_t)H * T * e * es;
  const size_t ns = (size_t)N * H * d * e * sizeof(float);
  if (kv_out && kv_out == kv0) return LA2_ERR_INVALID;
  la2_status st = check_varlen(
      N, H, T, d, e, dt, cu_seqlens, lambda,
      {{q, nq}, {k, nq}, {v, nv}, {lambda, (size_t)H * 4}, {kv0, kv0 ? ns : 0},
       {cu_seqlens, (size_t)(N + 1) * 8}},
      {{o, nv}, {kv_out, kv_out ? ns : 0}}, T > 0 && (!q || !k || !v || !o));
  if (st != LA2_OK) return st;
  if (T == 0) {  // every sequence is empty
    if (!kv_out) return LA2_OK;
    return to_status(kv0 ? cudaMemcpyAsync(kv_out, kv0, ns, cudaMemcpyDeviceToDevice, stream)
                         : cudaMemsetAsync(kv_out, 0, ns, stream));
  }
  Path p = choose_path(d, e, dt);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  Geo g = plan_varlen(N, H, T, cu_seqlens);
  cudaError_t err;
  if (p == PATH_TC) {
    err = la2::tc::forward_varlen(q, k, v, lambda, kv0, o, kv_out, g, stream,
                                  [&](int, auto &&fn) { return timed(K_TC_FWD, stream, fn); });
  } else if (dt == LA2_F32) {
    err = LA2_DISPATCH_DE(d, e, simt_forward, float, q, k, v, lambda, kv0, o, kv_out, nullptr, g,
                          stream);
  } else {
    err = LA2_DISPATCH_DE(d, e, simt_forward, __nv_bfloat16, q, k, v, lambda, kv0, o, kv_out,
                          nullptr, g, stream);
  }
  return to_status(err);
}

la2_status la2_backward_varlen(const void *q, const void *k, const void *v, const float *lambda,
                               const int64_t *cu_seqlens, const float *kv0, const void *dO,
                               void *dq, void *dk, void *dv, float *dkv0, int N, int H,
                               int64_t T, int d, int e, la2_dtype dt, cudaStream_t stream) {
  if (N == 0 || H == 0) return (N < 0 || H < 0 || T < 0) ? LA2_ERR_INVALID : LA2_OK;
  const size_t es = (dt == LA2_F32 || dt == LA2_BF16) ? esize(dt) : 0;
  const size_t nq = (size_t)H * T * d * es, nv = (size_t)H * T * e * es;
  const size_t ns = (size_t)N * H * d * e * sizeof(float);
  la2_status st = check_varlen(
      N, H, T, d, e, dt, cu_seqlens, lambda,
      {{q, nq}, {k, nq}, {v, nv}, {dO, nv}, {lambda, (size_t)H * 4}, {kv0, kv0 ? ns : 0},
       {cu_seqlens, (size_t)(N + 1) * 8}},
      {{dq, nq}, {dk, nq}, {dv, nv}, {dkv0, dkv0 ? ns : 0}},
      T > 0 && (!q || !k || !v || !dO || !dq || !dk || !dv));
  if (st != LA2_OK) return st;
  if (T == 0) return dkv0 ? to_status(cudaMemsetAsync(dkv0, 0, ns, stream)) : LA2_OK;
  Path p = choose_path(d, e, dt);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  Geo g = plan_varlen(N, H, T, cu_seqlens);
  g.rev_pair = p == PATH_TC && g_opt_bwd_form.load() != 1;
  cudaError_t err;
  if (p == PATH_TC) {
    err = la2::tc::backward_varlen(q, k, v, lambda, kv0, dO, dq, dk, dv, dkv0, g, stream,
                                   [&](int which, auto &&fn) {
                                     return timed(which == 2   ? K_TC_DQ
                                                  : which == 5 ? K_TC_DV
                                                  : which == 6 ? K_TC_DK
                                                               : K_TC_DKDV,
                                                  stream, fn);
                                   });
  } else if (dt == LA2_F32) {
    err = LA2_DISPATCH_DE(d, e, simt_backward, float, q, k, v, lambda, kv0, dO, dq, dk, dv, dkv0,
                          nullptr, g, false, stream);
  } else {
    err = LA2_DISPATCH_DE(d, e, simt_backward, __nv_bfloat16, q, k, v, lambda, kv0, dO, dq, dk,
                          dv, dkv0, nullptr, g, false, stream);
  }
  return to_status(err);
}

la2_status la2_forward_pool(const void *q, const void *k, const void *v, const float *lambda,
                            float *kv_pool, const int32_t *slots, int pool_size, void *o,
                            unsigned flags, int B, int H, int64_t L, int d, int e, la2_dtype dt,
                            void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (flags & ~(unsigned)LA2_POOL_CONTINUE) return LA2_ERR_INVALID;
  if (B < 0 || H < 0 || L < 1 || pool_size < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (BH == 0) return LA2_OK;
  if (!q || !k || !v || !lambda || !kv_pool || !slots || !o) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{
           (const void *)q, (const void *)k, (const void *)v, (const void *)lambda,
           (const void *)kv_pool, (const void *)o, workspace})
    if (p && !aligned16(p)) return LA2_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(slots) % 4 != 0) return LA2_ERR_INVALID;
  const size_t es = esize(dt);
  const size_t nq = (size_t)BH * L * d * es, nv = (size_t)BH * L * e * es;
  std::vector<Span> ins = {{q, nq}, {k, nq}, {v, nv}, {lambda, (size_t)H * 4},
                           {slots, (size_t)B * 4}};
  std::vector<Span> outs = {{o, nv},
                            {kv_pool, (size_t)pool_size * H * d * e * sizeof(float)},
                            {workspace, workspace_bytes}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  Path p = choose_path(d, e, dt);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  Geo g = plan(B, H, L, block_rows(p), p);
  g.slots = slots;
  g.pool = pool_size;
  g.variant = 0;  // the slot table exists in the warp-specialised kernel only
  const size_t need = ws_bytes(LA2_OP_FORWARD, g, d, e);
  if (need > 0 && (!workspace || workspace_bytes < need)) return LA2_ERR_INVALID;
  float *ws = (float *)workspace;
  const float *kv0 = (flags & LA2_POOL_CONTINUE) ? kv_pool : nullptr;
  cudaError_t err;
  if (p == PATH_TC) {
    err = la2::tc::forward(q, k, v, lambda, kv0, o, kv_pool, ws, g, stream,
                           [&](int which, auto &&fn) {
                             return timed(which == 0 ? K_TC_FWD_STATE : which == 1 ? K_SCAN_FWD : K_TC_FWD,
                                          stream, fn);
                           });
  } else if (dt == LA2_F32) {
    err = LA2_DISPATCH_DE(d, e, simt_forward, float, q, k, v, lambda, kv0, o, kv_pool, ws, g,
                          stream);
  } else {
    err = LA2_DISPATCH_DE(d, e, simt_forward, __nv_bfloat16, q, k, v, lambda, kv0, o, kv_pool,
                          ws, g, stream);
  }
  return to_status(err);
}

// ------------------------------------------------------------ shards
namespace {

// The chunk-state passes over every sub-chunk of one shard.
Geo shard_geo(const Geo &g) {
  Geo s = g;
  s.S = g.Ssub;
  s.Lc = g.Ls;
  s.M = 1;
  s.nst = g.Ssub;
  s.c0 = 0;
  s.wsS = g.Ssub + 1;
  s.variant = 0;
  return s;
}

}  // namespace

la2_status la2_shard_state(const void *a, const void *b, const float *lambda, float *out,
                           int B, int H, int64_t L, int d, int e, la2_dtype dt, int reverse,
                           void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || H < 0 || L < 1) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (BH == 0) return LA2_OK;
  if (!a || !b || !lambda || !out || !workspace) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{a, b, (const void *)lambda,
                                                          (const void *)out, workspace})
    if (!aligned16(p)) return LA2_ERR_INVALID;
  const size_t es = esize(dt);
  std::vector<Span> ins = {{a, (size_t)BH * L * d * es}, {b, (size_t)BH * L * e * es},
                           {lambda, (size_t)H * 4}};
  std::vector<Span> outs = {{out, (size_t)BH * d * e * 4}, {workspace, workspace_bytes}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  Path p = choose_path(d, e, dt);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  const Geo g = plan(B, H, L, block_rows(p), p);
  if (workspace_bytes < ws_bytes(LA2_OP_SHARD_STATE, g, d, e)) return LA2_ERR_INVALID;
  const Geo gs = shard_geo(g);
  float *ws = (float *)workspace;
  cudaError_t err;
  if (p == PATH_TC) {
    err = la2::tc::shard_state(a, b, lambda, ws, gs, reverse != 0, stream,
                               [&](int which, auto &&fn) {
                                 return timed(which == 0 ? K_TC_FWD_STATE : K_TC_REV_STATE, stream, fn);
                               });
  } else if (dt == LA2_F32) {
    err = LA2_DISPATCH_DE(d, e, simt_shard_state, float, a, b, lambda, ws, gs, reverse != 0, stream);
  } else {
    err = LA2_DISPATCH_DE(d, e, simt_shard_state, __nv_bfloat16, a, b, lambda, ws, gs, reverse != 0,
                          stream);
  }
  if (err == cudaSuccess)
    err = LA2_DISPATCH_DE(d, e, combine, float, ws, gs, lambda, reverse != 0, out, stream);
  return to_status(err);
}

la2_status la2_state_prefix(const float *delta, const float *kv0, const float *lambda,
                            float *out, int R, int B, int H, int64_t L_shard, int d, int e,
                            int reverse, cudaStream_t stream) {
  if (R < 0 || B < 0 || H < 0 || L_shard < 0) return LA2_ERR_INVALID;
  if (!shape_supported(d, e, LA2_F32)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (BH == 0 || R == 0) return LA2_OK;
  if (!delta || !lambda || !out) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{(const void *)delta, (const void *)kv0,
                                                          (const void *)lambda, (const void *)out})
    if (p && !aligned16(p)) return LA2_ERR_INVALID;
  const size_t all_states = (size_t)R * BH * d * e * 4;
  std::vector<Span> ins = {{delta, all_states}, {kv0, kv0 ? (size_t)BH * d * e * 4 : 0},
                           {lambda, (size_t)H * 4}};
  std::vector<Span> outs = {{out, all_states}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  return to_status(LA2_DISPATCH_DE(d, e, prefix, float, delta, reverse ? nullptr : kv0, lambda, R,
                                   B, H, L_shard, reverse != 0, out, stream));
}

la2_status la2_backward_shard(const void *q, const void *k, const void *v, const float *lambda,
                              const float *kv0, const void *dO, const float *dstate_end,
                              void *dq, void *dk, void *dv, float *dkv0, int B, int H,
                              int64_t L, int d, int e, la2_dtype dt, void *workspace,
                              size_t workspace_bytes, unsigned flags, cudaStream_t stream) {
  if (flags & ~(unsigned)LA2_BWD_REUSE_FORWARD_STATES) return LA2_ERR_INVALID;
  const bool reuse = (flags & LA2_BWD_REUSE_FORWARD_STATES) != 0;
  if (B < 0 || H < 0 || L < 1) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (BH == 0) return LA2_OK;
  const size_t es = esize(dt);
  const size_t nq = (size_t)BH * L * d * es, nv = (size_t)BH * L * e * es;
  const size_t ns = (size_t)BH * d * e * sizeof(float);
  if (!lambda || !q || !k || !v || !dO || !dq || !dk || !dv) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{
           (const void *)q, (const void *)k, (const void *)v, (const void *)lambda,
           (const void *)kv0, (const void *)dO, (const void *)dstate_end, (const void *)dq,
           (const void *)dk, (const void *)dv, (const void *)dkv0, workspace})
    if (p && !aligned16(p)) return LA2_ERR_INVALID;
  std::vector<Span> ins = {{q, nq}, {k, nq}, {v, nv}, {dO, nv}, {lambda, (size_t)H * 4},
                           {kv0, kv0 ? ns : 0}, {dstate_end, dstate_end ? ns : 0}};
  std::vector<Span> outs = {{dq, nq}, {dk, nq}, {dv, nv}, {dkv0, dkv0 ? ns : 0},
                            {workspace, workspace_bytes}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  Path p = choose_path(d, e, dt);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  Geo g = plan(B, H, L, block_rows(p), p);
  const Geo gr = plan_rev(B, H, L, p);
  const size_t need = ws_bwd_bytes(g, gr, d, e);
  if (need > 0 && (!workspace || workspace_bytes < need)) return LA2_ERR_INVALID;
  float *ws = (float *)workspace;
  cudaError_t err;
  if (p == PATH_TC) {
    err = la2::tc::backward(q, k, v, lambda, kv0, dO, dq, dk, dv, dkv0, ws, g, gr, reuse, stream,
                            [&](int which, auto &&fn) {
                              static const int ids[] = {K_TC_FWD_STATE, K_SCAN_FWD, K_TC_DQ,
                                                        K_TC_REV_STATE, K_SCAN_REV, K_TC_DV,
                                                        K_TC_DK, K_TC_DKDV};
                              return timed(ids[which], stream, fn);
                            },
                            dstate_end);
  } else if (dt == LA2_F32) {
    err = LA2_DISPATCH_DE(d, e, simt_backward, float, q, k, v, lambda, kv0, dO, dq, dk, dv, dkv0,
                          ws, g, reuse, stream, dstate_end);
  } else {
    err = LA2_DISPATCH_DE(d, e, simt_backward, __nv_bfloat16, q, k, v, lambda, kv0, dO, dq, dk,
                          dv, dkv0, ws, g, reuse, stream, dstate_end);
  }
  return to_status(err);
}

namespace {
// split: chunk the sequences as la2_workspace_size(LA2_OP_DLAMBDA) planned
// (the workspace must then hold that much); otherwise one chunk per (b,h).
la2_status dlambda_call(const void *q, const void *k, const void *v, const float *lambda,
                        const float *kv0, const void *dO, float *dlambda, int B, int H,
                        int64_t L, int d, int e, la2_dtype dt, void *workspace,
                        size_t workspace_bytes, bool split, cudaStream_t stream) {
  if (B < 0 || H < 0 || L < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (H == 0) return LA2_OK;
  if (!lambda || !dlambda || (BH > 0 && L > 0 && (!q || !k || !v || !dO))) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{
           (const void *)q, (const void *)k, (const void *)v, (const void *)lambda,
           (const void *)kv0, (const void *)dO, (const void *)dlambda, workspace})
    if (p && !aligned16(p)) return LA2_ERR_INVALID;
  const size_t es = esize(dt);
  const size_t nq = (size_t)BH * L * d * es, nv = (size_t)BH * L * e * es;
  std::vector<Span> ins = {{q, nq}, {k, nq}, {v, nv}, {dO, nv}, {lambda, (size_t)H * 4},
                           {kv0, kv0 ? (size_t)BH * d * e * 4 : 0}};
  std::vector<Span> outs = {{dlambda, (size_t)H * 4}, {workspace, workspace ? workspace_bytes : 0}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  if (BH == 0 || L == 0) {  // no token depends on lambda
    return to_status(cudaMemsetAsync(dlambda, 0, (size_t)H * sizeof(float), stream));
  }
  const Path p = choose_path(d, e, dt);
  if (p == PATH_NONE) return LA2_ERR_UNSUPPORTED;
  const Geo g = plan_dlambda(B, H, L, split, block_rows(p));
  const size_t need = ws_bytes(LA2_OP_DLAMBDA, g, d, e);
  if (need > 0 && (!workspace || workspace_bytes < need)) return LA2_ERR_INVALID;
  float *ws = (float *)workspace;
  if (p == PATH_TC)
    return to_status(la2::tcd::dlambda(q, k, v, dO, lambda, kv0, dlambda, ws, g, stream,
                                       [&](int which, auto &&fn) {
                                         static const int ids[] = {K_TC_DLAMBDA_STATE,
                                                                   K_SIMT_DLAMBDA_SCAN,
                                                                   K_TC_DLAMBDA};
                                         return timed(ids[which], stream, fn);
                                       }));
  cudaError_t err =
      dt == LA2_F32
          ? LA2_DISPATCH_DE(d, e, simt_dlambda, float, q, k, v, dO, lambda, kv0, dlambda, ws, g,
                            stream)
          : LA2_DISPATCH_DE(d, e, simt_dlambda, __nv_bfloat16, q, k, v, dO, lambda, kv0, dlambda,
                            ws, g, stream);
  return to_status(err);
}
}  // namespace

la2_status la2_backward_dlambda(const void *q, const void *k, const void *v,
                                const float *lambda, const float *kv0, const void *dO,
                                float *dlambda, int B, int H, int64_t L, int d, int e,
                                la2_dtype dt, cudaStream_t stream) {
  return dlambda_call(q, k, v, lambda, kv0, dO, dlambda, B, H, L, d, e, dt, nullptr, 0, false,
                      stream);
}

la2_status la2_backward_dlambda_ex(const void *q, const void *k, const void *v,
                                   const float *lambda, const float *kv0, const void *dO,
                                   float *dlambda, int B, int H, int64_t L, int d, int e,
                                   la2_dtype dt, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
  return dlambda_call(q, k, v, lambda, kv0, dO, dlambda, B, H, L, d, e, dt, workspace,
                      workspace_bytes, true, stream);
}

la2_status la2_decode_step(const void *q, const void *k, const void *v, const float *lambda,
                           float *kv, void *o, int B, int H, int d, int e, la2_dtype dt,
                           cudaStream_t stream) {
  if (B < 0 || H < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (BH == 0) return LA2_OK;
  if (!q || !k || !v || !lambda || !kv || !o) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{(const void *)q, (const void *)k, (const void *)v, (const void *)lambda,
                        (const void *)kv, (const void *)o})
    if (!aligned16(p)) return LA2_ERR_INVALID;
  const size_t es = esize(dt);
  std::vector<Span> ins = {{q, BH * d * es}, {k, BH * d * es}, {v, BH * e * es},
                           {lambda, (size_t)H * 4}};
  std::vector<Span> outs = {{kv, BH * d * e * sizeof(float)}, {o, BH * e * es}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  cudaError_t err =
      dt == LA2_F32
          ? LA2_DISPATCH_DE(d, e, decode, float, q, k, v, lambda, kv, nullptr, B, o, B, H, 1, stream)
          : LA2_DISPATCH_DE(d, e, decode, __nv_bfloat16, q, k, v, lambda, kv, nullptr, B, o, B, H,
                            1, stream);
  return to_status(err);
}

la2_status la2_feature_map(const void *q, const void *k, void *phi_q, void *phi_k, int64_t n,
                           la2_dtype dt, cudaStream_t stream) {
  return fmap_call<false>(q, k, nullptr, nullptr, phi_q, phi_k, n, dt, stream);
}

la2_status la2_feature_map_backward(const void *q, const void *k, const void *dphi_q,
                                    const void *dphi_k, void *dq, void *dk, int64_t n,
                                    la2_dtype dt, cudaStream_t stream) {
  return fmap_call<true>(q, k, dphi_q, dphi_k, dq, dk, n, dt, stream);
}

la2_status la2_decode_tokens(const void *q, const void *k, const void *v, const float *lambda,
                             float *kv_pool, const int32_t *slots, int pool_size, void *o,
                             int B, int H, int T, int d, int e, la2_dtype dt,
                             cudaStream_t stream) {
  if (B < 0 || H < 0 || T < 0 || pool_size < 0) return LA2_ERR_INVALID;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_UNSUPPORTED;
  if (!shape_supported(d, e, dt)) return LA2_ERR_UNSUPPORTED;
  const int64_t BH = (int64_t)B * H;
  if (BH == 0 || T == 0) return LA2_OK;
  if (!slots && pool_size < B) return LA2_ERR_INVALID;
  if (!q || !k || !v || !lambda || !kv_pool || !o) return LA2_ERR_INVALID;
  for (const void *p : std::initializer_list<const void *>{
           (const void *)q, (const void *)k, (const void *)v, (const void *)lambda,
           (const void *)kv_pool, (const void *)o})
    if (!aligned16(p)) return LA2_ERR_INVALID;
  if (slots && reinterpret_cast<uintptr_t>(slots) % 4 != 0) return LA2_ERR_INVALID;
  const size_t es = esize(dt);
  std::vector<Span> ins = {{q, BH * T * d * es}, {k, BH * T * d * es}, {v, BH * T * e * es},
                           {lambda, (size_t)H * 4}, {slots, slots ? (size_t)B * 4 : 0}};
  std::vector<Span> outs = {{kv_pool, (size_t)pool_size * H * d * e * sizeof(float)},
                            {o, BH * T * e * es}};
  if (any_overlap(outs, ins)) return LA2_ERR_INVALID;
  // From kDecodeBlockTokens tokens per request on, one block of the chunk
  // schedule (tensor cores, the state read and written once per call) beats
  // the token-by-token register update; the [B,H,T,.] layout is the
  // forward's.
  const int from = g_opt_decode_block.load() > 0 ? g_opt_decode_block.load() : kDecodeBlockTokens;
  if (T >= from && choose_path(d, e, dt) == PATH_TC) {
    Geo g = plan(B, H, T, block_rows(PATH_TC), PATH_TC);
    g.slots = slots;
    g.pool = pool_size;
    g.variant = 0;
    // up to one block per request: one CTA per SM walks (request, head)
    // units back to back (a range of units spans at most two heads)
    const int64_t P = BH < device_sms() ? BH : device_sms();
    if (T <= la2::tc::BLOCK && (BH + P - 1) / P <= B) {
      g.L = T;
      return to_status(la2::tc::decode_units(q, k, v, lambda, kv_pool, o, g, (int)P, stream,
                                             [&](int, auto &&fn) { return timed(K_TC_DECODE_UNITS, stream, fn); }));
    }
    g.S = 1;  // one chunk per request: no workspace
    g.Lc = g.Ls = T;
    g.M = g.Ssub = g.wsS = 1;
    g.nst = 0;
    return to_status(la2::tc::forward(q, k, v, lambda, kv_pool, o, kv_pool, nullptr, g, stream,
                                      [&](int, auto &&fn) { return timed(K_TC_FWD, stream, fn); }));
  }
  cudaError_t err =
      dt == LA2_F32 ? LA2_DISPATCH_DE(d, e, decode, float, q, k, v, lambda, kv_pool, slots,
                                      pool_size, o, B, H, T, stream)
                    : LA2_DISPATCH_DE(d, e, decode, __nv_bfloat16, q, k, v, lambda, kv_pool, slots,
                                      pool_size, o, B, H, T, stream);
  return to_status(err);
}

la2_status la2_last_device_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return LA2_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, la2::g_error_word, sizeof(word)) != cudaSuccess)
    return LA2_ERR_CUDA;
  if (word && cudaMemcpyToSymbol(la2::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return LA2_ERR_CUDA;
  if (word & la2::ERR_TIMEOUT) return LA2_ERR_TIMEOUT;
  if (word & la2::ERR_BOUNDS) return LA2_ERR_INVALID;  // e.g. bad varlen offsets
  if (word) return LA2_ERR_CUDA;
  return LA2_OK;
}

size_t la2_trace_read(uint64_t *out, size_t n) {
  const size_t total = (size_t)la2::kTraceEvents * la2::kTraceBlocks;
  if (!out || n == 0) return total;
  if (cudaDeviceSynchronize() != cudaSuccess) return 0;
  const size_t m = n < total ? n : total;
  if (cudaMemcpyFromSymbol(out, la2::g_trace, m * sizeof(uint64_t)) != cudaSuccess) return 0;
  static const unsigned long long zeros[la2::kTraceEvents * la2::kTraceBlocks] = {0};
  cudaMemcpyToSymbol(la2::g_trace, zeros, sizeof(zeros));
  return m;
}

void la2_profile_enable(int on) { g_prof_on.store(on ? 1 : 0); }

size_t la2_profile_report(char *buf, size_t buf_bytes) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  double ms[K_COUNT] = {0};
  long n[K_COUNT] = {0};
  for (auto &r : g_prof) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess) {
      ms[r.kid] += t;
      n[r.kid] += 1;
    }
    g_ev_pool.push_back(r.a);
    g_ev_pool.push_back(r.b);
  }
  g_prof.clear();
  std::string s = "{";
  bool first = true;
  for (int i = 0; i < K_COUNT; i++) {
    if (!n[i]) continue;
    char tmp[160];
    snprintf(tmp, sizeof(tmp), "%s\"%s\": {\"launches\": %ld, \"ms\": %.6f}", first ? "" : ", ",
             kKernelName[i], n[i], ms[i]);
    s += tmp;
    first = false;
  }
  s += "}";
  if (buf && buf_bytes) {
    size_t m = s.size() < buf_bytes - 1 ? s.size() : buf_bytes - 1;
    memcpy(buf, s.data(), m);
    buf[m] = 0;
  }
  return s.size() + 1;
}

}  // extern "C"

// ------------------------------------------------------------------------
// Forward pass for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: plug-ins
// whose host framework owns every byte of device memory through its own
// allocator, latency-critical code paths where cudaMalloc's implicit device
// synchronisation would stall other streams, and callbacks that receive only
// device pointers and have no allocator at hand.  For them la2_forward_noalloc
// takes the chunk-boundary states from the fixed array below instead of a
// caller-provided workspace.  The array is part of the library's device
// image: every GPU that loads the library holds it until the process exits.
namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device; looked up once per
// device (host code cannot use the array's name as a device address).
void *noalloc_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" la2_status la2_forward_noalloc(const void *q, const void *k, const void *v,
                                          const float *lambda, const float *kv0, void *o,
                                          float *kv_out, int B, int H, int64_t L, int d, int e,
                                          la2_dtype dt, cudaStream_t stream) {
  // la2_forward's argument checks first: a call it would refuse touches
  // neither the device nor the array.
  bool empty = false;
  const la2_status chk = forward_checks(q, k, v, lambda, kv0, o, kv_out, B, H, L, d, e, dt,
                                        nullptr, 0, &empty);
  if (chk != LA2_OK || empty) return chk;
  // Same plan as la2_forward; refuse plans whose scratch exceeds the array.
  if (L > 0 && la2_workspace_size(LA2_OP_FORWARD, B, H, L, d, e, dt) > kNoallocScratchBytes)
    return LA2_ERR_UNSUPPORTED;
  void *scratch = noalloc_scratch_ptr();
  if (!scratch) return LA2_ERR_CUDA;
  return la2_forward(q, k, v, lambda, kv0, o, kv_out, B, H, L, d, e, dt, scratch,
                     kNoallocScratchBytes, stream);
}
