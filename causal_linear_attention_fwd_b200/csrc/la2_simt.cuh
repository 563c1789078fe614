// la2_simt.cuh -- portable fp32-FMA kernels for every supported shape.
//
// These kernels are the fp32 I/O path (fp32 FMA keeps the 1e-4 accuracy that
// tf32 tensor-core products would miss) and the path for head sizes the
// tensor-core kernels do not cover.  They follow the same block schedule as
// the tensor-core kernels -- intra-block masked dense part plus inter-block
// part through a carried d x e state (Lightning Attention-2 notes page,
// "Tiling." paragraph) -- with a smaller block (C = 32 rows) and all tiles in
// shared memory as fp32.
//
// Per (b,h) the sequence is cut into S chunks of Lc rows (Lc a multiple of the
// block size); chunks run in parallel CTAs.  Chunk entry states come from a
// pre-pass (the chunk's own state contribution, started from zero) and a
// short scan over chunks:  KV_in[c] = lambda^Lc KV_in[c-1] + dKV[c-1].
//
// Block i covers rows [p, p+cb), local rows s, t in [0, cb):
//   forward  O_i = (Q_i K_i^T (.) M) V_i + diag(lambda^(s+1)) Q_i KV
//            KV <- lambda^cb KV + (diag(lambda^(cb-1-t)) K_i)^T V_i
//   dQ       dQ_i = (dO_i V_i^T (.) M) K_i + diag(lambda^(s+1)) dO_i KV^T
//   dK, dV   (reverse scan over D = sum_{t beyond the block} lambda^.. q_t^T dO_t)
//            dK_i = (dO_i V_i^T (.) M)^T Q_i + diag(lambda^(cb-s)) V_i D^T
//            dV_i = (Q_i K_i^T (.) M)^T dO_i + diag(lambda^(cb-s)) K_i D
//            D <- lambda^cb D + (diag(lambda^s) Q_i)^T dO_i
// with M[s,t] = lambda^(s-t) for t <= s.
#pragma once

#include "la2_common.cuh"

namespace la2 {

struct Geo {
  int B, H;
  int64_t L;
  int S;        // chunks per (b,h)
  int64_t Lc;   // rows per chunk (multiple of the block size); last may be short
  // The chunk-state pre-passes may run on a finer split: M sub-chunks of Ls
  // rows per chunk (Lc = M * Ls), Ssub of them over the sequence, so that
  // they fill the GPU too.  The workspace holds wsS d x e states per (b,h)
  // (one per sub-chunk); a chunk-state pass processes nst (sub-)chunks
  // starting at index c0.  M = 1 is the plain split.
  int M;
  int64_t Ls;
  int Ssub;
  int wsS;
  int nst;
  int c0;
  // Packed variable-length batch (NULL otherwise): B = N sequences, sequence
  // n owning rows [cu[n], cu[n+1]) of every head's slab of L rows; tensors
  // are [H, L, d|e], states [N, H, d, e]; S = 1.
  const int64_t *cu;
  // Packed batch of at most 64 sequences: the tensor-core passes take the
  // sequences longest first (list scheduling of unequal CTAs), see
  // lpt_sequence.
  int lpt;
  // State pool (NULL otherwise): the initial / final state of (b,h) is
  // pool state slots[b] * H + h of the kv0 / kv_out arrays, [pool, H, d, e];
  // a negative slot means none (zero initial state, final state dropped).
  const int *slots;
  int pool;
  int inject;   // test hook: CTA 0 of a tensor-core pass withholds one MMA
                // completion signal so that its bounded wait runs out
  int variant;  // tensor-core kernel form (0: warp-specialised, 1: phase-serial)
  int trace;    // tensor-core pass whose CTA 0 stamps the trace buffer (-1: none)
  int rev_pair = 0;  // tensor-core backward: dV and dK as one paired launch
  // tensor-core passes: the head sizes of the tensors (64 or 128; the
  // kernels work on 128 columns, a 64-column tensor read with zeros beyond
  // its width and its states padded to 128 x 128 by the caller)
  int d = 128, e = 128;
};

// What one CTA of a pass works on: state slot bh (the (b,h) or (sequence,
// head) index), slab (the outer index of the [.., L, d] tensors), rows
// [a, b) of that slab, head h and chunk c.  A varlen range that is not
// inside the slab is recorded as a bounds error and treated as empty.
struct Span {
  int64_t bh, slab, a, b;
  int h, c;
};
// seq >= 0 (packed batch, one CTA per (sequence, head)): the CTA serves that
// sequence and head cta % H instead of its own index's sequence.  cta: the
// CTA's index in the pass (blockIdx.x unless several CTAs share a work
// unit, as the two of a cluster in the paired reverse pass do).
__device__ __forceinline__ Span span_of(const Geo &g, int nch, int c_first, int64_t seq = -1,
                                        int64_t cta = -1) {
  Span s;
  if (cta < 0) cta = blockIdx.x;
  const int64_t q = seq >= 0 ? seq * g.H + cta % g.H : cta / nch;
  s.bh = q;
  s.h = (int)(q % g.H);
  s.c = (int)(cta % nch) + c_first;
  if (g.cu) {
    int64_t lo = g.cu[q / g.H], hi = g.cu[q / g.H + 1];
    if (!(0 <= lo && lo <= hi && hi <= g.L)) {
      if (threadIdx.x == 0) raise_error(ERR_BOUNDS);
      lo = hi = 0;
    }
    s.slab = s.h;
    s.a = lo;
    s.b = hi;
  } else {
    s.slab = q;
    s.a = (int64_t)s.c * g.Lc;
    s.b = g.L < s.a + g.Lc ? g.L : s.a + g.Lc;
  }
  return s;
}

// Longest-first order of a packed batch of N <= 64 sequences (ties in index
// order), computed by one warp from the offsets: the index of the sequence
// whose rank is R.  The lengths stay in registers (lane i holds sequences i
// and i + 32) and each lane counts the sequences that precede its own in
// the order; the order is total, so every rank names exactly one sequence.
__device__ __forceinline__ int lpt_sequence(const int64_t *cu, int N, int R) {
  const int lane = threadIdx.x & 31;
  const int64_t l0 = lane < N ? cu[lane + 1] - cu[lane] : -1;
  const int64_t l1 = lane + 32 < N ? cu[lane + 33] - cu[lane + 32] : -1;
  int r0 = 0, r1 = 0;
  for (int m = 0; m < N; m++) {
    const int64_t lm = __shfl_sync(0xffffffffu, m < 32 ? l0 : l1, m & 31);
    r0 += (lm > l0) || (lm == l0 && m < lane);
    r1 += (lm > l1) || (lm == l1 && m < lane + 32);
  }
  const unsigned h0 = __ballot_sync(0xffffffffu, lane < N && r0 == R);
  const unsigned h1 = __ballot_sync(0xffffffffu, lane + 32 < N && r1 == R);
  return h0 ? __ffs(h0) - 1 : (h1 ? 31 + __ffs(h1) : 0);
}

// Index of (b,h)'s state in the kv0 / kv_out arrays: bh itself, or through
// the state pool's slot table; -1 for none.  A slot past the pool is a
// bounds error and treated as none.
__device__ __forceinline__ int64_t state_slot(const Geo &g, int64_t bh) {
  if (!g.slots) return bh;
  const int64_t s = g.slots[bh / g.H];
  if (s < 0) return -1;
  if (s >= g.pool) {
    raise_error(ERR_BOUNDS);
    return -1;
  }
  return s * g.H + bh % g.H;
}

// Geometry of a chunk-state pre-pass and its scan: the (sub-)chunk split,
// forward (chunks 0 .. S-2 of the main split, as (S-1)*M sub-chunks from
// index 0) or reverse (everything after chunk 0: sub-chunks M .. Ssub-1).
inline Geo state_geo(const Geo &g, bool reverse) {
  Geo s = g;
  s.S = g.Ssub;
  s.Lc = g.Ls;
  s.M = 1;
  s.nst = reverse ? g.Ssub - g.M : (g.S - 1) * g.M;
  s.c0 = reverse ? g.M : 0;
  return s;
}

namespace simt {

constexpr int C = 32;         // block rows
constexpr int NT = 256;       // threads per CTA

template <typename T, int W>
__device__ __forceinline__ void load_tile(float *dst, int ld, const T *src,
                                          int cb) {
  // rows >= cb are zero-filled
  for (int idx = threadIdx.x; idx < C * W; idx += NT) {
    int r = idx / W, c = idx % W;
    dst[r * ld + c] = r < cb ? io<T>::ld(src + (int64_t)r * W + c) : 0.f;
  }
}

__device__ __forceinline__ void fill_pow(float *pw, float lam) {
  for (int n = threadIdx.x; n <= C; n += NT) pw[n] = (float)pow_int((double)lam, n);
}

// ------------------------------------------------------------- forward
// OUT = true : full forward for chunk c (grid = B*H*S)
// OUT = false: chunk-state pre-pass for chunks 0..S-2 (grid = B*H*(S-1));
//              writes the chunk's state, started from zero, to ws slot c+1.
template <typename T, int D, int E, bool OUT>
__global__ void __launch_bounds__(NT)
fwd_kernel(const T *__restrict__ q, const T *__restrict__ k,
           const T *__restrict__ v, const float *__restrict__ lambda,
           const float *__restrict__ kv0, T *__restrict__ o,
           float *__restrict__ kv_out, float *__restrict__ ws, Geo g) {
  constexpr int LDQ = D + 1, LDV = E, LDP = C + 1, LDS = E + 1;
  extern __shared__ float sm[];
  float *KV = sm;                     // D x (E+1)
  float *Qs = KV + D * LDS;           // C x (D+1)
  float *Ks = Qs + C * LDQ;           // C x (D+1)
  float *Vs = Ks + C * LDQ;           // C x E
  float *Ps = Vs + C * LDV;           // C x (C+1)
  float *pw = Ps + C * LDP;           // C+1

  // output pass: one CTA per chunk; state pass: g.nst (sub-)chunks from c0
  const int nch = OUT ? g.S : g.nst;
  const Span sp = span_of(g, nch, OUT ? 0 : g.c0);
  const int64_t bh = sp.bh, a = sp.a, slab = sp.slab;
  // a state-pool request that is inactive (negative slot) or out of the
  // pool (reported by state_slot): no rows
  const int64_t b =
      (OUT && g.slots && (unsigned)g.slots[bh / g.H] >= (unsigned)g.pool) ? a : sp.b;
  const int c = sp.c, h = sp.h;

  fill_pow(pw, lambda[h]);
  const float *init = nullptr;
  const int64_t so = state_slot(g, bh);
  if (OUT) {
    if (g.S > 1) init = ws + (bh * g.S + c) * (int64_t)D * E;
    else init = (kv0 && so >= 0) ? kv0 + so * D * E : nullptr;
  }
  for (int idx = threadIdx.x; idx < D * E; idx += NT)
    KV[(idx / E) * LDS + idx % E] = init ? init[idx] : 0.f;
  __syncthreads();

  for (int64_t p = a; p < b; p += C) {
    const int cb = (int)(b - p < C ? b - p : C);
    if (OUT) load_tile<T, D>(Qs, LDQ, q + (slab * g.L + p) * D, cb);
    load_tile<T, D>(Ks, LDQ, k + (slab * g.L + p) * D, cb);
    load_tile<T, E>(Vs, LDV, v + (slab * g.L + p) * E, cb);
    __syncthreads();
    if (OUT) {
      // P = (Q K^T) (.) M over the causal triangle
      for (int idx = threadIdx.x; idx < C * C; idx += NT) {
        int s = idx / C, t = idx % C;
        float val = 0.f;
        if (t <= s && s < cb) {
          float acc = 0.f;
#pragma unroll 8
          for (int i = 0; i < D; i++) acc += Qs[s * LDQ + i] * Ks[t * LDQ + i];
          val = acc * pw[s - t];
        }
        Ps[s * LDP + t] = val;
      }
      __syncthreads();
      // O = P V + diag(lambda^(s+1)) Q KV
      for (int idx = threadIdx.x; idx < C * E; idx += NT) {
        int s = idx / E, j = idx % E;
        if (s >= cb) continue;
        float acc1 = 0.f, acc2 = 0.f;
        for (int t = 0; t <= s; t++) acc1 += Ps[s * LDP + t] * Vs[t * LDV + j];
#pragma unroll 8
        for (int i = 0; i < D; i++) acc2 += Qs[s * LDQ + i] * KV[i * LDS + j];
        io<T>::st(o + (slab * g.L + p + s) * E + j, acc1 + pw[s + 1] * acc2);
      }
      __syncthreads();
    }
    // KV <- lambda^cb KV + (diag(lambda^(cb-1-t)) K)^T V
    for (int idx = threadIdx.x; idx < D * E; idx += NT) {
      int i = idx / E, j = idx % E;
      float acc = 0.f;
      for (int t = 0; t < cb; t++)
        acc += pw[cb - 1 - t] * Ks[t * LDQ + i] * Vs[t * LDV + j];
      KV[i * LDS + j] = pw[cb] * KV[i * LDS + j] + acc;
    }
    __syncthreads();
  }
  float *dst = nullptr;
  if (OUT) dst = (kv_out && c == g.S - 1 && so >= 0) ? kv_out + so * D * E : nullptr;
  else dst = ws + (bh * g.wsS + c + 1) * (int64_t)D * E;
  if (dst)
    for (int idx = threadIdx.x; idx < D * E; idx += NT)
      dst[idx] = KV[(idx / E) * LDS + idx % E];
}

// Forward chunk-entry scan, one thread per state element:
// run = kv0 (or 0); for c = 1..S-1: run = lambda^Lc run + ws[c]; ws[c] = run.
template <int D, int E>
__global__ void __launch_bounds__(NT)
scan_fwd_kernel(float *__restrict__ ws, const float *__restrict__ kv0,
                const float *__restrict__ lambda, Geo g) {
  const int64_t bh = blockIdx.y;
  const int idx = blockIdx.x * NT + threadIdx.x;
  if (idx >= D * E) return;
  const float decay = (float)pow_int((double)lambda[bh % g.H], g.Lc);
  const int64_t so = state_slot(g, bh);
  float run = (kv0 && so >= 0) ? kv0[so * D * E + idx] : 0.f;
  // slot c holds the contribution of (sub-)chunk c-1, c = 1..nst (all full);
  // eight slots' loads are issued before the running sum walks them
  float *base = ws + bh * g.wsS * (int64_t)D * E + idx;
  // slot 0 takes the initial state itself: the split passes read every
  // chunk's entry state here, never kv0, so kv_out may be kv0's storage
  base[0] = run;
  for (int c0 = 1; c0 <= g.nst; c0 += 8) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; j++)
      if (c0 + j <= g.nst) v[j] = base[(int64_t)(c0 + j) * D * E];
#pragma unroll
    for (int j = 0; j < 8; j++)
      if (c0 + j <= g.nst) {
        run = decay * run + v[j];
        base[(int64_t)(c0 + j) * D * E] = run;
      }
  }
}

// ------------------------------------------------------------- backward dQ
template <typename T, int D, int E>
__global__ void __launch_bounds__(NT)
dq_kernel(const T *__restrict__ k, const T *__restrict__ v,
          const T *__restrict__ dO, const float *__restrict__ lambda,
          const float *__restrict__ kv0, T *__restrict__ dq,
          const float *__restrict__ ws, Geo g) {
  constexpr int LDS = E + 1, LDG = E + 1, LDK = D, LDP = C + 1;
  extern __shared__ float sm[];
  float *KV = sm;                 // D x (E+1)
  float *Gs = KV + D * LDS;       // C x (E+1)   dO
  float *Vs = Gs + C * LDG;       // C x (E+1)
  float *Ks = Vs + C * LDG;       // C x D
  float *Ps = Ks + C * LDK;       // C x (C+1)
  float *pw = Ps + C * LDP;

  const Span sp = span_of(g, g.S, 0);
  const int64_t bh = sp.bh, a = sp.a, b = sp.b, slab = sp.slab;
  const int c = sp.c, h = sp.h;
  fill_pow(pw, lambda[h]);
  const float *init = g.S > 1 ? ws + (bh * g.S + c) * (int64_t)D * E
                              : (kv0 ? kv0 + bh * D * E : nullptr);
  for (int idx = threadIdx.x; idx < D * E; idx += NT)
    KV[(idx / E) * LDS + idx % E] = init ? init[idx] : 0.f;
  __syncthreads();

  for (int64_t p = a; p < b; p += C) {
    const int cb = (int)(b - p < C ? b - p : C);
    load_tile<T, E>(Gs, LDG, dO + (slab * g.L + p) * E, cb);
    load_tile<T, E>(Vs, LDG, v + (slab * g.L + p) * E, cb);
    load_tile<T, D>(Ks, LDK, k + (slab * g.L + p) * D, cb);
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * C; idx += NT) {
      int s = idx / C, t = idx % C;
      float val = 0.f;
      if (t <= s && s < cb) {
        float acc = 0.f;
#pragma unroll 8
        for (int j = 0; j < E; j++) acc += Gs[s * LDG + j] * Vs[t * LDG + j];
        val = acc * pw[s - t];
      }
      Ps[s * LDP + t] = val;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * D; idx += NT) {
      int s = idx / D, i = idx % D;
      if (s >= cb) continue;
      float acc1 = 0.f, acc2 = 0.f;
      for (int t = 0; t <= s; t++) acc1 += Ps[s * LDP + t] * Ks[t * LDK + i];
#pragma unroll 8
      for (int j = 0; j < E; j++) acc2 += Gs[s * LDG + j] * KV[i * LDS + j];
      io<T>::st(dq + (slab * g.L + p + s) * D + i, acc1 + pw[s + 1] * acc2);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < D * E; idx += NT) {
      int i = idx / E, j = idx % E;
      float acc = 0.f;
      for (int t = 0; t < cb; t++)
        acc += pw[cb - 1 - t] * Ks[t * LDK + i] * Vs[t * LDG + j];
      KV[i * LDS + j] = pw[cb] * KV[i * LDS + j] + acc;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------ backward dK, dV
// Reverse chunk states: for chunks c = 1..S-1 (grid B*H*(S-1)) the chunk's own
// contribution to the reverse state at its first row,
//   dD[c] = sum_{t in chunk c} lambda^(t - a_c) q_t^T dO_t,
// written to ws slot c-1.
template <typename T, int D, int E>
__global__ void __launch_bounds__(NT)
rev_state_kernel(const T *__restrict__ q, const T *__restrict__ dO,
                 const float *__restrict__ lambda, float *__restrict__ ws, Geo g) {
  constexpr int LDQ = D, LDG = E;
  extern __shared__ float sm[];
  float *Dst = sm;               // D x E
  float *Qs = Dst + D * E;       // C x D
  float *Gs = Qs + C * LDQ;      // C x E
  float *pw = Gs + C * LDG;

  const Span sp = span_of(g, g.nst, g.c0);
  const int64_t bh = sp.bh, a = sp.a, b = sp.b, slab = sp.slab;
  const int c = sp.c, h = sp.h;
  fill_pow(pw, lambda[h]);
  for (int idx = threadIdx.x; idx < D * E; idx += NT) Dst[idx] = 0.f;
  __syncthreads();
  const int64_t nb = (b - a + C - 1) / C;
  for (int64_t ib = nb - 1; ib >= 0; ib--) {
    const int64_t p = a + ib * C;
    const int cb = (int)(b - p < C ? b - p : C);
    load_tile<T, D>(Qs, LDQ, q + (slab * g.L + p) * D, cb);
    load_tile<T, E>(Gs, LDG, dO + (slab * g.L + p) * E, cb);
    __syncthreads();
    for (int idx = threadIdx.x; idx < D * E; idx += NT) {
      int i = idx / E, j = idx % E;
      float acc = 0.f;
      for (int s = 0; s < cb; s++) acc += pw[s] * Qs[s * LDQ + i] * Gs[s * LDG + j];
      Dst[idx] = pw[cb] * Dst[idx] + acc;
    }
    __syncthreads();
  }
  float *dst = ws + (bh * g.wsS + c - 1) * (int64_t)D * E;
  for (int idx = threadIdx.x; idx < D * E; idx += NT) dst[idx] = Dst[idx];
}

// Reverse scan: run = 0; for c = S-2..0: run = lambda^len(c+1) run + ws[c];
// ws[c] = run.  Afterwards ws[c] is the reverse state entering chunk c from
// the right (the state at its last row + 1).
template <int D, int E>
__global__ void __launch_bounds__(NT)
scan_rev_kernel(float *__restrict__ ws, const float *__restrict__ lambda,
                const float *__restrict__ dend, Geo g) {
  const int64_t bh = blockIdx.y;
  const int idx = blockIdx.x * NT + threadIdx.x;
  if (idx >= D * E) return;
  const double lam = (double)lambda[bh % g.H];
  const float full = (float)pow_int(lam, g.Lc);
  const float last = (float)pow_int(lam, g.L - (int64_t)(g.S - 1) * g.Lc);
  // the reverse state past the sequence end (NULL: zero)
  float run = dend ? dend[bh * D * E + idx] : 0.f;
  // slot c holds the contribution of (sub-)chunk c+1, c+1 = c0..S-1, walked
  // downwards with eight slots' loads in flight
  float *base = ws + bh * g.wsS * (int64_t)D * E + idx;
  const int lo = g.c0 - 1;
  for (int c1 = g.S - 2; c1 >= lo; c1 -= 8) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; j++)
      if (c1 - j >= lo) v[j] = base[(int64_t)(c1 - j) * D * E];
#pragma unroll
    for (int j = 0; j < 8; j++)
      if (c1 - j >= lo) {
        const int c = c1 - j;
        run = (c + 1 == g.S - 1 ? last : full) * run + v[j];
        base[(int64_t)c * D * E] = run;
      }
  }
}

template <typename T, int D, int E>
__global__ void __launch_bounds__(NT)
dkdv_kernel(const T *__restrict__ q, const T *__restrict__ k,
            const T *__restrict__ v, const T *__restrict__ dO,
            const float *__restrict__ lambda, T *__restrict__ dk,
            T *__restrict__ dv, float *__restrict__ dkv0,
            const float *__restrict__ ws, const float *__restrict__ dend, Geo g) {
  constexpr int LDQ = D + 1, LDG = E + 1, LDS = E + 1, LDP = C + 1;
  extern __shared__ float sm[];
  float *Dst = sm;                 // D x (E+1)
  float *Qs = Dst + D * LDS;       // C x (D+1)
  float *Ks = Qs + C * LDQ;        // C x (D+1)
  float *Vs = Ks + C * LDQ;        // C x (E+1)
  float *Gs = Vs + C * LDG;        // C x (E+1)
  float *Pt = Gs + C * LDG;        // C x (C+1)  (Q K^T (.) M)^T
  float *dPt = Pt + C * LDP;       // C x (C+1)  (dO V^T (.) M)^T
  float *pw = dPt + C * LDP;

  const Span sp = span_of(g, g.S, 0);
  const int64_t bh = sp.bh, a = sp.a, b = sp.b, slab = sp.slab;
  const int c = sp.c, h = sp.h;
  fill_pow(pw, lambda[h]);
  const float *init = c == g.S - 1 ? (dend ? dend + bh * D * E : nullptr)
                                   : ws + (bh * g.S + c) * (int64_t)D * E;
  for (int idx = threadIdx.x; idx < D * E; idx += NT)
    Dst[(idx / E) * LDS + idx % E] = init ? init[idx] : 0.f;
  __syncthreads();

  const int64_t nb = (b - a + C - 1) / C;
  for (int64_t ib = nb - 1; ib >= 0; ib--) {
    const int64_t p = a + ib * C;
    const int cb = (int)(b - p < C ? b - p : C);
    load_tile<T, D>(Qs, LDQ, q + (slab * g.L + p) * D, cb);
    load_tile<T, D>(Ks, LDQ, k + (slab * g.L + p) * D, cb);
    load_tile<T, E>(Vs, LDG, v + (slab * g.L + p) * E, cb);
    load_tile<T, E>(Gs, LDG, dO + (slab * g.L + p) * E, cb);
    __syncthreads();
    // transposed masked products, [t][s] with s >= t
    for (int idx = threadIdx.x; idx < C * C; idx += NT) {
      int t = idx / C, s = idx % C;
      float pv = 0.f, dpv = 0.f;
      if (s >= t && s < cb) {
        float a1 = 0.f, a2 = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; i++) a1 += Qs[s * LDQ + i] * Ks[t * LDQ + i];
#pragma unroll 8
        for (int j = 0; j < E; j++) a2 += Gs[s * LDG + j] * Vs[t * LDG + j];
        pv = a1 * pw[s - t];
        dpv = a2 * pw[s - t];
      }
      Pt[t * LDP + s] = pv;
      dPt[t * LDP + s] = dpv;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * D; idx += NT) {
      int t = idx / D, i = idx % D;
      if (t >= cb) continue;
      float acc1 = 0.f, acc2 = 0.f;
      for (int s = t; s < cb; s++) acc1 += dPt[t * LDP + s] * Qs[s * LDQ + i];
#pragma unroll 8
      for (int j = 0; j < E; j++) acc2 += Vs[t * LDG + j] * Dst[i * LDS + j];
      io<T>::st(dk + (slab * g.L + p + t) * D + i, acc1 + pw[cb - t] * acc2);
    }
    for (int idx = threadIdx.x; idx < C * E; idx += NT) {
      int t = idx / E, j = idx % E;
      if (t >= cb) continue;
      float acc1 = 0.f, acc2 = 0.f;
      for (int s = t; s < cb; s++) acc1 += Pt[t * LDP + s] * Gs[s * LDG + j];
#pragma unroll 8
      for (int i = 0; i < D; i++) acc2 += Ks[t * LDQ + i] * Dst[i * LDS + j];
      io<T>::st(dv + (slab * g.L + p + t) * E + j, acc1 + pw[cb - t] * acc2);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < D * E; idx += NT) {
      int i = idx / E, j = idx % E;
      float acc = 0.f;
      for (int s = 0; s < cb; s++) acc += pw[s] * Qs[s * LDQ + i] * Gs[s * LDG + j];
      Dst[i * LDS + j] = pw[cb] * Dst[i * LDS + j] + acc;
    }
    __syncthreads();
  }
  if (c == 0 && dkv0) {
    const float lam = lambda[h];
    for (int idx = threadIdx.x; idx < D * E; idx += NT)
      dkv0[bh * D * E + idx] = lam * Dst[(idx / E) * LDS + idx % E];
  }
}

// Shared-memory bytes of each kernel (must match the carve-ups above).
template <int D, int E> constexpr size_t fwd_smem() {
  return sizeof(float) * (D * (E + 1) + 2 * C * (D + 1) + C * E + C * (C + 1) + C + 1);
}
template <int D, int E> constexpr size_t dq_smem() {
  return sizeof(float) * (D * (E + 1) + 2 * C * (E + 1) + C * D + C * (C + 1) + C + 1);
}
template <int D, int E> constexpr size_t rev_smem() {
  return sizeof(float) * (D * E + C * D + C * E + C + 1);
}
template <int D, int E> constexpr size_t dkdv_smem() {
  return sizeof(float) * (D * (E + 1) + 2 * C * (D + 1) + 2 * C * (E + 1) +
                          2 * C * (C + 1) + C + 1);
}

// Asynchronous copy of rows [0, cb) of a C-row tile (row length W, type T)
// into `raw` (C x W, dense), 16 bytes per copy; rows >= cb are filled with
// zeros (a zero-byte source read from row 0, which exists).
template <typename T, int W>
__device__ __forceinline__ void stage_tile(T *raw, const T *src, int cb) {
  constexpr int PER = 16 / (int)sizeof(T), CH = W / PER;
  for (int idx = threadIdx.x; idx < C * CH; idx += NT) {
    const int r = idx / CH, ch = idx % CH;
    const T *s = src + (int64_t)(r < cb ? r : 0) * W + ch * PER;
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(raw + r * W + ch * PER);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(s),
                 "r"(r < cb ? 16 : 0)
                 : "memory");
  }
}
__device__ __forceinline__ void stage_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void stage_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// fp32 copy of a staged tile into a padded tile (row stride ld).
template <typename T, int W>
__device__ __forceinline__ void unstage_tile(float *dst, int ld, const T *raw) {
  for (int idx = threadIdx.x; idx < C * W; idx += NT) {
    const int r = idx / W, c = idx % W;
    dst[r * ld + c] = io<T>::ld(raw + idx);
  }
}

// ------------------------------------------------------------ d lambda
// Gradient of sum(o * dO) with respect to lambda_h, added into dlam[h].
// With the carried states at the start of a block of rows p.. (local t, j):
//   KV = sum_{j<p} lambda^(p-1-j) k_j^T v_j,
//   W  = sum_{j<p} (p-1-j) lambda^(p-1-j) k_j^T v_j,
// the derivative of o_t splits into the block's own pairs
//   sum_{j<t} (t-j) lambda^(t-j-1) (q_t . k_j) v_j
// and the earlier rows  lambda^t ((t+1) q_t KV + q_t W)  (KV = kv0, W = 0
// before the first row: d/dlambda of lambda^(t+1) q_t kv0); both are dotted
// with dO_t.  Then W <- lambda^cb (cb KV + W) + sum_j (cb-1-j) lambda^(cb-1-j)
// k_j^T v_j and KV <- lambda^cb KV + sum_j lambda^(cb-1-j) k_j^T v_j.  No
// division by lambda, so lambda = 0 is exact.  The same pair of updates over
// a whole chunk of Lc rows composes chunks:  W' = lambda^Lc (Lc KV + W) + dW,
// KV' = lambda^Lc KV + dKV.
//
// Layout: the 256 threads form a 16 x 16 grid; thread (ti, tc) keeps the
// entries (ti + 16 i, tc + 16 j) of KV and of W, i < D/16, j < E/16, in
// registers for the whole chunk, so the per-row work is outer products of a
// q (k) row slice with a dO (v) row slice read from shared memory (the 16
// threads of a row read 16 consecutive words: no bank conflicts).  The
// block's own pairs take 2 x 2 tiles of S = Q K^T and G = dO V^T per thread.
// STATE = true: the chunk-state pre-pass (from zero, no gradient) over the
// g.nst sub-chunks of Ls rows before the last chunk: writes sub-chunk u's
// (dKV, dW) to workspace slot u+1 of the (b,h)'s wsS slots.  The gradient
// pass's chunk c (Lc = M Ls rows) enters with the pair in slot c M.
template <typename T, int D, int E>
constexpr size_t dlam_smem() {
  return sizeof(float) * (2 * C * (D + 1) + 2 * C * (E + 1) + (C + 2)) + sizeof(double) * (NT / 32) +
         16 + sizeof(T) * (2 * C * D + 2 * C * E);
}

template <typename T, int D, int E, bool STATE>
__global__ void __launch_bounds__(NT, 1)
dlambda_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
               const T *__restrict__ dO, const float *__restrict__ lambda,
               const float *__restrict__ kv0, float *__restrict__ ws, float *__restrict__ dlam,
               Geo g) {
  constexpr int LQ = D + 1, LV = E + 1;  // odd row strides: row r starts at bank r
  constexpr int TI = D / 16, TC = E / 16;
  extern __shared__ float sm[];
  float *Qs = sm;                  // C x LQ
  float *Ks = Qs + C * LQ;         // C x LQ
  float *Vs = Ks + C * LQ;         // C x LV
  float *Gs = Vs + C * LV;         // C x LV   dO
  float *pw = Gs + C * LV;         // C+1
  double *red = reinterpret_cast<double *>(pw + C + 2);  // NT/32
  // the next block's rows in flight while the current one is computed (16-
  // byte aligned: the copies move 16 bytes; every row is a multiple of 16)
  T *rQ = reinterpret_cast<T *>((reinterpret_cast<uintptr_t>(red + NT / 32) + 15) &
                                ~static_cast<uintptr_t>(15));  // C x D each, then C x E
  T *rK = rQ + C * D, *rV = rK + C * D, *rG = rV + C * E;

  const int nch = STATE ? g.nst : g.S;
  const int64_t len = STATE ? g.Ls : g.Lc;
  const int64_t bh = blockIdx.x / nch;
  const int c = blockIdx.x % nch;
  const int h = (int)(bh % g.H);
  const int64_t a = (int64_t)c * len;
  const int64_t b = g.L < a + len ? g.L : a + len;
  const int tid = threadIdx.x;
  const int ti = tid >> 4, tc = tid & 15;
  fill_pow(pw, lambda[h]);

  float KV[TI][TC], Wt[TI][TC];
  {
    const float *ikv = nullptr, *iw = nullptr;
    if (!STATE) {
      if (g.S > 1) {
        ikv = ws + ((bh * g.wsS + (int64_t)c * g.M) * 2) * (int64_t)D * E;
        iw = ikv + D * E;
      } else if (kv0) {
        ikv = kv0 + bh * (int64_t)D * E;
      }
    }
#pragma unroll
    for (int i = 0; i < TI; i++)
#pragma unroll
      for (int j = 0; j < TC; j++) {
        KV[i][j] = ikv ? ikv[(ti + 16 * i) * E + tc + 16 * j] : 0.f;
        Wt[i][j] = iw ? iw[(ti + 16 * i) * E + tc + 16 * j] : 0.f;
      }
  }
  double acc = 0.0;
  auto stage = [&](int64_t p) {
    const int cb = (int)(b - p < C ? b - p : C);
    if (!STATE) stage_tile<T, D>(rQ, q + (bh * g.L + p) * D, cb);
    stage_tile<T, D>(rK, k + (bh * g.L + p) * D, cb);
    stage_tile<T, E>(rV, v + (bh * g.L + p) * E, cb);
    if (!STATE) stage_tile<T, E>(rG, dO + (bh * g.L + p) * E, cb);
    stage_commit();
  };
  if (a < b) stage(a);

  for (int64_t p = a; p < b; p += C) {
    const int cb = (int)(b - p < C ? b - p : C);
    stage_wait();
    __syncthreads();  // the block's rows have landed; the previous block is done
    if (!STATE) unstage_tile<T, D>(Qs, LQ, rQ);
    unstage_tile<T, D>(Ks, LQ, rK);
    unstage_tile<T, E>(Vs, LV, rV);
    if (!STATE) unstage_tile<T, E>(Gs, LV, rG);
    __syncthreads();
    if (p + C < b) stage(p + C);
    if (!STATE) {
      float part = 0.f;
      // the earlier rows: lambda^t ((t+1) q_t KV dO_t + q_t W dO_t), the
      // thread's tile of the double sums
      for (int t = 0; t < cb; t++) {
        float qv[TI], gv[TC];
#pragma unroll
        for (int i = 0; i < TI; i++) qv[i] = Qs[t * LQ + ti + 16 * i];
#pragma unroll
        for (int j = 0; j < TC; j++) gv[j] = Gs[t * LV + tc + 16 * j];
        float s1 = 0.f, s0 = 0.f;
#pragma unroll
        for (int i = 0; i < TI; i++) {
          float r1 = 0.f, r0 = 0.f;
#pragma unroll
          for (int j = 0; j < TC; j++) {
            r1 = fmaf(KV[i][j], gv[j], r1);
            r0 = fmaf(Wt[i][j], gv[j], r0);
          }
          s1 = fmaf(qv[i], r1, s1);
          s0 = fmaf(qv[i], r0, s0);
        }
        part += pw[t] * fmaf((float)(t + 1), s1, s0);
      }
      // the block's own pairs j < t: 2 x 2 of S = Q K^T and G = dO V^T
      {
        const int t0 = 2 * ti, j0 = 2 * tc;
        float S[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, G[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        if (j0 < t0 + 1 && t0 < cb) {
#pragma unroll 4
          for (int x = 0; x < D; x++) {
            const float qa = Qs[t0 * LQ + x], qb = Qs[(t0 + 1) * LQ + x];
            const float ka = Ks[j0 * LQ + x], kb = Ks[(j0 + 1) * LQ + x];
            S[0][0] = fmaf(qa, ka, S[0][0]); S[0][1] = fmaf(qa, kb, S[0][1]);
            S[1][0] = fmaf(qb, ka, S[1][0]); S[1][1] = fmaf(qb, kb, S[1][1]);
          }
#pragma unroll 4
          for (int x = 0; x < E; x++) {
            const float ga = Gs[t0 * LV + x], gb = Gs[(t0 + 1) * LV + x];
            const float va = Vs[j0 * LV + x], vb = Vs[(j0 + 1) * LV + x];
            G[0][0] = fmaf(ga, va, G[0][0]); G[0][1] = fmaf(ga, vb, G[0][1]);
            G[1][0] = fmaf(gb, va, G[1][0]); G[1][1] = fmaf(gb, vb, G[1][1]);
          }
#pragma unroll
          for (int u = 0; u < 2; u++)
#pragma unroll
            for (int w = 0; w < 2; w++) {
              const int t = t0 + u, j = j0 + w;
              if (j < t && t < cb) part += (float)(t - j) * pw[t - j - 1] * S[u][w] * G[u][w];
            }
        }
      }
      acc += (double)part;
    }
    // W from the old KV, then KV; then the block's rows
    const float dec = pw[cb];
#pragma unroll
    for (int i = 0; i < TI; i++)
#pragma unroll
      for (int j = 0; j < TC; j++) {
        Wt[i][j] = dec * fmaf((float)cb, KV[i][j], Wt[i][j]);
        KV[i][j] = dec * KV[i][j];
      }
    for (int jr = 0; jr < cb; jr++) {
      const float bj = pw[cb - 1 - jr], wj = (float)(cb - 1 - jr) * bj;
      float kv_[TI], vv[TC];
#pragma unroll
      for (int i = 0; i < TI; i++) kv_[i] = Ks[jr * LQ + ti + 16 * i];
#pragma unroll
      for (int j = 0; j < TC; j++) vv[j] = Vs[jr * LV + tc + 16 * j];
#pragma unroll
      for (int i = 0; i < TI; i++) {
        const float kb = bj * kv_[i], kw = wj * kv_[i];
#pragma unroll
        for (int j = 0; j < TC; j++) {
          KV[i][j] = fmaf(kb, vv[j], KV[i][j]);
          Wt[i][j] = fmaf(kw, vv[j], Wt[i][j]);
        }
      }
    }
  }
  if constexpr (STATE) {
    float *okv = ws + ((bh * g.wsS + c + 1) * 2) * (int64_t)D * E, *ow = okv + D * E;
#pragma unroll
    for (int i = 0; i < TI; i++)
#pragma unroll
      for (int j = 0; j < TC; j++) {
        okv[(ti + 16 * i) * E + tc + 16 * j] = KV[i][j];
        ow[(ti + 16 * i) * E + tc + 16 * j] = Wt[i][j];
      }
  } else {
    // block sum, then one atomic add per CTA
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((tid & 31) == 0) red[tid >> 5] = acc;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < NT / 32; w++) t += red[w];
      atomicAdd(dlam + h, (float)t);
    }
  }
}

// Sub-chunk entry states of the decay gradient, in place over the
// workspace's [B*H, wsS, 2, D, E] slots: slot u+1 holds sub-chunk u's (dKV,
// dW) (all Ls rows); afterwards slot u holds the (KV, W) entering sub-chunk
// u, slot 0 the initial (kv0 or 0, 0).
template <int D, int E>
__global__ void __launch_bounds__(NT)
dlam_scan_kernel(float *__restrict__ ws, const float *__restrict__ kv0,
                 const float *__restrict__ lambda, Geo g) {
  const int64_t bh = blockIdx.y;
  const int idx = blockIdx.x * NT + threadIdx.x;
  if (idx >= D * E) return;
  const float f = (float)pow_int((double)lambda[bh % g.H], g.Ls);
  const float n = (float)g.Ls;
  float *base = ws + bh * g.wsS * 2 * (int64_t)D * E + idx;
  float kv = kv0 ? kv0[bh * D * E + idx] : 0.f, w = 0.f;
  base[0] = kv;
  base[D * E] = w;
  for (int c = 1; c <= g.nst; c++) {
    float *s = base + (int64_t)c * 2 * D * E;
    const float dkv = s[0], dw = s[D * E];
    w = fmaf(f, fmaf(n, kv, w), dw);
    kv = fmaf(f, kv, dkv);
    s[0] = kv;
    s[D * E] = w;
  }
}

}  // namespace simt
}  // namespace la2
