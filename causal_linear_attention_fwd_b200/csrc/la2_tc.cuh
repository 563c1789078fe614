// la2_tc.cuh -- tensor-core kernels (tcgen05 + TMEM + TMA) for bf16, d = e = 128.
//
// One CTA owns one chunk of one (b,h) sequence and walks its blocks of
// C = 128 rows in order, keeping the d x e state on chip (fp32 in TMEM) the
// whole way -- the intra-block / inter-block split of the Lightning
// Attention-2 notes page ("Tiling." paragraph), re-derived for sm_100a:
//
//   S  = A0 B1^T                 (QK^T; dQ pass: dO V^T)        -> TMEM S
//   X  = A0 KV                   (state term; dQ pass: dO KV^T)  -> TMEM X
//   P  = S (.) M  (bf16)         written back into TMEM over S   (CUDA cores)
//   Y  = P B2                    (A operand read from TMEM)      -> TMEM Y
//   B1 <- diag(lambda^(cb-1-t)) B1   in place in shared memory    (CUDA cores)
//   KV <- lambda^cb KV + Kb^T V  (accumulated in TMEM)
//   O  = Y + diag(lambda^(s+1)) X   -> bf16 -> shared -> TMA store
//
// with M[s,t] = lambda^(s-t) for t <= s.  The forward pass uses
// (A0, B1, B2) = (Q, K, V); the backward runs the same schedule three more
// times with other tiles, factors and directions (see the MODE_ list below):
// dQ by a forward scan, dV and dK by reverse scans over the reverse state
// D = sum_{t beyond the block} lambda^.. q_t^T dO_t.  The chunk-state
// pre-passes run only the state recurrence from a zero state and write the
// chunk's state to the workspace.
//
// Data path: TMA (128-byte swizzle, two 64-column boxes per 128 x 128 tile)
// double-buffers the next block's tiles while the current one is processed;
// every MMA is M = 128, N = 128, K = 16 steps issued by one thread;
// completion is signalled through mbarriers, and every wait is bounded (see
// la2_sm100.cuh).  TMEM: S [0,128), X [128,256), Y [256,384), KV [384,512).
#pragma once

#include <cuda.h>

#include "la2_common.cuh"
#include "la2_simt.cuh"
#include "la2_sm100.cuh"

namespace la2 {
namespace tc {

constexpr int BLOCK = 128;       // rows per block (MMA M)
constexpr int NT = 256;          // 8 warps: (lane quarter) x (column half)
constexpr uint32_t BOX = 16384;  // 128 rows x 64 bf16 (one TMA box)
constexpr uint32_t TILE = 32768; // 128 rows x 128 bf16

// Passes of the one chunk kernel.  (A0, B1, B2) are the three tiles each
// block loads; S = A0 B1^T, Y = P B2, X = A0 (state or state^T), and the
// state update is B1s^T B2 or B2^T B1s with B1s = B1 after its row decay.
//   FWD    (Q,  K,  V ) forward order, O  = Y + lambda^(s+1)  X,  KV += (b K)^T V
//   DQ     (dO, V,  K ) forward order, dQ = Y + lambda^(s+1)  X,  KV += K^T (b V)
//   DV     (K,  Q,  dO) reverse order, dV = Y + lambda^(cb-t) X,  D  += (g Q)^T dO
//   DK     (V,  dO, Q ) reverse order, dK = Y + lambda^(cb-t) X,  D  += Q^T (g dO)
//   STATE  (-,  K,  V ) forward chunk state from zero
//   RSTATE (-,  Q,  dO) reverse chunk state from zero
// b_t = lambda^(cb-1-t) (key side, forward), g_s = lambda^s (query side, reverse).
// The reverse passes use the transposed mask: S^T[t][s] kept for s >= t.
// RPAIR is DV or DK chosen per CTA at run time (the paired reverse launch):
// one body serves both, so the two SMs of a pair run the same instructions.
enum { MODE_FWD = 0, MODE_DQ = 1, MODE_STATE = 2, MODE_DV = 3, MODE_DK = 4, MODE_RSTATE = 5,
       MODE_RPAIR = 6 };

template <int MODE> struct Traits {
  static constexpr bool OUT = MODE != MODE_STATE && MODE != MODE_RSTATE;
  static constexpr bool REV =
      MODE == MODE_DV || MODE == MODE_DK || MODE == MODE_RSTATE || MODE == MODE_RPAIR;
  static constexpr bool SWAP = MODE == MODE_DQ || MODE == MODE_DK;  // state A/B from (B2, B1)
  static constexpr bool X_MN = MODE == MODE_FWD || MODE == MODE_DV; // X's B operand MN-major
};

template <int MODE> struct Layout {
  static constexpr bool OUT = Traits<MODE>::OUT;
  static constexpr int NSTAGE = OUT ? 2 : 3;
  static constexpr uint32_t STAGE = OUT ? 3 * TILE : 2 * TILE;
  static constexpr uint32_t KVBF = NSTAGE * STAGE;
  static constexpr uint32_t MISC = KVBF + (OUT ? TILE : 0);
  // full[NS], mma, done (abort path), then the TMEM slot, the abort flag
  // and the decay table
  static constexpr uint32_t MISC_BYTES = 8 * (NSTAGE + 2) + 16 + 4 * (BLOCK + 1);
  static constexpr uint32_t SMEM = MISC + MISC_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = OUT ? 512 : 128;
  static constexpr uint32_t COL_S = 0, COL_X = 128, COL_Y = 256;
  static constexpr uint32_t COL_KV = OUT ? 384 : 0;
};

inline bool supports(int d, int e, bool bf16) { return bf16 && d == 128 && e == 128; }

// Chunks per (b,h).  One CTA per SM at a time (each uses all of TMEM), and
// a block's time is set mostly by its latency chain, not by its share of
// HBM bandwidth, so a single wave of long chunks beats several waves of
// short ones: when B*H leaves SMs idle, split each sequence into
// floor(SMs / (B*H)) chunks, else not at all.  (Measured on the H = 32
// length sweep: L = 32K, B*H = 64 is fastest at S = 2, L = 64K, B*H = 32 at
// S = 4; more chunks, or two waves, were slower because the chunk-state
// pre-pass grows with S.)
inline int64_t auto_split(int64_t BH, int64_t nblk, int sms) {
  (void)nblk;
  if (BH >= sms) return 1;
  return sms / BH;
}

using namespace la2::sm100;

// Write 32 fp32 values as bf16 into row `row`, logical 16-byte chunks
// [chunk0, chunk0+4) of a 128-byte-swizzled [rows][64] box at `box`.
__device__ __forceinline__ void st_row_bf16_sw128(uint8_t *box, int row, int chunk0,
                                                  const float *v) {
#pragma unroll
  for (int q = 0; q < 4; q++) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    const int chunk = chunk0 + q;
    *reinterpret_cast<uint4 *>(box + row * 128 + ((chunk ^ (row & 7)) << 4)) = w;
  }
}

// Multiply one 64-element row of a swizzled box by f, in place.
__device__ __forceinline__ void scale_row_sw128(uint8_t *box, int row, float f) {
#pragma unroll
  for (int c = 0; c < 8; c++) {
    uint4 *p = reinterpret_cast<uint4 *>(box + row * 128 + ((c ^ (row & 7)) << 4));
    uint4 w = *p;
    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int j = 0; j < 4; j++) {
      __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&u[j]);
      float2 f2 = __bfloat1622float2(x);
      u[j] = pack_bf16x2(f2.x * f, f2.y * f);
    }
    *p = w;
  }
}

template <int MODE>
__global__ void __launch_bounds__(NT, 1)
chunk_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
             const __grid_constant__ CUtensorMap tm2, const __grid_constant__ CUtensorMap tmo,
             const float *__restrict__ lambda, const float *__restrict__ kv0,
             float *__restrict__ ws, float *__restrict__ kv_out, Geo g) {
  using LY = Layout<MODE>;
  using TR = Traits<MODE>;
  constexpr bool OUT = LY::OUT;
  constexpr bool REV = TR::REV;
  constexpr int NS = LY::NSTAGE;
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
  constexpr uint32_t IDESC_X = idesc_bf16(128, 128, false, TR::X_MN);
  constexpr uint32_t IDESC_Y = idesc_bf16(128, 128, false, true);
  constexpr uint32_t IDESC_D = idesc_bf16(128, 128, true, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + LY::MISC);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NS + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *pw = reinterpret_cast<float *>(tmem_slot + 4);
  const uint32_t bar_full0 = smem_u32(bars);
  const uint32_t bar_mma = smem_u32(bars + NS);
  const uint32_t bar_done = smem_u32(bars + NS + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int row = quarter * 32 + lane;
  const int nch = OUT ? g.S : g.nst;
  const int64_t bh = blockIdx.x / nch;
  const int c = blockIdx.x % nch + (OUT ? 0 : g.c0);
  const int h = (int)(bh % g.H);
  const int64_t a = (int64_t)c * g.Lc;
  const int64_t b = g.L < a + g.Lc ? g.L : a + g.Lc;
  const int nblk = (int)((b - a + BLOCK - 1) / BLOCK);

  if (tid <= BLOCK) pw[tid] = (float)pow_int((double)lambda[h], tid);
  if (tid == 0) {
    for (int s = 0; s < NS; s++) mbar_init(bar_full0 + 8 * s, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (OUT) tma_prefetch_desc(&tm0);
    tma_prefetch_desc(&tm1);
    tma_prefetch_desc(&tm2);
    if (OUT) tma_prefetch_desc(&tmo);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), LY::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);  // this warp's lane quarter

  // block visited at step j (reverse passes walk the chunk backwards)
  auto block_of = [&](int j) { return REV ? nblk - 1 - j : j; };
  auto issue_load = [&](int j, int st) {
    const int y = (int)(a + (int64_t)block_of(j) * BLOCK), z = (int)bh;
    const uint32_t bar = bar_full0 + 8 * st;
    uint32_t dst = sbase + st * LY::STAGE;
    mbar_expect_tx(bar, LY::STAGE);
    if (OUT) {
      tma_load_3d(dst, &tm0, bar, 0, y, z);
      tma_load_3d(dst + BOX, &tm0, bar, 64, y, z);
      dst += TILE;
    }
    tma_load_3d(dst, &tm1, bar, 0, y, z);
    tma_load_3d(dst + BOX, &tm1, bar, 64, y, z);
    tma_load_3d(dst + TILE, &tm2, bar, 0, y, z);
    tma_load_3d(dst + TILE + BOX, &tm2, bar, 64, y, z);
  };
  int issued = 0;
  if (tid == 0)
    for (; issued < NS && issued < nblk; issued++) issue_load(issued, issued);

  // initial state -> TMEM (fp32) and, for the output passes, a bf16 copy in
  // shared memory (row d = this thread's row, columns e of this half)
  {
    const float *init = nullptr;
    if (MODE == MODE_FWD || MODE == MODE_DQ) {
      // a split pass reads every chunk's entry state from the workspace (the
      // scan put the initial one in slot 0), never kv0, which kv_out may reuse
      if (g.S > 1) {
        init = ws + (bh * g.wsS + (int64_t)c * g.M) * (int64_t)128 * 128;
      } else {
        const int64_t so = state_slot(g, bh);
        init = (kv0 && so >= 0) ? kv0 + so * 128 * 128 : nullptr;
      }
    } else if (MODE == MODE_DV || MODE == MODE_DK) {
      if (c != g.S - 1) init = ws + (bh * g.wsS + (int64_t)(c + 1) * g.M - 1) * (int64_t)128 * 128;
      else init = kv0 ? kv0 + bh * 128 * 128 : nullptr;
    }
    uint8_t *kvbf = smem + LY::KVBF + half * BOX;
#pragma unroll
    for (int part = 0; part < 2; part++) {
      const int col = half * 64 + part * 32;
      uint32_t r[32];
      float f[32];
      if (init) {
        const float4 *src = reinterpret_cast<const float4 *>(init + (int64_t)row * 128 + col);
#pragma unroll
        for (int j = 0; j < 8; j++) {
          float4 x = src[j];
          f[4 * j] = x.x; f[4 * j + 1] = x.y; f[4 * j + 2] = x.z; f[4 * j + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; j++) f[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 32; j++) r[j] = __float_as_uint(f[j]);
      tmem_st32(tl + LY::COL_KV + col, r);
      if (OUT) st_row_bf16_sw128(kvbf, row, part * 4, f);
    }
    tmem_wait_st();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  uint32_t mma_phase = 0;
  bool aborted = false;
  int i = 0;
  for (; i < nblk; i++) {
    const int st = i % NS;
    const int64_t p = a + (int64_t)block_of(i) * BLOCK;
    const int cb = (int)(b - p < BLOCK ? b - p : BLOCK);
    uint8_t *stage = smem + st * LY::STAGE;
    const uint32_t sT0 = sbase + st * LY::STAGE;
    const uint32_t sT1 = OUT ? sT0 + TILE : sT0;
    const uint32_t sT2 = sT1 + TILE;
    uint8_t *T0 = stage;
    uint8_t *T1 = OUT ? stage + TILE : stage;
    const uint32_t sKV = sbase + LY::KVBF;

    bool ok = mbar_wait(bar_full0 + 8 * st, (uint32_t)((i / NS) & 1), abort_flag);
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    tc_fence_after();

    if (OUT) {
      // ---- phase 1: S = A0 B1^T, X = A0 KV
      if (tid == 0) {
#pragma unroll
        for (int k = 0; k < 8; k++) {
          const uint32_t koff = (k >> 2) * BOX + (k & 3) * 32;
          mma_ss(tmem + LY::COL_S, sdesc_sw128(sT0 + koff, 16, 1024),
                 sdesc_sw128(sT1 + koff, 16, 1024), IDESC_S, k > 0);
        }
#pragma unroll
        for (int k = 0; k < 8; k++) {
          const uint32_t koff = (k >> 2) * BOX + (k & 3) * 32;
          const uint64_t bd = TR::X_MN ? sdesc_sw128(sKV + k * 2048, BOX, 1024)
                                       : sdesc_sw128(sKV + koff, 16, 1024);
          mma_ss(tmem + LY::COL_X, sdesc_sw128(sT0 + koff, 16, 1024), bd, IDESC_X, k > 0);
        }
        // test hook: withhold this signal once so the waits below run out
        if (!(g.inject && blockIdx.x == 0 && i == 0)) mma_commit(bar_mma);
      }
      ok = mbar_wait(bar_mma, mma_phase, abort_flag);
      mma_phase ^= 1;
      if (__syncthreads_or(!ok)) { aborted = true; break; }
      tc_fence_after();

      // ---- phase 2a: P = S (.) M -> bf16, into the S columns of this half
      //      (forward: keep col <= row, factor lambda^(row-col);
      //       reverse, S^T: keep col >= row, factor lambda^(col-row))
#pragma unroll
      for (int part = 0; part < 2; part++) {
        const int col0 = half * 64 + part * 32;
        uint32_t r[32];
        tmem_ld32(tl + LY::COL_S + col0, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; j++) {
          const int t0 = col0 + 2 * j, t1 = t0 + 1;
          float f0, f1;
          if (REV) {
            f0 = t0 >= row ? __uint_as_float(r[2 * j]) * pw[t0 - row] : 0.f;
            f1 = t1 >= row ? __uint_as_float(r[2 * j + 1]) * pw[t1 - row] : 0.f;
          } else {
            f0 = t0 <= row ? __uint_as_float(r[2 * j]) * pw[row - t0] : 0.f;
            f1 = t1 <= row ? __uint_as_float(r[2 * j + 1]) * pw[row - t1] : 0.f;
          }
          pk[j] = pack_bf16x2(f0, f1);
        }
        tmem_st16(tl + LY::COL_S + half * 64 + part * 16, pk);
      }
    }
    // ---- phase 2b: B1 rows decayed in place for the state update
    //      (forward lambda^(cb-1-t), reverse lambda^s; rows past the block end: 0)
    {
      const float f = row < cb ? (REV ? pw[row] : pw[cb - 1 - row]) : 0.f;
      scale_row_sw128(T1 + half * BOX, row, f);
    }
    // ---- phase 2c: KV acc *= lambda^cb
    {
      const float dec = pw[cb];
#pragma unroll
      for (int part = 0; part < 2; part++) {
        const uint32_t col = LY::COL_KV + half * 64 + part * 32;
        uint32_t r[32];
        tmem_ld32(tl + col, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j++) r[j] = __float_as_uint(__uint_as_float(r[j]) * dec);
        tmem_st32(tl + col, r);
      }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- phase 3: Y = P B2 (P from TMEM), KV += A^T B (state update)
    if (tid == 0) {
      if (OUT) {
#pragma unroll
        for (int k = 0; k < 8; k++) {
          const uint32_t pa = tmem + LY::COL_S + (k >> 2) * 64 + (k & 3) * 8;
          mma_ts(tmem + LY::COL_Y, pa, sdesc_sw128(sT2 + k * 2048, BOX, 1024), IDESC_Y, k > 0);
        }
      }
      const uint32_t sA = TR::SWAP ? sT2 : sT1;
      const uint32_t sB = TR::SWAP ? sT1 : sT2;
#pragma unroll
      for (int k = 0; k < 8; k++)
        mma_ss(tmem + LY::COL_KV, sdesc_sw128(sA + k * 2048, BOX, 1024),
               sdesc_sw128(sB + k * 2048, BOX, 1024), IDESC_D, 1);
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, mma_phase, abort_flag);
    mma_phase ^= 1;
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    tc_fence_after();

    if (OUT) {
      // ---- phase 4: out = Y + diag(factor) X -> bf16 -> staging (A0's slot);
      //               state -> bf16 copy for the next block's X
      const float as = REV ? pw[cb - row < 0 ? 0 : cb - row] : pw[row + 1];
      uint8_t *stg = T0 + half * BOX;
      uint8_t *kvbf = smem + LY::KVBF + half * BOX;
#pragma unroll
      for (int part = 0; part < 2; part++) {
        const int col = half * 64 + part * 32;
        uint32_t ry[32], rx[32];
        tmem_ld32(tl + LY::COL_Y + col, ry);
        tmem_ld32(tl + LY::COL_X + col, rx);
        tmem_wait_ld();
        float o[32];
#pragma unroll
        for (int j = 0; j < 32; j++) o[j] = __uint_as_float(ry[j]) + as * __uint_as_float(rx[j]);
        st_row_bf16_sw128(stg, row, part * 4, o);
        uint32_t rk[32];
        tmem_ld32(tl + LY::COL_KV + col, rk);
        tmem_wait_ld();
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; j++) f[j] = __uint_as_float(rk[j]);
        st_row_bf16_sw128(kvbf, row, part * 4, f);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tma_store_3d(&tmo, sT0, 0, (int)p, (int)bh);
        tma_store_3d(&tmo, sT0 + BOX, 64, (int)p, (int)bh);
        tma_store_commit();
        tma_store_wait_read0();  // the slot is refilled below
      }
    }
    if (tid == 0 && issued < nblk) {
      issue_load(issued, issued % NS);
      issued++;
    }
  }

  if (!aborted) {
    // final state of the chunk
    float *dst = nullptr;
    float scale = 1.f;
    if (MODE == MODE_FWD) {
      const int64_t so = state_slot(g, bh);
      dst = (kv_out && c == g.S - 1 && so >= 0) ? kv_out + so * 128 * 128 : nullptr;
    }
    if (MODE == MODE_STATE) dst = ws + (bh * g.wsS + c + 1) * (int64_t)128 * 128;
    if (MODE == MODE_RSTATE) dst = ws + (bh * g.wsS + c - 1) * (int64_t)128 * 128;
    if (MODE == MODE_DV && c == 0 && kv_out) {  // dkv0 = lambda * D(0)
      dst = kv_out + bh * 128 * 128;
      scale = lambda[h];
    }
    if (dst) {
#pragma unroll
      for (int part = 0; part < 2; part++) {
        const int col = half * 64 + part * 32;
        uint32_t r[32];
        tmem_ld32(tl + LY::COL_KV + col, r);
        tmem_wait_ld();
        float4 *d4 = reinterpret_cast<float4 *>(dst + (int64_t)row * 128 + col);
#pragma unroll
        for (int j = 0; j < 8; j++)
          d4[j] = make_float4(scale * __uint_as_float(r[4 * j]), scale * __uint_as_float(r[4 * j + 1]),
                              scale * __uint_as_float(r[4 * j + 2]), scale * __uint_as_float(r[4 * j + 3]));
      }
    }
  } else if (tid == 0) {
    // drain the loads still in flight before the shared memory is released,
    // and the MMAs issued (a wait that gave up may have left some running)
    // before TMEM is
    volatile int dummy = 0;
    for (int j = i; j < issued; j++)
      mbar_wait(bar_full0 + 8 * (j % NS), (uint32_t)((j / NS) & 1), &dummy);
    mma_commit(bar_done);
    mbar_wait(bar_done, 0, &dummy);
  }
  if (OUT && tid == 0) tma_store_wait0();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, LY::TMEM_COLS);
  }
}

// ================================================================ v2
// Warp-specialised form of the same schedule.  Roles (448 threads):
//   warp 0       TMA producer (one thread): fills the stage ring
//   warp 1       MMA issuer (one thread)
//   warps 2-5    "mask" warpgroup: P = S (.) M into TMEM
//   warps 6-9    "epilogue" warpgroup: out -> bf16 -> TMA store, state ->
//                bf16 operand copy, state *= lambda^cb for the next block
//   warps 10-13  "decay" warpgroup: row decays of A0 and B1 in shared memory
// The row factor of the state term is folded into A0 (A0 <- diag(f) A0 after
// S = A0 B1^T has read it), so Y and X share one accumulator:
//   O = P B2 + A0f * state.
// TMEM: S double-buffered [0,128) and [128,256), O [256,384), state [384,512);
// the MMA for S of block i+1 is issued while block i is still being masked
// and stored, so tensor-core, CUDA-core and copy work overlap.
constexpr int NT2 = 448;

// Multiply one 64-element row of a swizzled box by f with packed bf16x2
// multiplies (f rounded once to bf16; no unpack/repack through fp32).
__device__ __forceinline__ void scale_row_sw128_bf16(uint8_t *box, int row, __nv_bfloat162 f2) {
#pragma unroll
  for (int c = 0; c < 8; c++) {
    uint4 *p = reinterpret_cast<uint4 *>(box + row * 128 + ((c ^ (row & 7)) << 4));
    uint4 w = *p;
    __nv_bfloat162 *u = reinterpret_cast<__nv_bfloat162 *>(&w);
#pragma unroll
    for (int j = 0; j < 4; j++) u[j] = __hmul2(u[j], f2);
    *p = w;
  }
}

// One 128-element bf16 row of a two-box tile (d 0..63 in the first 128-byte
// swizzled box, 64..127 in the second) as sixteen 16-byte chunks, chunk c
// holding elements 8c..8c+7.  All loads are issued before any result is
// used.
__device__ __forceinline__ void ld_row_sw128(const uint8_t *tile, int row, uint4 (&w)[16]) {
#pragma unroll
  for (int c = 0; c < 16; c++)
    w[c] = *reinterpret_cast<const uint4 *>(tile + (c >> 3) * BOX + row * 128 +
                                            (((c & 7) ^ (row & 7)) << 4));
}
__device__ __forceinline__ void st_row_sw128(uint8_t *tile, int row, const uint4 (&w)[16]) {
#pragma unroll
  for (int c = 0; c < 16; c++)
    *reinterpret_cast<uint4 *>(tile + (c >> 3) * BOX + row * 128 + (((c & 7) ^ (row & 7)) << 4)) =
        w[c];
}

// Multiply one 128-element row of a two-box tile by f2 in place, the whole
// row in flight at once (packed bf16x2 multiplies: f rounded once to bf16).
__device__ __forceinline__ void scale_row2_sw128(uint8_t *tile, int row, __nv_bfloat162 f2) {
  uint4 w[16];
  ld_row_sw128(tile, row, w);
#pragma unroll
  for (int c = 0; c < 16; c++) {
    __nv_bfloat162 *u = reinterpret_cast<__nv_bfloat162 *>(&w[c]);
#pragma unroll
    for (int m = 0; m < 4; m++) u[m] = __hmul2(u[m], f2);
  }
  st_row_sw128(tile, row, w);
}

template <int MODE> struct Layout2 {
  static constexpr bool OUT = Traits<MODE>::OUT;
  static constexpr int NSTAGE = OUT ? 2 : 3;
  static constexpr uint32_t STAGE = OUT ? 3 * TILE : 2 * TILE;
  static constexpr uint32_t KVBF = NSTAGE * STAGE;
  static constexpr uint32_t MISC = KVBF + (OUT ? TILE : 0);
  // Per stage two tile groups with their own full/empty barriers: "ab" =
  // (A0, B1), freed as soon as the block's products are done; "c" = B2,
  // which doubles as the output staging tile and is freed after the store.
  // full_ab[NS] full_c[NS] empty_ab[NS] empty_c[NS] sfull[2] pfull[NS]
  // ofull oempty done
  static constexpr uint32_t NBAR = 5 * NSTAGE + 5;
  static constexpr uint32_t AB_BYTES = OUT ? 2 * TILE : TILE;
  static constexpr uint32_t C_OFF = AB_BYTES;
  // decay tables: twice 32 zeros then lambda^0..lambda^128 (see chunk_kernel2)
  static constexpr uint32_t MISC_BYTES = 8 * NBAR + 16 + 4 * 2 * (32 + BLOCK + 1);
  static constexpr uint32_t SMEM = MISC + MISC_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = OUT ? 512 : 128;
  static constexpr uint32_t COL_O = 256;
  static constexpr uint32_t COL_KV = OUT ? 384 : 0;
};

// OR of `v` over the `n` threads that share named barrier `id`.
__device__ __forceinline__ bool role_any(bool v, int id, int n) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void role_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Trace stamp (only CTA 0 of the traced pass records; events listed where used).
#define LA2_TRACE(ev, blk)                                                                \
  do {                                                                                    \
    if (tracing && (blk) < kTraceBlocks) g_trace[(ev) * kTraceBlocks + (blk)] = globaltimer(); \
  } while (0)

// The MMA issuer's pause between idle probe rounds.
constexpr uint32_t kIdlePauseCycles = 64;
__device__ __forceinline__ uint32_t clock_u32() {
  uint32_t c;
  asm volatile("mov.u32 %0, %%clock;" : "=r"(c));
  return c;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// TRACE: the instantiation that records the trace stamps (LA2_OPT_TRACE);
// the stamps' branches cost a few percent, so the other launches compile
// without them.
// VARLEN: the packed variable-length form (output passes only): one CTA
// per (sequence, head) over rows [cu[n], cu[n+1]) of the head's slab.  A
// sequence's last block reads the next sequence's rows, so the reverse
// passes mask the columns past the block's end and that block's output rows
// go out by plain stores (`outp`) instead of a TMA box.
// KIND: 0 the plain form, 1 the packed (VARLEN) form, 2 the decode-unit form
// (forward only): the B*H (request, head) units of a call of T <= 128 tokens
// per request, head-major, cut into gridDim.x contiguous ranges; each unit is
// one block with its own state, read from and written back to the state
// pool, so one CTA per SM walks ~B*H/SMs units back to back (a range spans
// at most two heads: two decay tables).
constexpr int KIND_PLAIN = 0, KIND_VARLEN = 1, KIND_UNITS = 2;
// The body of one pass for one CTA.  cta / ncta: the CTA's index among the
// pass's CTAs and their number (blockIdx.x / gridDim.x, except in the paired
// reverse pass, where the two CTAs of a cluster serve the same chunk);
// trace_me: this CTA's pass is the traced one (TRACE instantiations only);
// is_dk: MODE_RPAIR only, the CTA computes dK (else dV).
template <int MODE, bool TRACE, int KIND>
__device__ __forceinline__ void
chunk_body(const CUtensorMap *tm0, const CUtensorMap *tm1, const CUtensorMap *tm2,
           const CUtensorMap *tmo, const float *__restrict__ lambda, const float *__restrict__ kv0,
           float *__restrict__ ws, float *__restrict__ kv_out, __nv_bfloat16 *__restrict__ outp,
           const Geo &g, const int64_t cta, const int64_t ncta, const bool trace_me,
           const bool is_dk = false) {
  using LY = Layout2<MODE>;
  using TR = Traits<MODE>;
  constexpr bool VARLEN = KIND == KIND_VARLEN, UNITS = KIND == KIND_UNITS;
  constexpr bool OUT = LY::OUT;
  constexpr bool REV = TR::REV;
  constexpr int NS = LY::NSTAGE;
  // the state term's B operand layout and the state update's operand order
  // (fixed per mode; chosen per CTA in the paired reverse launch)
  const bool X_MN = MODE == MODE_RPAIR ? !is_dk : TR::X_MN;
  const bool SWAP = MODE == MODE_RPAIR ? is_dk : TR::SWAP;
  // the output tensor has 64 columns (the second box is not stored): O and
  // dV have e columns, dQ and dK have d
  const bool out_is_e =
      MODE == MODE_FWD || MODE == MODE_DV || (MODE == MODE_RPAIR && !is_dk);
  const bool out64 = (out_is_e ? g.e : g.d) == 64;
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
  const uint32_t IDESC_X =
      X_MN ? idesc_bf16(128, 128, false, true) : idesc_bf16(128, 128, false, false);
  constexpr uint32_t IDESC_Y = idesc_bf16(128, 128, false, true);
  constexpr uint32_t IDESC_D = idesc_bf16(128, 128, true, true);
  constexpr int BAR_EPI = 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + LY::MISC);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + LY::NBAR);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  // pwz[k] = lambda^(k-32) for 32 <= k <= 160, 0 below: pw = pwz + 32 holds
  // lambda^0..lambda^128 and pw[n] for n in [-32, 0) reads as 0, which is
  // the causal mask (a negative distance means a masked entry; the mask
  // looks up distances down to -31).  pw2, laid out the same way after
  // another 32 zeros, is the next head's table (decode-unit form).
  float *pwz = reinterpret_cast<float *>(tmem_slot + 4);
  float *pw = pwz + 32;
  float *pw2 = pw + (BLOCK + 1) + 32;
  const uint32_t b_fab = smem_u32(bars);
  const uint32_t b_fc = b_fab + 8 * NS;
  const uint32_t b_eab = b_fc + 8 * NS;
  const uint32_t b_ec = b_eab + 8 * NS;
  const uint32_t b_sfull = b_ec + 8 * NS;
  const uint32_t b_pfull = b_sfull + 16;
  const uint32_t b_ofull = b_pfull + 8 * NS;
  const uint32_t b_oempty = b_ofull + 8;
  const uint32_t b_done = b_oempty + 8;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nch = OUT ? g.S : g.nst;
  int64_t bh, a, b, slab;
  int c, h;
  int64_t u0 = 0;  // decode-unit form: the CTA's units [u0, u0 + nblk)
  if constexpr (UNITS) {
    const int64_t U = (int64_t)g.B * g.H;
    u0 = cta * U / ncta;
    const int64_t u1 = (cta + 1) * U / ncta;
    bh = slab = 0;
    c = 0;
    h = (int)(u0 / g.B);  // the range's first head
    a = 0;
    b = u1 - u0;  // one block per unit
  } else if constexpr (VARLEN) {
    int64_t seq = -1;
    if (g.lpt) {  // longest sequences first
      if (warp == 0) {
        const int n = lpt_sequence(g.cu, g.B, (int)(cta / g.H));
        if (lane == 0) tmem_slot[2] = (uint32_t)n;
      }
      __syncthreads();
      seq = tmem_slot[2];
    }
    const Span sp = span_of(g, 1, 0, seq, cta);
    bh = sp.bh, a = sp.a, b = sp.b, slab = sp.slab, c = sp.c, h = sp.h;
  } else {
    bh = cta / nch;
    c = (int)(cta % nch) + (OUT ? 0 : g.c0);
    h = (int)(bh % g.H);
    a = (int64_t)c * g.Lc;
    b = g.L < a + g.Lc ? g.L : a + g.Lc;
    slab = bh;
    // a state-pool request that is inactive (negative slot) or out of the
    // pool (reported by state_slot): no rows
    if (MODE == MODE_FWD && g.slots && (unsigned)g.slots[bh / g.H] >= (unsigned)g.pool) b = a;
  }
  const int nblk = UNITS ? (int)(b - a) : (int)((b - a + BLOCK - 1) / BLOCK);
  auto block_of = [&](int j) { return REV ? nblk - 1 - j : j; };
  auto p_of = [&](int j) { return UNITS ? (int64_t)0 : a + (int64_t)block_of(j) * BLOCK; };
  auto cb_of = [&](int j) {
    const int64_t r = (UNITS ? g.L : b) - p_of(j);
    return (int)(r < BLOCK ? r : BLOCK);
  };
  // decode-unit form: block j is unit u0 + j = (head, request), head-major
  auto unit_head = [&](int j) { return (u0 + j) / g.B; };
  auto slab_of = [&](int j) -> int64_t {
    if constexpr (UNITS) {
      const int64_t hh = unit_head(j);
      return (u0 + j - hh * g.B) * g.H + hh;
    } else {
      return slab;
    }
  };
  // the decay table of block j's head
  auto tab_of = [&](int j) -> const float * {
    if constexpr (UNITS) return unit_head(j) == h ? pw : pw2;
    else return pw;
  };
  // trace events: 0 load issued, 1 S issued, 2 P.B2/X/state issued, 3 mask
  // start, 4 mask done, 5 epilogue start, 6 state handed back, 7 store read
  // done, 8 kernel entry, 9 set-up done, 12 S issue begins, 13 products
  // issue begin, 14 row decays done, 15 output tile staged
  const bool tracing = TRACE && trace_me && cta == 0;
  const bool tracing_all = TRACE;  // per-CTA entry / exit (events 10, 11)
  if (tid == 0) LA2_TRACE(8, 0);
  if (tid == 0 && tracing_all && blockIdx.x < kTraceBlocks)
    g_trace[10 * kTraceBlocks + blockIdx.x] = globaltimer();

  if (tid <= BLOCK) pw[tid] = (float)pow_int((double)lambda[h], tid);
  if (tid < 32) {
    pwz[tid] = 0.f;
    pw[BLOCK + 1 + tid] = 0.f;
  }
  if (UNITS && tid > BLOCK && tid <= 2 * BLOCK + 1)
    pw2[tid - BLOCK - 1] = (float)pow_int((double)lambda[h + 1 < g.H ? h + 1 : h], tid - BLOCK - 1);
  if (tid == 0) {
    for (int s = 0; s < NS; s++) {
      mbar_init(b_fab + 8 * s, 1);
      mbar_init(b_fc + 8 * s, 1);
      mbar_init(b_eab + 8 * s, 1);
      mbar_init(b_ec + 8 * s, 1);
      // P written (mask warps, output passes) and the A0 / B1 row decays
      // applied (decay warps); one arrival per warp
      mbar_init(b_pfull + 8 * s, OUT ? 8 : 4);
    }
    mbar_init(b_sfull, 1);
    mbar_init(b_sfull + 8, 1);
    mbar_init(b_ofull, 1);
    mbar_init(b_oempty, 4);
    mbar_init(b_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (OUT) tma_prefetch_desc(tm0);
    tma_prefetch_desc(tm1);
    tma_prefetch_desc(tm2);
    if (OUT) tma_prefetch_desc(tmo);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), LY::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) LA2_TRACE(9, 0);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int nab = 0, nc = 0;  // blocks whose (A0, B1) / B2 loads were issued
      for (int j = 0; j < nblk; j++) {
        const int st = j % NS;
        const uint32_t ph = (uint32_t)((j / NS - 1) & 1);
        const int y = (int)p_of(j), z = (int)slab_of(j);
        uint32_t dst = sbase + st * LY::STAGE;
        // (A0, B1): their slots free once block j-NS's products are done
        if (j >= NS && !mbar_wait(b_eab + 8 * st, ph, abort_flag)) break;
        mbar_expect_tx(b_fab + 8 * st, LY::AB_BYTES);
        if (OUT) {
          tma_load_3d(dst, tm0, b_fab + 8 * st, 0, y, z);
          tma_load_3d(dst + BOX, tm0, b_fab + 8 * st, 64, y, z);
          dst += TILE;
        }
        tma_load_3d(dst, tm1, b_fab + 8 * st, 0, y, z);
        tma_load_3d(dst + BOX, tm1, b_fab + 8 * st, 64, y, z);
        nab++;
        // B2: its slot free once block j-NS's output has left it
        if (j >= NS && !mbar_wait(b_ec + 8 * st, ph, abort_flag)) break;
        dst = sbase + st * LY::STAGE + LY::C_OFF;
        mbar_expect_tx(b_fc + 8 * st, TILE);
        tma_load_3d(dst, tm2, b_fc + 8 * st, 0, y, z);
        tma_load_3d(dst + BOX, tm2, b_fc + 8 * st, 64, y, z);
        nc++;
        LA2_TRACE(0, j);
      }
      // every issued load has landed before shared memory is released
      volatile int never = 0;
      for (int k = nab - NS < 0 ? 0 : nab - NS; k < nab; k++)
        mbar_wait(b_fab + 8 * (k % NS), (uint32_t)((k / NS) & 1), &never);
      for (int k = nc - NS < 0 ? 0 : nc - NS; k < nc; k++)
        mbar_wait(b_fc + 8 * (k % NS), (uint32_t)((k / NS) & 1), &never);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      auto stage_addr = [&](int j) { return sbase + (j % NS) * LY::STAGE; };
      auto issue_S = [&](int j) {
        const uint32_t sA0 = stage_addr(j), sB1 = sA0 + TILE;
        const uint32_t d = tmem + 128u * (uint32_t)(j & 1);
#pragma unroll
        for (int k = 0; k < 8; k++) {
          const uint32_t koff = (k >> 2) * BOX + (k & 3) * 32;
          mma_ss(d, sdesc_sw128(sA0 + koff, 16, 1024), sdesc_sw128(sB1 + koff, 16, 1024),
                 IDESC_S, k > 0);
        }
        mma_commit(b_sfull + 8 * (j & 1));
        LA2_TRACE(1, j);
      };
      auto issue_P3 = [&](int i) {
        const uint32_t sA0 = stage_addr(i);
        const uint32_t sB1 = OUT ? sA0 + TILE : sA0;
        const uint32_t sB2 = sA0 + LY::C_OFF;
        if (OUT) {
          const uint32_t pa = tmem + 128u * (uint32_t)(i & 1);
          const uint32_t sKV = sbase + LY::KVBF;
#pragma unroll
          for (int k = 0; k < 8; k++)
            mma_ts(tmem + LY::COL_O, pa + 8 * k, sdesc_sw128(sB2 + k * 2048, BOX, 1024), IDESC_Y,
                   k > 0);
#pragma unroll
          for (int k = 0; k < 8; k++) {
            const uint32_t koff = (k >> 2) * BOX + (k & 3) * 32;
            const uint64_t bd = X_MN ? sdesc_sw128(sKV + k * 2048, BOX, 1024)
                                     : sdesc_sw128(sKV + koff, 16, 1024);
            mma_ss(tmem + LY::COL_O, sdesc_sw128(sA0 + koff, 16, 1024), bd, IDESC_X, 1);
          }
        }
        const uint32_t sA = SWAP ? sB2 : sB1;
        const uint32_t sB = SWAP ? sB1 : sB2;
#pragma unroll
        for (int k = 0; k < 8; k++)
          mma_ss(tmem + LY::COL_KV, sdesc_sw128(sA + k * 2048, BOX, 1024),
                 sdesc_sw128(sB + k * 2048, BOX, 1024), IDESC_D, 1);
        // test hook: CTA 0 withholds its first completion signal
        if (!(g.inject && blockIdx.x == 0 && i == 0)) mma_commit(b_ofull);
        mma_commit(b_eab + 8 * (i % NS));  // A0, B1 slots reusable
        LA2_TRACE(2, i);
      };
      // Two streams of work are issued as their inputs become ready, polled
      // without blocking: S of block j (tiles loaded, its TMEM buffer free,
      // i.e. the products of block j-2 done) and the products of block i (P
      // and row decays ready, state handed back).  The products take
      // priority.  nS / nP count issued S / product groups, seen counts
      // completed product groups; at most one product group is in flight and
      // S of block j needs products j-2 done, so no waiter can fall two
      // phases behind a barrier.
      int nS = 0, nP = 0, seen = 0;
      uint32_t idle = 0;
      uint64_t t_last = globaltimer();
      while (nP < nblk) {
        bool did = false;
        if (OUT && nS < nblk && seen >= nS - 1 &&
            mbar_test(b_fab + 8 * (nS % NS), (uint32_t)((nS / NS) & 1))) {
          tc_fence_after();
          LA2_TRACE(12, nS);
          issue_S(nS);
          nS++;
          did = true;
        }
        if ((!OUT || nS > nP) && seen >= nP &&
            mbar_test(b_pfull + 8 * (nP % NS), (uint32_t)((nP / NS) & 1)) &&
            mbar_test(b_fc + 8 * (nP % NS), (uint32_t)((nP / NS) & 1)) &&
            mbar_test(b_oempty, (uint32_t)(nP & 1))) {
          tc_fence_after();
          LA2_TRACE(13, nP);
          issue_P3(nP);
          nP++;
          did = true;
        }
        if (seen < nP && mbar_test(b_ofull, (uint32_t)(seen & 1))) {
          seen++;
          did = true;
        }
        if (did) {
          idle = 0;
        } else if ((++idle & 63) == 0) {
          // an idle probe round costs shared-memory cycles the other roles
          // need, so the abort flag and the clock are read every 64th round
          if (*abort_flag) break;
          const uint64_t now = globaltimer();
          if (idle == 64) t_last = now;
          if (now - t_last > kWaitTimeoutNs) {
            *abort_flag = 1;
            raise_error(ERR_TIMEOUT);
            break;
          }
        } else {
          const uint32_t c0 = clock_u32();
          while (clock_u32() - c0 < kIdlePauseCycles) {
          }
        }
      }
      // all MMAs issued by this thread have finished before TMEM is freed
      mma_commit(b_done);
      volatile int never = 0;
      mbar_wait(b_done, 0, &never);
    }
  } else if (warp < 6) {
    // -------------------------------------------------------- mask warps
    // Warp quarter q owns rows 32q..32q+31 and splits S into four 32-column
    // parts p.  Parts wholly above the diagonal (below it in the reverse
    // passes) are zero; the diagonal part p == q looks its factors up in the
    // zero-extended table; in the other parts the factor of column 32p + k
    // is a * lambda^(31-k) with a = lambda^(row-32p-31) (reverse: a *
    // lambda^k, a = lambda^(32p-row)), a <= 1, generated by two chains of
    // multiplications by lambda^2 from the largest factor down: no
    // shared-memory lookup per element, and at most 16 roundings per factor.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    float lam1 = pw[1], lam2 = pw[2];
    for (int i = 0; OUT && i < nblk; i++) {
      const int st = i % NS;
      const float *pt = tab_of(i);
      if constexpr (UNITS) {
        lam1 = pt[1];
        lam2 = pt[2];
      }
      bool ok = mbar_wait(b_sfull + 8 * (i & 1), (uint32_t)((i >> 1) & 1), abort_flag);
      // a warp vote suffices: no later step syncs the mask warps together
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      if (row == 0) LA2_TRACE(3, i);
      const uint32_t sb = 128u * (uint32_t)(i & 1);
#pragma unroll
      for (int part = 0; part < 4; part++) {
        uint32_t pk[16];
        if (REV ? part < q : part > q) {
#pragma unroll
          for (int j = 0; j < 16; j++) pk[j] = 0u;
        } else {
          uint32_t r[32];
          tmem_ld32(tl + sb + part * 32, r);
          tmem_wait_ld();
          if constexpr (VARLEN && REV) {
            // columns past the block's end belong to the next sequence
            const int cbi = cb_of(i);
            if (cbi < BLOCK) {
#pragma unroll
              for (int k = 0; k < 32; k++)
                if (part * 32 + k >= cbi) r[k] = 0u;
            }
          }
          if (part == q) {
#pragma unroll
            for (int j = 0; j < 16; j++) {
              // distance < 0 reads 0 from the table: the causal mask
              const int n0 = REV ? 2 * j - lane : lane - 2 * j;
              const float f0 = __uint_as_float(r[2 * j]) * pt[n0];
              const float f1 = __uint_as_float(r[2 * j + 1]) * pt[REV ? n0 + 1 : n0 - 1];
              pk[j] = pack_bf16x2(f0, f1);
            }
          } else {
            const float a = REV ? pt[32 * part - row] : pt[row - 32 * part - 31];
            // xe, xo: factors of the pair's even and odd column
            float xe = REV ? a : a * lam1, xo = REV ? a * lam1 : a;
#pragma unroll
            for (int jj = 0; jj < 16; jj++) {
              const int j = REV ? jj : 15 - jj;
              pk[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * xe, __uint_as_float(r[2 * j + 1]) * xo);
              xe *= lam2;
              xo *= lam2;
            }
          }
        }
        tmem_st16(tl + sb + part * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      if (row == 0) LA2_TRACE(4, i);
      __syncwarp();
      if (lane == 0) mbar_arrive(b_pfull + 8 * st);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------- epilogue warps
    const int row = (warp & 3) * 32 + lane;
    const int wtid = tid - 6 * 32;  // 0..127
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint8_t *kvbf = smem + LY::KVBF;
    // a state into TMEM (already decayed by `dec` for its first block's
    // update) and, output passes, its bf16 operand copy; NULL: zero
    auto load_state = [&](const float *init, float dec) {
#pragma unroll
      for (int part = 0; part < 4; part++) {
        float f[32];
        if (init) {
          const float4 *src = reinterpret_cast<const float4 *>(init + (int64_t)row * 128 + part * 32);
#pragma unroll
          for (int j = 0; j < 8; j++) {
            float4 x = src[j];
            f[4 * j] = x.x; f[4 * j + 1] = x.y; f[4 * j + 2] = x.z; f[4 * j + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; j++) f[j] = 0.f;
        }
        if (OUT) st_row_bf16_sw128(kvbf + (part >> 1) * BOX, row, (part & 1) * 4, f);
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 32; j++) r[j] = __float_as_uint(f[j] * dec);
        tmem_st32(tl + LY::COL_KV + part * 32, r);
      }
    };
    // decode-unit form: block j's state in the pool (NULL: inactive request)
    auto unit_state = [&](float *pool, int j) -> float * {
      const int64_t so = state_slot(g, slab_of(j));
      return (pool && so >= 0) ? pool + so * 128 * 128 : nullptr;
    };
    // initial state: TMEM (already decayed for block 0's update), bf16 copy
    {
      const float *init = nullptr;
      if (UNITS) {
        init = nblk > 0 ? unit_state(const_cast<float *>(kv0), 0) : nullptr;
      } else if (MODE == MODE_FWD || MODE == MODE_DQ) {
        // a split pass reads every chunk's entry state from the workspace (the
        // scan put the initial one in slot 0), never kv0, which kv_out may reuse
        if (g.S > 1) {
          init = ws + (bh * g.wsS + (int64_t)c * g.M) * (int64_t)128 * 128;
        } else {
          const int64_t so = state_slot(g, bh);
          init = (kv0 && so >= 0) ? kv0 + so * 128 * 128 : nullptr;
        }
      } else if (MODE == MODE_DV || MODE == MODE_DK || MODE == MODE_RPAIR) {
        // the last chunk starts from the reverse state past the sequence end
        // (kv0 carries it in the reverse passes; NULL: zero)
        if (c != g.S - 1) init = ws + (bh * g.wsS + (int64_t)(c + 1) * g.M - 1) * (int64_t)128 * 128;
        else init = kv0 ? kv0 + bh * 128 * 128 : nullptr;
      }
      load_state(init, tab_of(0)[nblk > 0 ? cb_of(0) : 0]);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_oempty);
    }
    float *dst = nullptr;
    float dscale = 1.f;
    if (MODE == MODE_FWD) {
      const int64_t so = state_slot(g, bh);
      dst = (kv_out && c == g.S - 1 && so >= 0) ? kv_out + so * 128 * 128 : nullptr;
    }
    if (MODE == MODE_STATE) dst = ws + (bh * g.wsS + c + 1) * (int64_t)128 * 128;
    if (MODE == MODE_RSTATE) dst = ws + (bh * g.wsS + c - 1) * (int64_t)128 * 128;
    if ((MODE == MODE_DV || (MODE == MODE_RPAIR && !is_dk)) && c == 0 && kv_out) {
      dst = kv_out + bh * 128 * 128;  // dkv0 = lambda * D(0)
      dscale = lambda[h];
    }
    for (int i = 0; i < nblk; i++) {
      const int st = i % NS;
      bool ok = mbar_wait(b_ofull, (uint32_t)(i & 1), abort_flag);
      if (role_any(!ok, BAR_EPI, 128)) break;
      tc_fence_after();
      if (wtid == 0) LA2_TRACE(5, i);
      uint8_t *stg = smem + st * LY::STAGE + LY::C_OFF;  // B2's slot
      if (OUT) {
#pragma unroll
        for (int pair = 0; pair < 2; pair++) {
          uint32_t r[64];
          tmem_ld32(tl + LY::COL_O + pair * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(tl + LY::COL_O + pair * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_wait_ld();
          st_row_bf16_sw128(stg + pair * BOX, row, 0, reinterpret_cast<const float *>(&r[0]));
          st_row_bf16_sw128(stg + pair * BOX, row, 4, reinterpret_cast<const float *>(&r[32]));
        }
      }
      if (wtid == 0) LA2_TRACE(15, i);
      // every unit of the decode-unit form ends with its only block
      const bool last = UNITS || i == nblk - 1;
      const float dec = last ? 1.f : tab_of(i + 1)[cb_of(i + 1)];
      float *dst_i = dst;
      if constexpr (UNITS) dst_i = unit_state(kv_out, i);
#pragma unroll
      for (int pair = 0; pair < 2; pair++) {
        uint32_t r[64];
        tmem_ld32(tl + LY::COL_KV + pair * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(tl + LY::COL_KV + pair * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_wait_ld();
        if (!last) {
          if (OUT) {
            st_row_bf16_sw128(kvbf + pair * BOX, row, 0, reinterpret_cast<const float *>(&r[0]));
            st_row_bf16_sw128(kvbf + pair * BOX, row, 4, reinterpret_cast<const float *>(&r[32]));
          }
#pragma unroll
          for (int j = 0; j < 64; j++) r[j] = __float_as_uint(__uint_as_float(r[j]) * dec);
          tmem_st32(tl + LY::COL_KV + pair * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_st32(tl + LY::COL_KV + pair * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        } else if (dst_i) {
          float4 *d4 = reinterpret_cast<float4 *>(dst_i + (int64_t)row * 128 + pair * 64);
#pragma unroll
          for (int j = 0; j < 16; j++)
            d4[j] = make_float4(dscale * __uint_as_float(r[4 * j]), dscale * __uint_as_float(r[4 * j + 1]),
                                dscale * __uint_as_float(r[4 * j + 2]), dscale * __uint_as_float(r[4 * j + 3]));
        }
      }
      if constexpr (UNITS) {
        // the next unit's state (its rows were prefetched into L2 a block
        // ago), and the one after it on its way to L2
        if (i + 1 < nblk) load_state(unit_state(const_cast<float *>(kv0), i + 1), tab_of(i + 1)[cb_of(i + 1)]);
        if (i + 2 < nblk) {
          const float *nx = unit_state(const_cast<float *>(kv0), i + 2);
          if (nx) {
#pragma unroll
            for (int k = 0; k < 4; k++)
              asm volatile("prefetch.global.L2 [%0];" ::"l"(nx + (int64_t)row * 128 + k * 32));
          }
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      if (wtid == 0) LA2_TRACE(6, i);
      __syncwarp();
      if (lane == 0) mbar_arrive(b_oempty);
      if (OUT) role_sync(BAR_EPI, 128);  // the whole output tile is in shared memory
      bool tail_rows = false;
      if constexpr (VARLEN) {
        // the sequence's last, partial block: its rows only, by plain stores
        const int cbi = cb_of(i);
        if (cbi < BLOCK) {
          tail_rows = true;
          if (row < cbi) {
            uint4 w[16];
            ld_row_sw128(stg, row, w);
            uint4 *gdst = reinterpret_cast<uint4 *>(outp + ((int64_t)slab * g.L + p_of(i) + row) * 128);
#pragma unroll
            for (int k = 0; k < 16; k++) gdst[k] = w[k];
          }
          role_sync(BAR_EPI, 128);  // the staging tile has been read
        }
      }
      if (wtid == 0) {
        // (an inactive request of the decode-unit form keeps its outputs)
        if (OUT && !tail_rows && (!UNITS || unit_state(kv_out, i))) {
          const uint32_t sst = sbase + st * LY::STAGE + LY::C_OFF;
          const int y = (int)p_of(i), z = (int)slab_of(i);
          tma_store_3d(tmo, sst, 0, y, z);
          if (!out64) tma_store_3d(tmo, sst + BOX, 64, y, z);
          tma_store_commit();
          tma_store_wait_read0();
        }
        LA2_TRACE(7, i);
        mbar_arrive(b_ec + 8 * st);  // B2 slot reusable
      }
    }
    if constexpr (VARLEN) {
      // an empty sequence: its final state is the initial one, dkv0 is 0
      if (nblk == 0 && dst) {
        const float *src0 = (MODE == MODE_FWD && kv0) ? kv0 + bh * 128 * 128 : nullptr;
        for (int k = 0; k < 128; k++)
          dst[(int64_t)row * 128 + k] = src0 ? src0[(int64_t)row * 128 + k] : 0.f;
      }
    }
    if (OUT && wtid == 0) tma_store_wait0();
  } else {
    // ------------------------------------------------------- decay warps
    // Row decays, in place, once S has read the tiles: A0 rows by the state
    // term's factor (output passes), B1 rows by the state update's decay.
    const int row = (warp & 3) * 32 + lane;
    for (int j = 0; j < nblk; j++) {
      const int st = j % NS;
      const int cbj = cb_of(j);
      const bool ok = OUT ? mbar_wait(b_sfull + 8 * (j & 1), (uint32_t)((j >> 1) & 1), abort_flag)
                          : mbar_wait(b_fab + 8 * st, (uint32_t)((j / NS) & 1), abort_flag);
      if (__any_sync(0xffffffffu, !ok)) break;  // as for the mask warps
      uint8_t *stage = smem + st * LY::STAGE;
      const float *pt = tab_of(j);
      if (OUT) {
        const float f = REV ? (row < cbj ? pt[cbj - row] : 0.f) : pt[row + 1];
        scale_row2_sw128(stage, row, __float2bfloat162_rn(f));
      }
      uint8_t *B1 = OUT ? stage + TILE : stage;
      const float fb = row < cbj ? (REV ? pt[row] : pt[cbj - 1 - row]) : 0.f;
      scale_row2_sw128(B1, row, __float2bfloat162_rn(fb));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_pfull + 8 * st);
      if (row == 0) LA2_TRACE(14, j);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && tracing_all && blockIdx.x < kTraceBlocks)
    g_trace[11 * kTraceBlocks + blockIdx.x] = globaltimer();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, LY::TMEM_COLS);
  }
}

template <int MODE, bool TRACE, int KIND>
__global__ void __launch_bounds__(NT2, 1)
chunk_kernel2(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
              const __grid_constant__ CUtensorMap tm2, const __grid_constant__ CUtensorMap tmo,
              const float *__restrict__ lambda, const float *__restrict__ kv0,
              float *__restrict__ ws, float *__restrict__ kv_out, __nv_bfloat16 *__restrict__ outp,
              Geo g) {
  chunk_body<MODE, TRACE, KIND>(&tm0, &tm1, &tm2, &tmo, lambda, kv0, ws, kv_out, outp, g,
                                blockIdx.x, gridDim.x, true);
}

// The reverse scan's two output passes in one launch: clusters of two CTAs,
// both on the same chunk, the even one writing dV (tiles K, Q, dO) and the
// odd one dK (tiles V, dO, Q).  Each carries its own copy of the reverse
// state D and neither waits for the other, but a cluster's CTAs start
// together and walk the same blocks at the same pace, so the Q and dO tiles
// one of them loads are still in L2 when the other asks for them: per block
// the pair reads K, Q, dO, V from HBM once and writes dK and dV, where two
// separate passes read Q and dO twice.  dkv0 comes from the dV member.
template <bool TRACE, int KIND>
__global__ void __launch_bounds__(NT2, 1)
rev_pair_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tq,
                const __grid_constant__ CUtensorMap tg, const __grid_constant__ CUtensorMap tv,
                const __grid_constant__ CUtensorMap tdv, const __grid_constant__ CUtensorMap tdk,
                const float *__restrict__ lambda, const float *__restrict__ dend,
                float *__restrict__ ws, float *__restrict__ dkv0, __nv_bfloat16 *__restrict__ outp_dv,
                __nv_bfloat16 *__restrict__ outp_dk, Geo g) {
  const int64_t cta = blockIdx.x >> 1, ncta = gridDim.x >> 1;
  const bool dk = blockIdx.x & 1;
  chunk_body<MODE_RPAIR, TRACE, KIND>(dk ? &tv : &tk, dk ? &tg : &tq, dk ? &tq : &tg,
                                      dk ? &tdk : &tdv, lambda, dend, ws, dk ? nullptr : dkv0,
                                      dk ? outp_dk : outp_dv, g, cta, ncta,
                                      g.trace == (dk ? MODE_DK : MODE_DV), dk);
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [BH, L, W] bf16 (W = 128 or 64), boxes of 128 rows x 64 columns, 128-byte
// swizzle; rows outside [0, L) read as zero and are not written.  With W =
// 64 the kernels' second box (columns 64..127) lies wholly outside the
// tensor: it loads as zeros (the head size padded to 128 with zero columns,
// which every product carries through exactly) and is not stored.
inline bool make_map(CUtensorMap *m, const void *ptr, int64_t BH, int64_t L, int W = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)L, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)W * 2, (cuuint64_t)L * W * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_chunk(const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &m2,
                         const CUtensorMap &mo, const float *lam, const float *kv0, float *ws,
                         float *kv_out, const Geo &g, cudaStream_t st, void *outp = nullptr) {
  const int64_t nch = Layout<MODE>::OUT ? g.S : g.nst;
  const int64_t grid = (int64_t)g.B * g.H * nch;
  if (g.variant == 1) {  // first (phase-serial) form of the kernel
    using LY = Layout<MODE>;
    auto k = chunk_kernel<MODE>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::SMEM);
    if (e != cudaSuccess) return e;
    k<<<(unsigned)grid, NT, LY::SMEM, st>>>(m0, m1, m2, mo, lam, kv0, ws, kv_out, g);
    return cudaGetLastError();
  }
  using LY = Layout2<MODE>;
  auto k = g.trace == MODE ? chunk_kernel2<MODE, true, KIND_PLAIN> : chunk_kernel2<MODE, false, KIND_PLAIN>;
  if constexpr (LY::OUT) {
    if (g.cu) k = chunk_kernel2<MODE, false, KIND_VARLEN>;
  }
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::SMEM);
  if (e != cudaSuccess) return e;
  k<<<(unsigned)grid, NT2, LY::SMEM, st>>>(m0, m1, m2, mo, lam, kv0, ws, kv_out,
                                          static_cast<__nv_bfloat16 *>(outp), g);
  return cudaGetLastError();
}

// The paired reverse pass (rev_pair_kernel): 2 CTAs per chunk, launched as
// clusters of two so that both members of a pair run at the same time.
template <int KIND>
cudaError_t launch_pair(const CUtensorMap &mk, const CUtensorMap &mq, const CUtensorMap &mg,
                        const CUtensorMap &mv, const CUtensorMap &mdv, const CUtensorMap &mdk,
                        const float *lam, const float *dend, float *ws, float *dkv0, void *outp_dv,
                        void *outp_dk, const Geo &g, cudaStream_t st) {
  using LY = Layout2<MODE_DV>;
  static_assert(Layout2<MODE_DV>::SMEM == Layout2<MODE_RPAIR>::SMEM, "the pair's layout");
  const int64_t units = (int64_t)g.B * g.H * g.S;
  const bool trace = g.trace == MODE_DV || g.trace == MODE_DK;
  auto k = trace ? rev_pair_kernel<true, KIND> : rev_pair_kernel<false, KIND>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * units));
  cfg.blockDim = dim3(NT2);
  cfg.dynamicSmemBytes = LY::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, mk, mq, mg, mv, mdv, mdk, lam, dend, ws, dkv0,
                            static_cast<__nv_bfloat16 *>(outp_dv),
                            static_cast<__nv_bfloat16 *>(outp_dk), g);
}

// States [BH, d, e] fp32 <-> [BH, 128, 128] fp32 with zeros outside d x e
// (the tensor-core passes' state shape for 64-column heads).
__global__ void pad_state_kernel(const float *__restrict__ src, float *__restrict__ dst, int d,
                                 int e) {
  const int64_t bh = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // < 128 * 128
  const int r = idx >> 7, c = idx & 127;
  dst[bh * 16384 + idx] = (r < d && c < e) ? src[(bh * d + r) * e + c] : 0.f;
}
__global__ void unpad_state_kernel(const float *__restrict__ src, float *__restrict__ dst, int d,
                                   int e) {
  const int64_t bh = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // < d * e
  if (idx >= d * e) return;
  const int r = idx / e, c = idx % e;
  dst[bh * d * e + idx] = src[bh * 16384 + r * 128 + c];
}
inline void pad_states(const float *src, float *dst, int64_t BH, int d, int e, cudaStream_t st) {
  pad_state_kernel<<<dim3(16384 / 256, (unsigned)BH), 256, 0, st>>>(src, dst, d, e);
}
inline void unpad_states(const float *src, float *dst, int64_t BH, int d, int e, cudaStream_t st) {
  unpad_state_kernel<<<dim3((d * e + 255) / 256, (unsigned)BH), 256, 0, st>>>(src, dst, d, e);
}

inline bool geometry_ok(const Geo &g) {
  return g.L < (int64_t(1) << 31) && (int64_t)g.B * g.H < (int64_t(1) << 31);
}

// Forward: [chunk states + scan] + main pass.
template <typename Timed>
cudaError_t forward(const void *q, const void *k, const void *v, const float *lam,
                    const float *kv0, void *o, float *kv_out, float *ws, const Geo &g,
                    cudaStream_t st, Timed &&timed) {
  if (!geometry_ok(g)) return cudaErrorInvalidValue;
  const int64_t BH = (int64_t)g.B * g.H;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, BH, g.L, g.d) || !make_map(&mk, k, BH, g.L, g.d) ||
      !make_map(&mv, v, BH, g.L, g.e) || !make_map(&mo, o, BH, g.L, g.e))
    return cudaErrorInvalidValue;
  cudaError_t err = cudaSuccess;
  if (g.S > 1) {
    const Geo gs = state_geo(g, false);
    err = timed(0, [&] { launch_chunk<MODE_STATE>(mk, mk, mv, mk, lam, nullptr, ws, nullptr, gs, st); });
    if (err) return err;
    err = timed(1, [&] {
      la2::simt::scan_fwd_kernel<128, 128>
          <<<dim3(128 * 128 / la2::simt::NT, (unsigned)BH), la2::simt::NT, 0, st>>>(ws, kv0, lam, gs);
    });
    if (err) return err;
  }
  return timed(2, [&] { launch_chunk<MODE_FWD>(mq, mk, mv, mo, lam, kv0, ws, kv_out, g, st, o); });
}

// Backward: dQ by a forward scan (chunk states of K, V + scan), then dV and
// dK by reverse scans (chunk states of Q, dO + reverse scan); dkv0 comes
// out of the dV pass's first chunk.  gr is the reverse passes' chunk plan:
// with gr.rev_pair the dV and dK passes run as one paired launch, two CTAs
// per chunk, so gr splits each sequence for half as many chunks as g (the
// reverse pre-pass then covers fewer chunk boundaries).  The reverse states
// follow the forward ones in the workspace.
template <typename Timed>
cudaError_t backward(const void *q, const void *k, const void *v, const float *lam,
                     const float *kv0, const void *dO, void *dq, void *dk, void *dv, float *dkv0,
                     float *ws, const Geo &g, const Geo &gr, bool reuse_fwd, cudaStream_t st,
                     Timed &&timed, const float *dend = nullptr) {
  if (!geometry_ok(g) || !geometry_ok(gr)) return cudaErrorInvalidValue;
  const int64_t BH = (int64_t)g.B * g.H;
  CUtensorMap mq, mk, mv, mg, mdq, mdk, mdv;
  if (!make_map(&mq, q, BH, g.L, g.d) || !make_map(&mk, k, BH, g.L, g.d) ||
      !make_map(&mv, v, BH, g.L, g.e) || !make_map(&mg, dO, BH, g.L, g.e) ||
      !make_map(&mdq, dq, BH, g.L, g.d) || !make_map(&mdk, dk, BH, g.L, g.d) ||
      !make_map(&mdv, dv, BH, g.L, g.e))
    return cudaErrorInvalidValue;
  float *wsf = ws;
  float *wsr = ws ? ws + (g.S > 1 ? (size_t)BH * g.wsS * 128 * 128 : 0) : nullptr;
  const dim3 sgrid(128 * 128 / la2::simt::NT, (unsigned)BH);
  const Geo gf = state_geo(g, false), grs = state_geo(gr, true);
  cudaError_t err = cudaSuccess;
  // the forward pass leaves the same chunk entry states in the same place
  if (g.S > 1 && !reuse_fwd) {
    err = timed(0, [&] { launch_chunk<MODE_STATE>(mk, mk, mv, mk, lam, nullptr, wsf, nullptr, gf, st); });
    if (err) return err;
    err = timed(1, [&] {
      la2::simt::scan_fwd_kernel<128, 128><<<sgrid, la2::simt::NT, 0, st>>>(wsf, kv0, lam, gf);
    });
    if (err) return err;
  }
  err = timed(2, [&] { launch_chunk<MODE_DQ>(mg, mv, mk, mdq, lam, kv0, wsf, nullptr, g, st, dq); });
  if (err) return err;
  if (gr.S > 1) {
    err = timed(3, [&] { launch_chunk<MODE_RSTATE>(mq, mq, mg, mq, lam, nullptr, wsr, nullptr, grs, st); });
    if (err) return err;
    err = timed(4, [&] {
      la2::simt::scan_rev_kernel<128, 128><<<sgrid, la2::simt::NT, 0, st>>>(wsr, lam, dend, grs);
    });
    if (err) return err;
  }
  if (gr.rev_pair)
    return timed(7, [&] {
      return launch_pair<KIND_PLAIN>(mk, mq, mg, mv, mdv, mdk, lam, dend, wsr, dkv0, nullptr, nullptr,
                                     gr, st);
    });
  err = timed(5, [&] { launch_chunk<MODE_DV>(mk, mq, mg, mdv, lam, dend, wsr, dkv0, gr, st, dv); });
  if (err) return err;
  return timed(6, [&] { launch_chunk<MODE_DK>(mv, mg, mq, mdk, lam, dend, wsr, nullptr, gr, st, dk); });
}

// Decode units: T <= 128 new tokens for each of B requests x H heads, [B,H,T,.]
// tensors, the state of (b,h) in the pool at slot slots[b] (b without a
// table) read and written in place; `ctas` CTAs walk the B*H units, head-
// major, one block each (the decode-unit form of chunk_kernel2).
template <typename Timed>
cudaError_t decode_units(const void *q, const void *k, const void *v, const float *lam,
                         float *pool, void *o, const Geo &g, int ctas, cudaStream_t st,
                         Timed &&timed) {
  const int64_t BH = (int64_t)g.B * g.H;
  if (!geometry_ok(g) || g.L < 1 || g.L > BLOCK || ctas < 1 || ctas > BH)
    return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, BH, g.L) || !make_map(&mk, k, BH, g.L) || !make_map(&mv, v, BH, g.L) ||
      !make_map(&mo, o, BH, g.L))
    return cudaErrorInvalidValue;
  using LY = Layout2<MODE_FWD>;
  auto kern = g.trace == MODE_FWD ? chunk_kernel2<MODE_FWD, true, KIND_UNITS>
                                  : chunk_kernel2<MODE_FWD, false, KIND_UNITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::SMEM);
  if (e != cudaSuccess) return e;
  return timed(2, [&] {
    kern<<<(unsigned)ctas, NT2, LY::SMEM, st>>>(mq, mk, mv, mo, lam, pool, nullptr, pool, nullptr, g);
  });
}

// Chunk-state pass over every sub-chunk of a shard (a: K or Q, b: V or dO):
// forward deltas into workspace slots 1..nst, reverse deltas into slots
// 0..nst-1 (the reverse pass writes slot c-1 for sub-chunk c, so its base is
// one slot further on).
template <typename Timed>
cudaError_t shard_state(const void *a, const void *b, const float *lam, float *ws,
                        const Geo &gs, bool reverse, cudaStream_t st, Timed &&timed) {
  if (!geometry_ok(gs)) return cudaErrorInvalidValue;
  const int64_t BH = (int64_t)gs.B * gs.H;
  CUtensorMap ma, mb;
  if (!make_map(&ma, a, BH, gs.L) || !make_map(&mb, b, BH, gs.L)) return cudaErrorInvalidValue;
  if (!reverse)
    return timed(0, [&] { launch_chunk<MODE_STATE>(ma, ma, mb, ma, lam, nullptr, ws, nullptr, gs, st); });
  return timed(3, [&] {
    launch_chunk<MODE_RSTATE>(ma, ma, mb, ma, lam, nullptr, ws + 128 * 128, nullptr, gs, st);
  });
}

// Packed variable-length batch: g.B = N sequences, g.L = T rows per head
// slab, g.cu the device offsets, S = 1 (one CTA per (sequence, head)).
// Tensor maps run over [H, T, 128].
template <typename Timed>
cudaError_t forward_varlen(const void *q, const void *k, const void *v, const float *lam,
                           const float *kv0, void *o, float *kv_out, const Geo &g,
                           cudaStream_t st, Timed &&timed) {
  if (!geometry_ok(g) || !g.cu || g.S != 1) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, q, g.H, g.L) || !make_map(&mk, k, g.H, g.L) || !make_map(&mv, v, g.H, g.L) ||
      !make_map(&mo, o, g.H, g.L))
    return cudaErrorInvalidValue;
  return timed(2, [&] { launch_chunk<MODE_FWD>(mq, mk, mv, mo, lam, kv0, nullptr, kv_out, g, st, o); });
}

template <typename Timed>
cudaError_t backward_varlen(const void *q, const void *k, const void *v, const float *lam,
                            const float *kv0, const void *dO, void *dq, void *dk, void *dv,
                            float *dkv0, const Geo &g, cudaStream_t st, Timed &&timed) {
  if (!geometry_ok(g) || !g.cu || g.S != 1) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mg, mdq, mdk, mdv;
  if (!make_map(&mq, q, g.H, g.L) || !make_map(&mk, k, g.H, g.L) || !make_map(&mv, v, g.H, g.L) ||
      !make_map(&mg, dO, g.H, g.L) || !make_map(&mdq, dq, g.H, g.L) ||
      !make_map(&mdk, dk, g.H, g.L) || !make_map(&mdv, dv, g.H, g.L))
    return cudaErrorInvalidValue;
  cudaError_t err = timed(2, [&] {
    launch_chunk<MODE_DQ>(mg, mv, mk, mdq, lam, kv0, nullptr, nullptr, g, st, dq);
  });
  if (err) return err;
  if (g.rev_pair)
    return timed(7, [&] {
      return launch_pair<KIND_VARLEN>(mk, mq, mg, mv, mdv, mdk, lam, nullptr, nullptr, dkv0, dv, dk,
                                      g, st);
    });
  err = timed(5, [&] { launch_chunk<MODE_DV>(mk, mq, mg, mdv, lam, nullptr, nullptr, dkv0, g, st, dv); });
  if (err) return err;
  return timed(6, [&] { launch_chunk<MODE_DK>(mv, mg, mq, mdk, lam, nullptr, nullptr, nullptr, g, st, dk); });
}

}  // namespace tc
}  // namespace la2
