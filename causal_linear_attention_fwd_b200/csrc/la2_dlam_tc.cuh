// la2_dlam_tc.cuh -- the gradient with respect to the decay on the tensor
// cores (tcgen05 + TMEM + TMA), bf16 inputs, d = e = 128.
//
// The same block recurrence as the fp32-FMA kernel (la2_simt.cuh,
// dlambda_kernel), with blocks of C = 128 rows and every product a tcgen05
// MMA.  With the carried pair at the start of a block of rows p.. (local
// rows t, j):
//   KV = sum_{j<p} lambda^(p-1-j) k_j^T v_j,
//   W  = sum_{j<p} (p-1-j) lambda^(p-1-j) k_j^T v_j,
// the block adds to d lambda
//   sum_{j<t} (t-j) lambda^(t-j-1) S[t][j] G[t][j]      S = Q K^T, G = dO V^T
//   + sum_t lambda^t ((t+1) Y1[t] + Y2[t]) . dO_t      Y1 = Q KV, Y2 = Q W
// and then updates W <- lambda^cb (cb KV + W) + Kw^T V and
// KV <- lambda^cb KV + Kb^T V, with Kb = diag(lambda^(cb-1-j)) K and
// Kw = diag(cb-1-j) Kb.  No division by lambda, so lambda = 0 is exact.
//
// Precision.  S and G are products of the bf16 inputs (exact in fp32).  The
// other products take operands that are not bf16 inputs -- the carried
// KV and W, and the decayed rows Kb and Kw -- and a single bf16 rounding of
// those (relative 2^-9) shows at ~3e-3 in d lambda, whose terms cancel.  So
// each such operand is split into a bf16 pair x = hi + lo (hi = bf16(x),
// lo = bf16(x - hi), relative error ~2^-17) and every such product is two
// MMAs accumulating into the same TMEM.
//
// Work split.  Each chunk of one (b,h) is served by two CTAs, one per half
// of the e columns (64 each): every term above is a sum over e (G, Y1 . dO,
// Y2 . dO) or is computed column-wise (the KV and W updates), so the half
// CTAs need no exchange and each adds its partial sum to d lambda.  Each
// loads Q and K whole and its halves of V and dO; S = Q K^T is computed by
// both.  Per CTA: Q, K (-> Kb hi -> Kw hi in place), a lo tile for Kb / Kw,
// the V and dO halves, and hi/lo bf16 copies of its KV and W halves: 192 KB
// of shared memory.
//
// Per block (phase-serial; 256 threads, thread (row, half) owns TMEM lane
// `row`; of a 128-column region the columns half*64 .. +63, of a 64-column
// one half*32 .. +31):
//   A  [MMA]  S = Q K^T -> TMEM[0,128), G = dO_h V_h^T -> TMEM[128,256)
//   B  [CUDA] the block's own pairs from S and G; TMEM state decay
//             (W <- lambda^cb (W + cb KV), KV <- lambda^cb KV); K -> Kb pair
//   C  [MMA]  Y1 = Q KV -> TMEM[0,64), Y2 = Q W -> TMEM[64,128) (the
//             entering state's pairs), KV += Kb^T V_h
//   D  [CUDA] Kb -> Kw pair; the earlier rows' term from Y1, Y2 and dO_h
//   E  [MMA]  W += Kw^T V_h; the next block's Q and dO_h are loaded
//   F  [CUDA] hi/lo copies of the new KV and W halves; the next K and V_h
// TMEM: S / Y [0,128), G [128,256), KV half [256,320), W half [320,384).
// STATE = true: the chunk-state pre-pass (from zero; K and V only) over the
// g.nst sub-chunks of Ls rows before the last chunk: writes sub-chunk u's
// (dKV, dW) to workspace slot u+1, like the fp32-FMA pre-pass.
#pragma once

#include <cuda.h>

#include "la2_common.cuh"
#include "la2_simt.cuh"
#include "la2_sm100.cuh"
#include "la2_tc.cuh"

namespace la2 {
namespace tcd {

using namespace la2::sm100;
using la2::tc::BOX;
using la2::tc::TILE;

constexpr int BLOCK = 128;
constexpr int NT = 256;
constexpr int EH = 64;  // e columns per CTA

constexpr uint32_t OFF_Q = 0, OFF_K = TILE, OFF_KL = 2 * TILE, OFF_V = 3 * TILE;
constexpr uint32_t OFF_G = OFF_V + BOX, OFF_KVH = OFF_G + BOX, OFF_KVL = OFF_KVH + BOX;
constexpr uint32_t OFF_WH = OFF_KVL + BOX, OFF_WL = OFF_WH + BOX, OFF_MISC = OFF_WL + BOX;
// barriers (qg, kv, mma, done), TMEM slot, abort flag | lambda^n | n lambda^(n-1) | partial sums
constexpr uint32_t OFF_PW = OFF_MISC + 48, OFF_WT = OFF_PW + 4 * 132, OFF_RED = OFF_WT + 4 * 132;
constexpr uint32_t SMEM = OFF_RED + 8 * (NT / 32) + 1024;  // + alignment slack
constexpr uint32_t COL_S = 0, COL_G = 128, COL_KV = 256, COL_W = 320;

__device__ __forceinline__ uint32_t smem_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// 32 fp32 values as bf16 pairs (hi, lo) into row `row`, logical chunks
// [chunk0, chunk0 + 4) of two 128-byte-swizzled [rows][64] boxes.
__device__ __forceinline__ void st_row_pair(uint8_t *bh, uint8_t *bl, int row, int chunk0,
                                            const float *v) {
#pragma unroll
  for (int q = 0; q < 4; q++) {
    uint32_t wh[4], wl[4];
#pragma unroll
    for (int m = 0; m < 4; m++) {
      const float x0 = v[8 * q + 2 * m], x1 = v[8 * q + 2 * m + 1];
      const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
      const float2 hf = __bfloat1622float2(h);
      const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
      wh[m] = *reinterpret_cast<const uint32_t *>(&h);
      wl[m] = *reinterpret_cast<const uint32_t *>(&l);
    }
    const uint32_t off = smem_off(row, chunk0 + q);
    *reinterpret_cast<uint4 *>(bh + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4 *>(bl + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  }
}

// Row `row` (64 values) of box bh (with, when `pair`, box bl added: the
// value is bh + bl) times f, written back as a bf16 pair into (bh, bl).
__device__ __forceinline__ void scale_row_pair(uint8_t *bh, uint8_t *bl, int row, float f,
                                               bool pair) {
  uint4 h[8], l[8];
#pragma unroll
  for (int c = 0; c < 8; c++) {
    h[c] = *reinterpret_cast<const uint4 *>(bh + smem_off(row, c));
    l[c] = pair ? *reinterpret_cast<const uint4 *>(bl + smem_off(row, c)) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int c = 0; c < 8; c++) {
    float x[8];
    const __nv_bfloat162 *hh = reinterpret_cast<const __nv_bfloat162 *>(&h[c]);
    const __nv_bfloat162 *ll = reinterpret_cast<const __nv_bfloat162 *>(&l[c]);
#pragma unroll
    for (int m = 0; m < 4; m++) {
      const float2 a = __bfloat1622float2(hh[m]), b = __bfloat1622float2(ll[m]);
      x[2 * m] = (a.x + b.x) * f;
      x[2 * m + 1] = (a.y + b.y) * f;
    }
    uint32_t wh[4], wl[4];
#pragma unroll
    for (int m = 0; m < 4; m++) {
      const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * m], x[2 * m + 1]);
      const float2 hf = __bfloat1622float2(hv);
      const __nv_bfloat162 lv = __floats2bfloat162_rn(x[2 * m] - hf.x, x[2 * m + 1] - hf.y);
      wh[m] = *reinterpret_cast<const uint32_t *>(&hv);
      wl[m] = *reinterpret_cast<const uint32_t *>(&lv);
    }
    *reinterpret_cast<uint4 *>(bh + smem_off(row, c)) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4 *>(bl + smem_off(row, c)) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  }
}

template <bool STATE>
__global__ void __launch_bounds__(NT, 1)
dlam_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tg,
            const float *__restrict__ lambda, const float *__restrict__ kv0,
            float *__restrict__ ws, float *__restrict__ dlam, Geo g) {
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
  constexpr uint32_t IDESC_Y = idesc_bf16(128, EH, false, true);
  constexpr uint32_t IDESC_D = idesc_bf16(128, EH, true, true);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_MISC);
  const uint32_t b_qg = smem_u32(bars), b_kv = b_qg + 8, b_mma = b_qg + 16, b_done = b_qg + 24;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *pw = reinterpret_cast<float *>(smem + OFF_PW);  // lambda^n, n = 0..128
  float *wt = reinterpret_cast<float *>(smem + OFF_WT);  // n lambda^(n-1), n = 0..128
  double *red = reinterpret_cast<double *>(smem + OFF_RED);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int row = quarter * 32 + lane;
  const int eh = blockIdx.x & 1;  // this CTA's half of the e columns
  const int64_t unit = blockIdx.x >> 1;
  const int nch = STATE ? g.nst : g.S;
  const int64_t len = STATE ? g.Ls : g.Lc;
  const int64_t bh = unit / nch;
  const int c = (int)(unit % nch);
  const int h = (int)(bh % g.H);
  const int64_t a = (int64_t)c * len;
  const int64_t b = g.L < a + len ? g.L : a + len;
  const int nblk = (int)((b - a + BLOCK - 1) / BLOCK);
  const int ecol = eh * EH + half * 32;  // this thread's first column of the state

  if (tid <= BLOCK) {
    const double lam = (double)lambda[h];
    pw[tid] = (float)pow_int(lam, tid);
    wt[tid] = tid == 0 ? 0.f : (float)((double)tid * pow_int(lam, tid - 1));
  }
  if (tid == 0) {
    mbar_init(b_qg, 1);
    mbar_init(b_kv, 1);
    mbar_init(b_mma, 1);
    mbar_init(b_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (!STATE) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tg);
    }
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);  // this warp's lane quarter

  // loads of block j (thread 0): Q and dO_h on b_qg, K and V_h on b_kv
  int n_qg = 0, n_kv = 0;
  auto load_qg = [&](int j) {
    const int y = (int)(a + (int64_t)j * BLOCK), z = (int)bh;
    mbar_expect_tx(b_qg, TILE + BOX);
    tma_load_3d(sbase + OFF_Q, &tq, b_qg, 0, y, z);
    tma_load_3d(sbase + OFF_Q + BOX, &tq, b_qg, 64, y, z);
    tma_load_3d(sbase + OFF_G, &tg, b_qg, eh * EH, y, z);
    n_qg++;
  };
  auto load_kv = [&](int j) {
    const int y = (int)(a + (int64_t)j * BLOCK), z = (int)bh;
    mbar_expect_tx(b_kv, TILE + BOX);
    tma_load_3d(sbase + OFF_K, &tk, b_kv, 0, y, z);
    tma_load_3d(sbase + OFF_K + BOX, &tk, b_kv, 64, y, z);
    tma_load_3d(sbase + OFF_V, &tv, b_kv, eh * EH, y, z);
    n_kv++;
  };
  if (tid == 0 && nblk > 0) {
    if (!STATE) load_qg(0);
    load_kv(0);
  }

  // the entering pair (this CTA's columns) -> TMEM (fp32) and, gradient
  // pass, its bf16 pair copies
  {
    const float *ikv = nullptr, *iw = nullptr;
    if (!STATE) {
      if (g.S > 1) {
        ikv = ws + ((bh * g.wsS + (int64_t)c * g.M) * 2) * (int64_t)(128 * 128);
        iw = ikv + 128 * 128;
      } else if (kv0) {
        ikv = kv0 + bh * (int64_t)(128 * 128);
      }
    }
    float f[32], w[32];
#pragma unroll
    for (int j = 0; j < 32; j++) {
      f[j] = ikv ? ikv[(int64_t)row * 128 + ecol + j] : 0.f;
      w[j] = iw ? iw[(int64_t)row * 128 + ecol + j] : 0.f;
    }
    uint32_t r[32];
#pragma unroll
    for (int j = 0; j < 32; j++) r[j] = __float_as_uint(f[j]);
    tmem_st32(tl + COL_KV + half * 32, r);
#pragma unroll
    for (int j = 0; j < 32; j++) r[j] = __float_as_uint(w[j]);
    tmem_st32(tl + COL_W + half * 32, r);
    if (!STATE) {
      st_row_pair(smem + OFF_KVH, smem + OFF_KVL, row, half * 4, f);
      st_row_pair(smem + OFF_WH, smem + OFF_WL, row, half * 4, w);
    }
    tmem_wait_st();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  auto mma_wait = [&](uint32_t &ph) {
    const bool ok = mbar_wait(b_mma, ph, abort_flag);
    ph ^= 1u;
    return ok;
  };
  auto sync_all = [&] {
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };
  const uint32_t sQ = sbase + OFF_Q, sK = sbase + OFF_K, sKL = sbase + OFF_KL;
  const uint32_t sV = sbase + OFF_V, sG = sbase + OFF_G;
  // a state update: acc += A^T V_h with A the pair (K tile, lo tile), both
  // MN-major (M = d over the two boxes, K = rows), V_h MN-major (N = 64)
  auto issue_update = [&](uint32_t col) {
#pragma unroll
    for (int k = 0; k < 8; k++)
      mma_ss(tmem + col, sdesc_sw128(sK + k * 2048, BOX, 1024), sdesc_sw128(sV + k * 2048, BOX, 1024),
             IDESC_D, 1);
#pragma unroll
    for (int k = 0; k < 8; k++)
      mma_ss(tmem + col, sdesc_sw128(sKL + k * 2048, BOX, 1024), sdesc_sw128(sV + k * 2048, BOX, 1024),
             IDESC_D, 1);
  };
  // Y = Q X with X a state pair (hi, lo boxes: rows d, this CTA's 64 columns)
  auto issue_y = [&](uint32_t col, uint32_t sXh, uint32_t sXl) {
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const uint32_t koff = (k >> 2) * BOX + (k & 3) * 32;
      mma_ss(tmem + col, sdesc_sw128(sQ + koff, 16, 1024), sdesc_sw128(sXh + k * 2048, BOX, 1024),
             IDESC_Y, k > 0);
    }
#pragma unroll
    for (int k = 0; k < 8; k++) {
      const uint32_t koff = (k >> 2) * BOX + (k & 3) * 32;
      mma_ss(tmem + col, sdesc_sw128(sQ + koff, 16, 1024), sdesc_sw128(sXl + k * 2048, BOX, 1024),
             IDESC_Y, 1);
    }
  };

  uint32_t mph = 0;
  double acc = 0.0;
  bool aborted = false;
  int waited = 0;  // blocks whose tiles were waited for successfully
  for (int i = 0; i < nblk; i++) {
    const int64_t p = a + (int64_t)i * BLOCK;
    const int cb = (int)(b - p < BLOCK ? b - p : BLOCK);
    const uint32_t par = (uint32_t)(i & 1);

    // ---- A: the block's tiles; S and G
    bool ok = mbar_wait(b_kv, par, abort_flag);
    if (!STATE) ok = ok && mbar_wait(b_qg, par, abort_flag);
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    waited = i + 1;
    tc_fence_after();
    float part = 0.f;
    if (!STATE) {
      if (tid == 0) {
#pragma unroll
        for (int k = 0; k < 8; k++) {
          const uint32_t koff = (k >> 2) * BOX + (k & 3) * 32;
          mma_ss(tmem + COL_S, sdesc_sw128(sQ + koff, 16, 1024), sdesc_sw128(sK + koff, 16, 1024),
                 IDESC_S, k > 0);
        }
#pragma unroll
        for (int k = 0; k < 4; k++)
          mma_ss(tmem + COL_G, sdesc_sw128(sG + k * 32, 16, 1024), sdesc_sw128(sV + k * 32, 16, 1024),
                 IDESC_S, k > 0);
        mma_commit(b_mma);
      }
      ok = mma_wait(mph);
      if (__syncthreads_or(!ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      // ---- B: the block's own pairs j < t (rows and columns past cb excluded)
#pragma unroll
      for (int pp = 0; pp < 2; pp++) {
        const int col0 = half * 64 + pp * 32;
        uint32_t rs[32], rg[32];
        tmem_ld32(tl + COL_S + col0, rs);
        tmem_ld32(tl + COL_G + col0, rg);
        tmem_wait_ld();
        if (row < cb) {
#pragma unroll
          for (int jj = 0; jj < 32; jj++) {
            const int j = col0 + jj;
            if (j < row) part += wt[row - j] * (__uint_as_float(rs[jj]) * __uint_as_float(rg[jj]));
          }
        }
      }
    }
    // TMEM state decay: W <- lambda^cb (W + cb KV), KV <- lambda^cb KV
    {
      const float dec = pw[cb], cbf = (float)cb;
      uint32_t rk[32], rw[32];
      tmem_ld32(tl + COL_KV + half * 32, rk);
      tmem_ld32(tl + COL_W + half * 32, rw);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; j++) {
        const float kvj = __uint_as_float(rk[j]);
        rw[j] = __float_as_uint(dec * fmaf(cbf, kvj, __uint_as_float(rw[j])));
        rk[j] = __float_as_uint(dec * kvj);
      }
      tmem_st32(tl + COL_KV + half * 32, rk);
      tmem_st32(tl + COL_W + half * 32, rw);
    }
    // K rows -> Kb pair (rows past the block end: 0)
    scale_row_pair(smem + OFF_K + half * BOX, smem + OFF_KL + half * BOX, row,
                   row < cb ? pw[cb - 1 - row] : 0.f, false);
    tmem_wait_st();
    sync_all();

    // ---- C: Y1 = Q KV, Y2 = Q W (entering state), KV += Kb^T V_h
    if (tid == 0) {
      if (!STATE) {
        issue_y(COL_S, sbase + OFF_KVH, sbase + OFF_KVL);
        issue_y(COL_S + EH, sbase + OFF_WH, sbase + OFF_WL);
      }
      issue_update(COL_KV);
      mma_commit(b_mma);
    }
    ok = mma_wait(mph);
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    tc_fence_after();

    // ---- D: Kb -> Kw pair; the earlier rows' term lambda^t ((t+1) Y1 + Y2) . dO_t
    scale_row_pair(smem + OFF_K + half * BOX, smem + OFF_KL + half * BOX, row,
                   row < cb ? (float)(cb - 1 - row) : 0.f, true);
    if (!STATE) {
      uint32_t r1[32], r2[32];
      tmem_ld32(tl + COL_S + half * 32, r1);
      tmem_ld32(tl + COL_S + EH + half * 32, r2);
      tmem_wait_ld();
      float s1 = 0.f, s0 = 0.f;
      const uint8_t *gbox = smem + OFF_G;
#pragma unroll
      for (int q4 = 0; q4 < 4; q4++) {
        const uint4 w = *reinterpret_cast<const uint4 *>(gbox + smem_off(row, half * 4 + q4));
        const __nv_bfloat162 *hv = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
        for (int m = 0; m < 4; m++) {
          const float2 gf = __bfloat1622float2(hv[m]);
          const int jj = q4 * 8 + 2 * m;
          s1 = fmaf(__uint_as_float(r1[jj]), gf.x, fmaf(__uint_as_float(r1[jj + 1]), gf.y, s1));
          s0 = fmaf(__uint_as_float(r2[jj]), gf.x, fmaf(__uint_as_float(r2[jj + 1]), gf.y, s0));
        }
      }
      if (row < cb) part += pw[row] * fmaf((float)(row + 1), s1, s0);
      acc += (double)part;
    }
    sync_all();

    // ---- E: W += Kw^T V_h; the next block's Q and dO_h (this block's are consumed)
    if (tid == 0) {
      issue_update(COL_W);
      mma_commit(b_mma);
      if (!STATE && i + 1 < nblk) load_qg(i + 1);
    }
    ok = mma_wait(mph);
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    tc_fence_after();

    // ---- F: pair copies of the new KV and W halves for the next block's products
    if (!STATE && i + 1 < nblk) {
      uint32_t rk[32], rw[32];
      tmem_ld32(tl + COL_KV + half * 32, rk);
      tmem_ld32(tl + COL_W + half * 32, rw);
      tmem_wait_ld();
      st_row_pair(smem + OFF_KVH, smem + OFF_KVL, row, half * 4, reinterpret_cast<const float *>(rk));
      st_row_pair(smem + OFF_WH, smem + OFF_WL, row, half * 4, reinterpret_cast<const float *>(rw));
    }
    sync_all();
    if (tid == 0 && i + 1 < nblk) load_kv(i + 1);
  }

  if (!aborted) {
    if constexpr (STATE) {
      float *okv = ws + ((bh * g.wsS + c + 1) * 2) * (int64_t)(128 * 128), *ow = okv + 128 * 128;
      uint32_t rk[32], rw[32];
      tmem_ld32(tl + COL_KV + half * 32, rk);
      tmem_ld32(tl + COL_W + half * 32, rw);
      tmem_wait_ld();
      float4 *dk4 = reinterpret_cast<float4 *>(okv + (int64_t)row * 128 + ecol);
      float4 *dw4 = reinterpret_cast<float4 *>(ow + (int64_t)row * 128 + ecol);
#pragma unroll
      for (int j = 0; j < 8; j++) {
        dk4[j] = make_float4(__uint_as_float(rk[4 * j]), __uint_as_float(rk[4 * j + 1]),
                             __uint_as_float(rk[4 * j + 2]), __uint_as_float(rk[4 * j + 3]));
        dw4[j] = make_float4(__uint_as_float(rw[4 * j]), __uint_as_float(rw[4 * j + 1]),
                             __uint_as_float(rw[4 * j + 2]), __uint_as_float(rw[4 * j + 3]));
      }
    } else {
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) red[warp] = acc;
      __syncthreads();
      if (tid == 0) {
        double t = 0.0;
        for (int w = 0; w < NT / 32; w++) t += red[w];
        atomicAdd(dlam + h, (float)t);
      }
    }
  } else if (tid == 0) {
    // every load issued has landed and every MMA issued has finished before
    // shared memory and TMEM are released (each wait bounded)
    volatile int never = 0;
    for (int j = waited; j < n_kv; j++) mbar_wait(b_kv, (uint32_t)(j & 1), &never);
    for (int j = waited; j < n_qg; j++) mbar_wait(b_qg, (uint32_t)(j & 1), &never);
    mma_commit(b_done);
    mbar_wait(b_done, 0, &never);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Chunked: the chunk-state pre-pass over the sub-chunks before the last
// chunk, the scan of the (KV, W) pairs (the fp32 scan kernel), then the
// gradient pass over every chunk; unsplit: the gradient pass alone.  Two
// CTAs per (sub-)chunk (the e halves).  dlam is zeroed first (each CTA adds
// its sum atomically).
template <typename Timed>
cudaError_t dlambda(const void *q, const void *k, const void *v, const void *dO, const float *lam,
                    const float *kv0, float *dlam, float *ws, const Geo &g, cudaStream_t st,
                    Timed &&timed) {
  const int64_t BH = (int64_t)g.B * g.H;
  if (!la2::tc::geometry_ok(g)) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mg;
  if (!la2::tc::make_map(&mq, q, BH, g.L) || !la2::tc::make_map(&mk, k, BH, g.L) ||
      !la2::tc::make_map(&mv, v, BH, g.L) || !la2::tc::make_map(&mg, dO, BH, g.L))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(dlam_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dlam_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(dlam, 0, (size_t)g.H * sizeof(float), st);
  if (e != cudaSuccess) return e;
  if (g.S > 1) {
    e = timed(0, [&] {
      dlam_kernel<true><<<(unsigned)(2 * BH * g.nst), NT, SMEM, st>>>(mq, mk, mv, mg, lam, nullptr,
                                                                       ws, nullptr, g);
    });
    if (e != cudaSuccess) return e;
    e = timed(1, [&] {
      la2::simt::dlam_scan_kernel<128, 128>
          <<<dim3(128 * 128 / la2::simt::NT, (unsigned)BH), la2::simt::NT, 0, st>>>(ws, kv0, lam, g);
    });
    if (e != cudaSuccess) return e;
  }
  return timed(2, [&] {
    dlam_kernel<false><<<(unsigned)(2 * BH * g.S), NT, SMEM, st>>>(mq, mk, mv, mg, lam, kv0, ws,
                                                                    dlam, g);
  });
}

}  // namespace tcd
}  // namespace la2
