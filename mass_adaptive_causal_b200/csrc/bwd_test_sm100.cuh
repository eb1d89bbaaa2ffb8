// bwd_test_sm100.cuh -- the backward's offline skip test for every legal tile
// (bf16, d = 128, 128 x 128 tiles), tcgen05 + TMEM + TMA.
//
// Rule (MassAlloc Attention; agihunt.info summary, backward paragraph;
// jaehun.me review, "Backward: offline sparse probabilities"): with the
// forward's final log-normalizer LSE, tile (query block i, key block j) is
// skipped iff every valid query row r has
//     max_c S_rc - LSE_r < ln tau - ln(r + 1).
// The thresholds are fixed (no state carries from tile to tile), so the test
// of all tiles is one pass of QK^T plus a row max; its result, one bit per
// tile, tells the backward's work pass which tiles need post-score work. The
// bits live in the backward's workspace (or the caller's trace buffer) for the
// duration of the call; nothing is kept from the forward pass.
//
// Structure as the forward kernel: a CTA takes query blocks A = 2c and
// B = 2c + 1, streams K_{2c+1}, K_{2c}, ..., K_0 through a 3-stage TMA ring
// and ping-pongs S_A / S_B in TMEM: warps 0-3 test A, warps 4-7 test B,
// warp 8 loads, warp 9 issues the MMAs. Thread r owns query row r of its
// block; a tile is kept if any row reaches its threshold (warpgroup OR-vote).
#pragma once

#include "fwd_sm100.cuh"

namespace mala {
namespace bwdtest {

using namespace sm100;
using fwd100::D;
using fwd100::HALF_BYTES;
using fwd100::IDESC_QK;
using fwd100::NSTAGE;
using fwd100::T;
using fwd100::TILE_BYTES;
using fwd100::wg_sync;
using fwd100::wg_vote_or;

constexpr int NT = 320;
constexpr int WARP_PRODUCER = 8;
constexpr int WARP_MMA = 9;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = 2 * TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_K + NSTAGE * TILE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 256;

struct Params {
  const float* LSE;
  int L;
  int nb;
  int npairs;
  float scale_log2;
  float log2_tau;
  uint32_t* bits;  // [Z][nb][nw]: bit j of row i set iff tile (i, j) is kept
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSTAGE];
  uint64_t k_empty[NSTAGE];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint32_t tmem_slot;
  int abort;
};

__global__ void __launch_bounds__(NT, 1)
    test_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(base + OFF_BAR);
  volatile int* abort = &bars.abort;
  const uint32_t sbase = smem_u32(base);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int c = p.npairs - 1 - (int)blockIdx.x;
  const int z = blockIdx.y;
  const int iA = 2 * c, iB = 2 * c + 1;
  const bool hasB = iB < p.nb;
  const int jtop = hasB ? iB : iA;
  const int ntiles = jtop + 1;
#define MALA_PART(X, t) ((X) == 0 ? (jtop - (t) <= iA) : hasB)

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_u32(&bars.s_full[x]), 1);
      mbar_init(smem_u32(&bars.s_free[x]), 1);
    }
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(&bars.tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_slot;

  if (warp == WARP_PRODUCER) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      const uint32_t qb = smem_u32(&bars.q_full);
      mbar_expect_tx(qb, (hasB ? 2 : 1) * TILE_BYTES);
      tma_load_3d(sbase + OFF_Q, &tmQ, 0, iA * T, z, qb);
      tma_load_3d(sbase + OFF_Q + HALF_BYTES, &tmQ, 64, iA * T, z, qb);
      if (hasB) {
        tma_load_3d(sbase + OFF_Q + TILE_BYTES, &tmQ, 0, iB * T, z, qb);
        tma_load_3d(sbase + OFF_Q + TILE_BYTES + HALF_BYTES, &tmQ, 64, iB * T, z, qb);
      }
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NSTAGE;
        if (t >= NSTAGE)
          mbar_wait(smem_u32(&bars.k_empty[s]), ((t / NSTAGE) - 1) & 1, abort, 0x211);
        const uint32_t kb = smem_u32(&bars.k_full[s]);
        const uint32_t dst = sbase + OFF_K + s * TILE_BYTES;
        mbar_expect_tx(kb, TILE_BYTES);
        tma_load_3d(dst, &tmK, 0, (jtop - t) * T, z, kb);
        tma_load_3d(dst + HALF_BYTES, &tmK, 64, (jtop - t) * T, z, kb);
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x212);
      uint32_t free_ph[2] = {0, 0};
      const uint64_t dq0 = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t dq1 = sdesc_sw128(sbase + OFF_Q + TILE_BYTES, 16, 1024);
      uint64_t dks[NSTAGE];
#pragma unroll
      for (int st = 0; st < NSTAGE; ++st) dks[st] = sdesc_sw128(sbase + OFF_K + st * TILE_BYTES, 16, 1024);
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NSTAGE;
        mbar_wait(smem_u32(&bars.k_full[s]), (t / NSTAGE) & 1, abort, 0x213);
        tc_fence_after();
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          if (!MALA_PART(X, t)) continue;
          if (t > 0 && MALA_PART(X, t - 1)) {  // S_X of the previous tile consumed
            mbar_wait_spin(smem_u32(&bars.s_free[X]), free_ph[X], abort, 0x214);
            free_ph[X] ^= 1;
            tc_fence_after();
          }
          const uint64_t dq = X ? dq1 : dq0;
          const uint64_t dk = s == 0 ? dks[0] : (s == 1 ? dks[1] : dks[2]);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16(tmem + X * 128, sdesc_kstep(dq, kk, HALF_BYTES), sdesc_kstep(dk, kk, HALF_BYTES),
                     IDESC_QK, kk > 0);
          mma_commit(smem_u32(&bars.s_full[X]));
        }
        mma_commit(smem_u32(&bars.k_empty[s]));
      }
    }
    __syncwarp();
  } else {
    const int X = warp >> 2;
    const int r = tid & 127;
    const int iX = X == 0 ? iA : iB;
    if (X == 0 || hasB) {
      const int bar_id = 1 + X;
      const int row = iX * T + r;
      // threshold in log2 units on the raw score: s * scale_log2 >= c2
      float c2 = __int_as_float(0x7f800000);  // invalid rows never keep
      if (row < p.L)
        c2 = p.LSE[(size_t)z * p.L + row] * kLog2e + p.log2_tau - __log2f((float)(row + 1));
      const float craw = c2 / p.scale_log2;
      const uint32_t t_s = tmem + ((uint32_t)((warp & 3) * 32) << 16) + X * 128;
      uint32_t s_ph = 0;
      const int nw = (p.nb + 31) >> 5;
      KeepBits kb;
      kb.init(r == 0 ? p.bits : nullptr, ((size_t)z * p.nb + iX) * nw);
      if (r == 0)
        for (int w = iX / 32 + 1; w < nw; ++w) p.bits[((size_t)z * p.nb + iX) * nw + w] = 0u;
      for (int t = 0; t < ntiles; ++t) {
        if (!MALA_PART(X, t)) continue;
        const int j = jtop - t;
        const bool diag = (j == iX);
        mbar_wait(smem_u32(&bars.s_full[X]), s_ph, abort, 0x215);
        s_ph ^= 1;
        tc_fence_after();
        const float mraw = tmem_rowmax128(t_s, diag, r);
        tc_fence_before();
        const int keep = wg_vote_or(mraw >= craw, bar_id);
        kb.set(j, keep != 0);
        if (r == 0) mbar_arrive(smem_u32(&bars.s_free[X]));
      }
      kb.flush();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
#undef MALA_PART
}

}  // namespace bwdtest
}  // namespace mala
