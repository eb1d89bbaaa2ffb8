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
// CTA = one query block i, 320 threads: warps 0-7 test (two threads per query
// row, 64 columns each), warp 8 streams K_i, K_{i-1}, ... through a 4-stage
// TMA ring, warp 9 issues QK^T into a ring of four S buffers in TMEM (all 512
// columns), running up to three tiles ahead of the test. A tile is kept if
// any row reaches its threshold (OR-vote over the 256 test threads).
#pragma once

#include "fwd_sm100.cuh"

namespace mala {
namespace bwdtest {

using namespace sm100;
using fwd100::D;
using fwd100::HALF_BYTES;
using fwd100::IDESC_QK;
using fwd100::T;
using fwd100::TILE_BYTES;

constexpr int NT = 320;
constexpr int NSOFT = 256;
constexpr int WARP_PRODUCER = 8;
constexpr int WARP_MMA = 9;
constexpr int NSB = 4;  // S buffers in TMEM
constexpr int NSK = 4;  // K stages in shared memory
constexpr int BAR_SOFT = 1;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_K + NSK * TILE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;

struct Params {
  const float* LSE;
  int L;
  int nb;
  float scale_log2;
  float log2_tau;
  uint32_t* bits;  // [Z][nb][nw]: bit j of row i set iff tile (i, j) is kept
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSK];
  uint64_t k_empty[NSK];
  uint64_t s_full[NSB];
  uint64_t s_free[NSB];
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

  const int i = p.nb - 1 - (int)blockIdx.x;
  const int z = blockIdx.y;
  const int ntiles = i + 1;

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 1);
    }
    for (int b = 0; b < NSB; ++b) {
      mbar_init(smem_u32(&bars.s_full[b]), 1);
      mbar_init(smem_u32(&bars.s_free[b]), 1);
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
      mbar_expect_tx(qb, TILE_BYTES);
      tma_load_3d(sbase + OFF_Q, &tmQ, 0, i * T, z, qb);
      tma_load_3d(sbase + OFF_Q + HALF_BYTES, &tmQ, 64, i * T, z, qb);
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NSK;
        if (t >= NSK) mbar_wait(smem_u32(&bars.k_empty[s]), ((t / NSK) - 1) & 1, abort, 0x211);
        const uint32_t kb = smem_u32(&bars.k_full[s]);
        const uint32_t dst = sbase + OFF_K + s * TILE_BYTES;
        mbar_expect_tx(kb, TILE_BYTES);
        tma_load_3d(dst, &tmK, 0, (i - t) * T, z, kb);
        tma_load_3d(dst + HALF_BYTES, &tmK, 64, (i - t) * T, z, kb);
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint64_t dq = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sbase + OFF_K, 16, 1024);
      mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x212);
      for (int t = 0; t < ntiles; ++t) {
        const int b = t % NSB;
        if (t >= NSB)  // buffer b: the test of tile t - NSB has read it
          mbar_wait_spin(smem_u32(&bars.s_free[b]), ((t / NSB) - 1) & 1, abort, 0x214);
        const int s = t % NSK;
        mbar_wait(smem_u32(&bars.k_full[s]), (t / NSK) & 1, abort, 0x213);
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((s * TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16(tmem + b * 128, sdesc_kstep(dq, kk, HALF_BYTES), sdesc_kstep(dk, kk, HALF_BYTES),
                   IDESC_QK, kk > 0);
        mma_commit(smem_u32(&bars.s_full[b]));
        mma_commit(smem_u32(&bars.k_empty[s]));
      }
    }
    __syncwarp();
  } else {
    const int h = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const int col0 = 64 * h;
    const int row = i * T + r;
    // threshold in log2 units on the raw score: s * scale_log2 >= c2
    float c2 = __int_as_float(0x7f800000);  // invalid rows never keep
    if (row < p.L)
      c2 = p.LSE[(size_t)z * p.L + row] * kLog2e + p.log2_tau - __log2f((float)(row + 1));
    const float craw = c2 / p.scale_log2;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int nw = (p.nb + 31) >> 5;
    KeepBits kb;
    kb.init(tid == 0 ? p.bits : nullptr, ((size_t)z * p.nb + i) * nw);
    if (tid == 0)
      for (int w = i / 32 + 1; w < nw; ++w) p.bits[((size_t)z * p.nb + i) * nw + w] = 0u;
    for (int t = 0; t < ntiles; ++t) {
      const int b = t % NSB;
      const int j = i - t;
      mbar_wait(smem_u32(&bars.s_full[b]), (t / NSB) & 1, abort, 0x215);
      tc_fence_after();
      const float hm = tmem_rowmax64(tmem + lane_base + b * 128 + col0, t == 0, r, col0);
      tc_fence_before();
      const int keep = bar_vote_or(hm >= craw, BAR_SOFT, NSOFT);
      kb.set(j, keep != 0);
      if (tid == 0) mbar_arrive(smem_u32(&bars.s_free[b]));
    }
    kb.flush();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace bwdtest
}  // namespace mala
