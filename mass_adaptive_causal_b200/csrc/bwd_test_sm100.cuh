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
// CTA = query blocks A = 2c and B = 2c + 1 sharing each streamed K tile
// (K_{2c+1}, K_{2c}, ..., K_0 through a 3-stage TMA ring: the shared tile
// halves L2 traffic per tensor-core FLOP). TMEM holds two S buffers per block
// (all 512 columns), so the MMA issuer keeps the next tile of each block
// queued while the current one is tested. A test thread owns one query row;
// it copies its S row out of TMEM, releases the buffer at once (mbarrier,
// 128 arrivals) and only then reduces and votes.
// Warps 0-3 test A, warps 4-7 test B, warp 8 loads, warp 9 issues the MMAs.
#pragma once

#include "sm100.cuh"

namespace mala {
namespace bwdtest {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr uint32_t TILE_BYTES = T * D * 2;   // 32 KB
constexpr uint32_t HALF_BYTES = T * 64 * 2;  // one 64-column swizzled block
constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, false, false);

// OR-vote over one 128-thread warpgroup on named barrier `id`.
__device__ __forceinline__ int wg_vote_or(int pred, int id) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.cta.red.or.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(out)
      : "r"(pred), "r"(id)
      : "memory");
  return (int)out;
}

constexpr int NT = 320;
constexpr int WARP_PRODUCER = 8;
constexpr int WARP_MMA = 9;
constexpr int NSK = 3;  // K stages
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = 2 * TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_K + NSK * TILE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;

struct Params {
  const float* LSE;
  int L;
  int nb;
  int npairs;
  float scale_log2;
  float log2_tau;
  uint32_t* bits;  // [Z][nb][nw]: bit j of row i set iff tile (i, j) is kept
  int Hq, G;       // query heads; G query heads share each key/value head
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSK];
  uint64_t k_empty[NSK];
  uint64_t s_full[2][2];  // [block][buffer]
  uint64_t s_free[2][2];  // 128 arrivals: every test thread of the block
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

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
  // block X takes part in tile t iff its query block >= key block; A starts
  // one tile later than B when B exists.
  const int startA = hasB ? 1 : 0;

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 1);
    }
    for (int x = 0; x < 2; ++x)
      for (int u = 0; u < 2; ++u) {
        mbar_init(smem_u32(&bars.s_full[x][u]), 1);
        mbar_init(smem_u32(&bars.s_free[x][u]), T);
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
        const int s = t % NSK;
        if (t >= NSK) mbar_wait(smem_u32(&bars.k_empty[s]), ((t / NSK) - 1) & 1, abort, 0x211);
        const uint32_t kb = smem_u32(&bars.k_full[s]);
        const uint32_t dst = sbase + OFF_K + s * TILE_BYTES;
        mbar_expect_tx(kb, TILE_BYTES);
        const int zkv = (z / p.Hq) * (p.Hq / p.G) + (z % p.Hq) / p.G;
        tma_load_3d(dst, &tmK, 0, (jtop - t) * T, zkv, kb);
        tma_load_3d(dst + HALF_BYTES, &tmK, 64, (jtop - t) * T, zkv, kb);
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      const uint64_t dq0 = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t dq1 = sdesc_sw128(sbase + OFF_Q + TILE_BYTES, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sbase + OFF_K, 16, 1024);
      mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x212);
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NSK;
        mbar_wait(smem_u32(&bars.k_full[s]), (t / NSK) & 1, abort, 0x213);
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((s * TILE_BYTES) >> 4);
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          if (X == 0 ? (t < startA) : !hasB) continue;
          const int n = X == 0 ? t - startA : t;  // this block's tile count
          const int u = n & 1;
          if (n >= 2) {  // buffer u was last filled for this block's tile n - 2
            mbar_wait_spin(smem_u32(&bars.s_free[X][u]), ((n >> 1) - 1) & 1, abort, 0x214);
            tc_fence_after();
          }
          const uint64_t dq = X ? dq1 : dq0;
          const uint32_t dst = tmem + X * 256 + u * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16(dst, sdesc_kstep(dq, kk, HALF_BYTES), sdesc_kstep(dk, kk, HALF_BYTES), IDESC_QK,
                     kk > 0);
          mma_commit(smem_u32(&bars.s_full[X][u]));
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
      const float craw =
          bwd_keep_bound_raw(p.LSE, (size_t)z * p.L, row, p.L, p.log2_tau, p.scale_log2);
      const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16) + X * 256;
      const int nw = (p.nb + 31) >> 5;
      KeepBits kb;
      kb.init(r == 0 ? p.bits : nullptr, ((size_t)z * p.nb + iX) * nw);
      if (r == 0)
        for (int w = iX / 32 + 1; w < nw; ++w) p.bits[((size_t)z * p.nb + iX) * nw + w] = 0u;
      const int nX = iX + 1;  // this block's tiles: key blocks iX, iX-1, ..., 0
      for (int n = 0; n < nX; ++n) {
        const int u = n & 1;
        const int j = iX - n;
        mbar_wait(smem_u32(&bars.s_full[X][u]), (n >> 1) & 1, abort, 0x215);
        tc_fence_after();
        float sa[64], sb[64];
        tmem_ld64(t_row + u * 128, sa);
        tmem_ld64(t_row + u * 128 + 64, sb);
        tc_fence_before();
        mbar_arrive(smem_u32(&bars.s_free[X][u]));  // S copied out: buffer free
        float mraw = kNegInf;
        if (n > 0) {
#pragma unroll
          for (int e = 0; e < 63; e += 2) mraw = fmax3f(mraw, sa[e], sa[e + 1]);
#pragma unroll
          for (int e = 0; e < 63; e += 2) mraw = fmax3f(mraw, sb[e], sb[e + 1]);
        } else {  // diagonal tile: keys after the query are masked
#pragma unroll
          for (int e = 0; e < 64; ++e) mraw = fmaxf(mraw, e > r ? kNegInf : sa[e]);
#pragma unroll
          for (int e = 0; e < 64; ++e) mraw = fmaxf(mraw, 64 + e > r ? kNegInf : sb[e]);
        }
        const int keep = wg_vote_or(mraw >= craw, bar_id);
        kb.set(j, keep != 0);
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
}

}  // namespace bwdtest
}  // namespace mala
