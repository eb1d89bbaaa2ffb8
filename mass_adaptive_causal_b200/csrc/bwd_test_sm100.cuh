// bwd_test_sm100.cuh -- the backward's offline skip test for every legal tile
// (bf16, d = 128, 128 x 128 tiles), tcgen05 on CTA pairs + TMEM + TMA.
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
// Cluster = two CTAs on two SMs and four query blocks: rank r holds blocks
// 4c + r (X = 0) and 4c + 2 + r (X = 1). Key tiles K_j, j = jtop .. 0, stream
// through a ring of half tiles: each CTA loads 64 of the 128 keys. Per key
// tile the leader issues two M = 256 MMAs (tcgen05 cta_group::2), one per X,
// each over both CTAs' block X; each CTA's TMEM receives its own rows. A
// one-SM M = 128 MMA reads both operands from shared memory at about the
// SM's whole shared-memory bandwidth; on a pair each SM reads its A and only
// half of B, and a key tile is loaded once for four query blocks.
//
// TMEM (512 columns per SM): S buffers [X][u], u = t % 2, 128 columns each.
// Test warps 0-3 own block X = 0, warps 4-7 block X = 1; a thread owns one
// query row. It copies its S row out of TMEM in one load, its warp releases
// the buffer at once (leader: a local arrival; rank 1: st.async into the
// leader's shared memory, counted on the leader's barrier) and then reduces
// (eight max chains) and votes. Warp 8 loads, warps 9 and 10 (leader) issue
// the MMAs of X = 0 and X = 1, so neither issuer's waits hold up the other's
// queued MMAs.
//
// Every wait is bounded; a wait that runs out records a timeout in the
// device status word and the thread carries on, so every thread reaches the
// final cluster barrier: the kernel always terminates.
#pragma once

#include "sm100.cuh"

namespace mala {
namespace bwdtest {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 352;
constexpr int WARP_PROD = 8;
constexpr int WARP_MMA0 = 9;  // also allocates TMEM (the same warp in both CTAs)
constexpr int NSK = 6;        // K half stages
constexpr uint32_t QB_BYTES = T * D * 2;   // 32 KB: one query block
constexpr uint32_t QH_BYTES = T * 64 * 2;  // one 64-column swizzled block of Q
constexpr uint32_t KH_BYTES = 64 * D * 2;  // 16 KB: 64 keys x 128 d
constexpr uint32_t KH_BLK = 64 * 64 * 2;   // 8 KB: one 64-column block of a K half
constexpr uint32_t OFF_Q = 0;              // [X] query blocks
constexpr uint32_t OFF_K = 2 * QB_BYTES;
constexpr uint32_t OFF_BAR = OFF_K + NSK * KH_BYTES;
constexpr uint32_t BAR_BYTES = 512;
constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_QK = idesc_bf16(256, 128, false, false);
constexpr uint32_t REL_LOCAL = 4;            // releasing warps per CTA and block
constexpr uint32_t REL_TX = 4 * REL_LOCAL;   // bytes of rank 1's releases per tile
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct Params {
  const float* LSE;
  int L;
  int nb;
  int nclus;  // clusters per (b, head): ceil(nb / 4)
  float scale_log2;
  float log2_tau;
  uint32_t* bits;  // [Z][nb][nw]: bit j of row i set iff tile (i, j) is kept
  int Hq, G;       // query heads; G query heads share each key/value head
};

struct Bars {
  uint64_t q_full;          // leader: both CTAs' query blocks
  uint64_t k_full[NSK];     // leader: both halves of a key tile
  uint64_t k_empty[NSK];    // each CTA: two arrivals, the MMAs of X = 0 and 1
  uint64_t s_full[2][2];    // each CTA: [X][u] S of the tile is in TMEM
  // leader: [X][u] S read by both CTAs -- REL_LOCAL arrivals of its own test
  // warps and one of the issuer, which arms 4 bytes per store of rank 1
  uint64_t s_free[2][2];
  int sink;                 // leader: target of rank 1's release stores
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(Bars) <= BAR_BYTES, "barrier block");

// OR-vote over one 128-thread warpgroup on named barrier 1 + X.
__device__ __forceinline__ int wg_vote_or(int pred, int X) {
  uint32_t out;
  if (X == 0)
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "barrier.cta.red.or.pred po, 1, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}\n"
        : "=r"(out)
        : "r"(pred)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "barrier.cta.red.or.pred po, 2, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}\n"
        : "=r"(out)
        : "r"(pred)
        : "memory");
  return (int)out;
}

__global__ void __launch_bounds__(NT, 1)
    test_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = smem_raw;
  // 128-byte swizzled operands need 1024-byte aligned stages; both CTAs of a
  // cluster have the same offset, so both leave here together if it is not
  if (smem_u32(base) & 1023u) {
    if (threadIdx.x == 0) record_layout_error(0x2f1);
    return;
  }
  Bars& bars = *reinterpret_cast<Bars*>(base + OFF_BAR);
  volatile int* abort = &bars.abort;
  const uint32_t sbase = smem_u32(base);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  const int z = blockIdx.y;
  const int c = p.nclus - 1 - (int)(blockIdx.x >> 1);  // longest clusters first
  const int jtop = min(4 * c + 3, p.nb - 1);
  const int ntiles = jtop + 1;  // tile t <-> key block jtop - t
  const int zkv = (z / p.Hq) * (p.Hq / p.G) + (z % p.Hq) / p.G;

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 2);
    }
    for (int x = 0; x < 2; ++x)
      for (int u = 0; u < 2; ++u) {
        mbar_init(smem_u32(&bars.s_full[x][u]), 1);
        mbar_init(smem_u32(&bars.s_free[x][u]), REL_LOCAL + 1);
      }
    bars.abort = 0;
    fence_mbar_init_cluster();
  }
  if (warp == WARP_MMA0) {
    tmem_alloc_pair(smem_u32(&bars.tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_slot;
  auto lead = [&](const void* x) { return mapa_rank(smem_u32(x), 0); };

  if (warp == WARP_PROD) {
    // ----------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      if (leader) mbar_expect_tx(smem_u32(&bars.q_full), 4 * QB_BYTES);
      for (int X = 0; X < 2; ++X) {
        // a block past the sequence reads zeros (out-of-range rows)
        const int iX = 4 * c + 2 * X + (int)rank;
        const uint32_t dst = sbase + OFF_Q + X * QB_BYTES;
        tma_load_3d_pair(dst, &tmQ, 0, iX * T, z, lead(&bars.q_full));
        tma_load_3d_pair(dst + QH_BYTES, &tmQ, 64, iX * T, z, lead(&bars.q_full));
      }
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NSK;
        if (t >= NSK && !mbar_wait(smem_u32(&bars.k_empty[s]), ((t / NSK) - 1) & 1, abort, 0x211))
          break;
        if (leader) mbar_expect_tx(smem_u32(&bars.k_full[s]), 2 * KH_BYTES);
        const int row = (jtop - t) * T + 64 * (int)rank;
        const uint32_t dst = sbase + OFF_K + s * KH_BYTES;
        tma_load_3d_pair(dst, &tmK, 0, row, zkv, lead(&bars.k_full[s]));
        tma_load_3d_pair(dst + KH_BLK, &tmK, 64, row, zkv, lead(&bars.k_full[s]));
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA0 || warp == WARP_MMA0 + 1) {
    // ------------------------------------- MMA issuers (leader only), one per X
    if (leader && lane == 0) {
      const int X = warp - WARP_MMA0;
      const uint64_t dq = sdesc_sw128(sbase + OFF_Q + X * QB_BYTES, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sbase + OFF_K, 16, 1024);
      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x212);
      tc_fence_after();
      for (int t = 0; ok && t < ntiles; ++t) {
        const int s = t % NSK, u = t & 1;
        ok = mbar_wait(smem_u32(&bars.k_full[s]), (t / NSK) & 1, abort, 0x213);
        if (!ok) break;
        if (t >= 2) {  // S buffer u of this X was last filled for tile t - 2
          const uint32_t fb = smem_u32(&bars.s_free[X][u]);
          mbar_expect_tx(fb, REL_TX);
          ok = mbar_wait_spin(fb, ((t - 2) >> 1) & 1, abort, 0x214);
          if (!ok) break;
        }
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((s * KH_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_pair(tmem + X * 256 + u * 128, sdesc_kstep(dq, kk, QH_BYTES),
                   sdesc_kstep(dk, kk, KH_BLK), IDESC_QK, kk > 0, 0u, 0u);
        commit_pair(smem_u32(&bars.s_full[X][u]), 3);
        commit_pair(smem_u32(&bars.k_empty[s]), 3);
      }
      // the last two tiles' releases have no later MMA to wait for them: wait
      // here, so that no store of rank 1 is on its way when the kernel ends
      for (int t = max(0, ntiles - 2); ok && t < ntiles; ++t) {
        const uint32_t fb = smem_u32(&bars.s_free[X][t & 1]);
        mbar_expect_tx(fb, REL_TX);
        ok = mbar_wait(fb, (t >> 1) & 1, abort, 0x216);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------ test (8 warps)
    const int X = warp >> 2;
    const int r = tid & (T - 1);
    const int iX = 4 * c + 2 * X + (int)rank;
    const bool mine = iX < p.nb;
    const int row = iX * T + r;
    const float craw = mine ? bwd_keep_bound_raw(p.LSE, (size_t)z * p.L, row, p.L, p.log2_tau,
                                                 p.scale_log2)
                            : __int_as_float(0x7f800000);
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16) + X * 256;
    const int nw = (p.nb + 31) >> 5;
    KeepBits kb;
    kb.init(r == 0 && mine ? p.bits : nullptr, ((size_t)z * p.nb + iX) * nw);
    if (r == 0 && mine)
      for (int w = iX / 32 + 1; w < nw; ++w) p.bits[((size_t)z * p.nb + iX) * nw + w] = 0u;
    auto release = [&](int t) {  // lane 0 of each warp: this warp has read tile t's S
      const uint32_t b = smem_u32(&bars.s_free[X][t & 1]);
      if (leader)
        mbar_arrive_relaxed(b);
      else
        st_async_u32(lead(&bars.sink), 0u, mapa_rank(b, 0));
    };
    for (int t = 0; t < ntiles; ++t) {
      const int j = jtop - t;
      // wait even when the tile is not legal for this block: this CTA's
      // release of the buffer must not run ahead of the buffer's previous use
      mbar_wait(smem_u32(&bars.s_full[X][t & 1]), (t >> 1) & 1, abort, 0x215);
      tc_fence_after();
      if (!mine || j > iX) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release(t);
        continue;
      }
      uint32_t v[128];
      tmem_ld128(t_row + (t & 1) * 128, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) release(t);
      // the diagonal tile masks the keys after the query
      const float mraw = row_max128(v, j == iX ? r : T - 1, 0);
      const int keep = wg_vote_or(mraw >= craw, X);
      kb.set(j, keep != 0);
    }
    kb.flush();
  }
  // a CTA that gave up on a wait may still have copies or MMAs in flight:
  // give them time to land before its shared memory and TMEM go
  if (*abort) drain_in_flight();
  // both CTAs finish every access to the other's shared memory and TMEM
  // before either frees TMEM or exits
  tc_fence_before();
  cluster_sync_all();
  if (warp == WARP_MMA0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace bwdtest
}  // namespace mala
