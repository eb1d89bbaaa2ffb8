// fwd_sm100.cuh -- MALA forward for bf16, d = 128, 128 x 128 tiles on the
// 5th-generation tensor cores (tcgen05 + TMEM), operands staged by TMA.
//
// Rule (MassAlloc Attention; agihunt.info summary, forward paragraph;
// jaehun.me review, "Forward: online sparse softmax"): per query block i the
// key tiles j = i, i-1, ..., 0 are visited from the diagonal back. Every
// tile's scores S = Q_i K_j^T are computed on the tensor cores; the tile is
// skipped iff every valid row r has  mt_r - m_r - ln l_r < ln tau - ln(r+1),
// i.e. exp(mt - m) / l < tau / Lq. Only kept tiles load V_j, update (m, l)
// and accumulate P V_j. The diagonal tile is always kept; the final
// log-normalizer goes to LSE. Work is in log2 units (s2 = s * scale * log2 e).
//
// CTA = two query blocks A = 2c and B = 2c + 1 of one (b, h) slice that
// share every K tile: K_{2c+1} (B's diagonal, B only), then K_{2c} ... K_0
// for both. Sharing halves the L2 -> SM traffic per tensor-core FLOP.
//
// Warp roles (352 threads):
//   warps 0-3  softmax/test warpgroup of A (thread r owns query row r = TMEM lane r)
//   warps 4-7  softmax/test warpgroup of B
//   warp  8    TMA producer: Q_A, Q_B, then the K ring (3 stages)
//   warp  9    MMA issuer of A (one thread): QK^T and PV of block A
//   warp  10   MMA issuer of B
// The two blocks ping-pong on the tensor pipe: one block's scores are
// computed while the other block's warpgroup runs its test. An issuing
// thread's own shared-memory reads (its mbarrier polls) wait for the MMAs it
// has queued, so each block gets its own issuer: while A's issuer waits for
// A's decision, B's MMAs stay queued and the pipe does not drain.
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// A kept tile's P = exp2(s2 - m) is written back over its own S columns as
// bf16 pairs: each 32-column chunk holds 16 columns of P_hi and 16 of P_lo
// (P = P_hi + P_lo to ~16 bits), and PV = P_hi V + P_lo V reads P from TMEM.
// O accumulates in TMEM; it is rescaled only when the running max grows by
// more than 2^8 (the ratio test is exact for any reference max, since
// exp(mt - m)/l is unchanged by a common shift of m and l).
// V_j is loaded (by the warpgroup's first thread) only after the warpgroup's
// vote says "keep"; skipped tiles cost one QK^T and a row max.
//
// Every mbarrier wait is bounded; a wait that runs out records a timeout in
// the device status word and the thread carries on, so that no warp is left
// behind at a named barrier: the kernel always terminates.
#pragma once

#include "sm100.cuh"

namespace mala {
namespace fwd100 {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 352;  // 11 warps: 3 share a sub-partition, so at most 168 registers
constexpr int WARP_PRODUCER = 8;
constexpr int WARP_MMA_A = 9;   // issues block A's MMAs; allocates TMEM
constexpr int WARP_MMA_B = 10;  // issues block B's MMAs
constexpr int NSTAGE = 3;
constexpr uint32_t TILE_BYTES = T * D * 2;   // 32 KB
constexpr uint32_t HALF_BYTES = T * 64 * 2;  // one 64-column swizzled block
constexpr uint32_t OFF_Q = 0;                            // Q_A, Q_B
constexpr uint32_t OFF_K = 2 * TILE_BYTES;               // K ring
constexpr uint32_t OFF_V = OFF_K + NSTAGE * TILE_BYTES;  // V_A, V_B
constexpr uint32_t OFF_BAR = OFF_V + 2 * TILE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, false, true);
constexpr float kRescaleLog2 = 8.f;  // lazy O rescale threshold (log2 units)

struct Params {
  __nv_bfloat16* O;
  float* O32;  // optional float32 copy of O (nullptr: not written)
  float* LSE;
  int L;
  int nb;      // query / key blocks
  int npairs;  // ceil(nb / 2)
  float scale_log2;
  float log2_tau;
  int never_skip;
  int32_t* kept_tiles;
  uint32_t* keep_bits;
  // optional, for the backward's test: raw score maxima of every row,
  // [Z][i(i+1)/2 + j][T] (query block i, key block j <= i), written only for
  // the tiles whose maxima can decide that test (see kNearSkip) and flagged
  // in rm_bits [Z][nb][ceil(nb/32)] (bit j of row i: tile (i, j) stored)
  float* rowmax;
  uint32_t* rm_bits;
};

// The backward keeps tile (i, j) iff some row's maximum reaches the bound set
// by the final log-normalizer, which is never below the partial one the
// forward tests against (the normalizer only grows as tiles are added). A
// tile the forward skips with every row's maximum below its bound by more
// than this relative margin therefore fails the backward's test too, whatever
// the rounding of either bound; its maxima are not stored. Kept tiles and
// tiles skipped by less are stored.
constexpr float kNearSkip = 1e-3f;

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSTAGE];
  uint64_t k_empty[NSTAGE];
  uint64_t s_full[2];
  uint64_t decision[2];
  uint64_t v_full[2];
  uint64_t pv_done[2];
  int keepflag[2];
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");
static_assert(NSTAGE == 3, "descriptor selection below assumes three K stages");

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
__device__ __forceinline__ void wg_sync(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

// S_X = Q_X K_t^T (8 MMAs of K = 16), completion signalled on s_full[X].
// dq / dk: base descriptors of Q_X and of the K stage holding tile t.
__device__ __forceinline__ void issue_qk(Bars& bars, uint32_t tmem, int X, uint64_t dq,
                                         uint64_t dk) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_bf16(tmem + X * 128, sdesc_kstep(dq, kk, HALF_BYTES), sdesc_kstep(dk, kk, HALF_BYTES),
             IDESC_QK, kk > 0);
  mma_commit(smem_u32(&bars.s_full[X]));
}

__device__ __forceinline__ void wait_k_full(Bars& bars, int t, volatile int* abort) {
  mbar_wait(smem_u32(&bars.k_full[t % NSTAGE]), (t / NSTAGE) & 1, abort, 0x113);
  tc_fence_after();
}

__global__ void __launch_bounds__(NT, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(base + OFF_BAR);
  volatile int* abort = &bars.abort;
  const uint32_t sbase = smem_u32(base);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int c = p.npairs - 1 - (int)blockIdx.x;  // longest pairs first
  const int z = blockIdx.y;
  const int iA = 2 * c, iB = 2 * c + 1;
  const bool hasB = iB < p.nb;
  const int jtop = hasB ? iB : iA;
  const int ntiles = jtop + 1;  // tile t <-> key block jtop - t
  // block X (0 = A, 1 = B) works on tile t iff its query block >= key block
#define MALA_PART(X, t) ((X) == 0 ? (jtop - (t) <= iA) : hasB)

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 2);  // one commit per issuer
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_u32(&bars.s_full[x]), 1);
      mbar_init(smem_u32(&bars.decision[x]), 1);
      mbar_init(smem_u32(&bars.v_full[x]), 1);
      mbar_init(smem_u32(&bars.pv_done[x]), 1);
    }
    bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA_A) {
    tmem_alloc(smem_u32(&bars.tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_slot;

  if (warp == WARP_PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
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
          mbar_wait(smem_u32(&bars.k_empty[s]), ((t / NSTAGE) - 1) & 1, abort, 0x111);
        const uint32_t kb = smem_u32(&bars.k_full[s]);
        const uint32_t dst = sbase + OFF_K + s * TILE_BYTES;
        mbar_expect_tx(kb, TILE_BYTES);
        tma_load_3d(dst, &tmK, 0, (jtop - t) * T, z, kb);
        tma_load_3d(dst + HALF_BYTES, &tmK, 64, (jtop - t) * T, z, kb);
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA_A || warp == WARP_MMA_B) {
    // ----------------------------------------------- MMA issuers (one per block)
    // Each block has its own issuing thread, so that one issuer waiting for
    // its block's decision never holds back the other block's MMAs: the
    // tensor pipe keeps the other block's work queued meanwhile.
    const int X = warp - WARP_MMA_A;
    if (lane == 0) {
      mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x112);
      uint32_t dec_ph = 0, v_ph = 0;
      int pv_count = 0;
      // base descriptors, computed once
      const uint64_t dq = sdesc_sw128(sbase + OFF_Q + X * TILE_BYTES, 16, 1024);
      uint64_t dks[NSTAGE];
#pragma unroll
      for (int st = 0; st < NSTAGE; ++st) dks[st] = sdesc_sw128(sbase + OFF_K + st * TILE_BYTES, 16, 1024);
      const uint64_t dv = sdesc_sw128(sbase + OFF_V + X * TILE_BYTES, HALF_BYTES, 1024);
      auto kdesc = [&](int t) -> uint64_t {
        const int st = t % NSTAGE;
        return st == 0 ? dks[0] : (st == 1 ? dks[1] : dks[2]);
      };
      // Both issuers commit k_empty once per tile (count 2), whether or not
      // their block takes part in it.
      if (MALA_PART(X, 0)) {
        wait_k_full(bars, 0, abort);
        issue_qk(bars, tmem, X, dq, kdesc(0));
      }
      mma_commit(smem_u32(&bars.k_empty[0]));
      for (int t = 0; t < ntiles; ++t) {
        if (MALA_PART(X, t)) {
          mbar_wait_spin(smem_u32(&bars.decision[X]), dec_ph, abort, 0x114);
          dec_ph ^= 1;
          if (*reinterpret_cast<volatile int*>(&bars.keepflag[X])) {
            mbar_wait(smem_u32(&bars.v_full[X]), v_ph, abort, 0x115);
            v_ph ^= 1;
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
              for (int kk = 0; kk < T / 16; ++kk) {
                const uint32_t a_t = tmem + X * 128 + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half;
                mma_bf16_ts(tmem + 256 + X * 128, a_t, dv + (uint64_t)((kk * 2048) >> 4),
                            IDESC_PV, (pv_count > 0 || half > 0 || kk > 0) ? 1u : 0u);
              }
            }
            mma_commit(smem_u32(&bars.pv_done[X]));
            ++pv_count;
          }
        }
        if (t + 1 < ntiles) {
          if (MALA_PART(X, t + 1)) {
            wait_k_full(bars, t + 1, abort);
            issue_qk(bars, tmem, X, dq, kdesc(t + 1));
          }
          mma_commit(smem_u32(&bars.k_empty[(t + 1) % NSTAGE]));
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------- softmax / test groups
    const int X = warp >> 2;  // 0 = A, 1 = B
    const int r = tid & 127;
    const int iX = X == 0 ? iA : iB;
    if (X == 0 || hasB) {
      const int bar_id = 1 + X;
      const int row = iX * T + r;
      const bool row_valid = row < p.L;
      const float thr = p.never_skip ? 0.f : (p.log2_tau - __log2f((float)(row + 1)));
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t t_s = tmem + lane_base + X * 128;
      const uint32_t t_o = tmem + lane_base + 256 + X * 128;
      const uint32_t vdst = sbase + OFF_V + X * TILE_BYTES;
      float m_ref = kNegInf, l = 0.f;
      // keep iff mraw * scale_log2 - m_ref - log2 l >= thr; cached as a raw
      // score bound, refreshed whenever (m_ref, l) change
      float bound_raw = kNegInf;
      int n_kept = 0;
      uint32_t s_ph = 0;
      const int nw = (p.nb + 31) >> 5;
      KeepBits kb;
      kb.init(r == 0 ? p.keep_bits : nullptr, ((size_t)z * p.nb + iX) * nw);
      if (r == 0 && p.keep_bits)
        for (int w = iX / 32 + 1; w < nw; ++w) p.keep_bits[((size_t)z * p.nb + iX) * nw + w] = 0u;
      float* rm = p.rowmax ? p.rowmax + ((size_t)z * ((size_t)p.nb * (p.nb + 1) / 2) +
                                         (size_t)iX * (iX + 1) / 2) * T + r
                           : nullptr;
      KeepBits kbs;  // which tiles' maxima are stored
      kbs.init(r == 0 ? p.rm_bits : nullptr, ((size_t)z * p.nb + iX) * nw);
      if (r == 0 && p.rm_bits)
        for (int w = iX / 32 + 1; w < nw; ++w) p.rm_bits[((size_t)z * p.nb + iX) * nw + w] = 0u;

      for (int t = 0; t < ntiles; ++t) {
        if (!MALA_PART(X, t)) continue;
        const int j = jtop - t;
        const bool diag = (j == iX);
        mbar_wait(smem_u32(&bars.s_full[X]), s_ph, abort, 0x116);
        s_ph ^= 1;
        tc_fence_after();
        // ---- row max of the tile (raw scores: the positive scale commutes)
        const float mraw = tmem_rowmax128(t_s, diag, r);
        const float mt = mraw * p.scale_log2;
        int want = diag || p.never_skip;
        if (!want && row_valid) want = mraw >= bound_raw;
        tc_fence_before();
        const int keep = wg_vote_or(want, bar_id);
        kb.set(j, keep != 0);
        if (!keep) {
          if (r == 0) {
            bars.keepflag[X] = 0;
            mbar_arrive(smem_u32(&bars.decision[X]));
          }
          // after the decision (off the issuer's path): is any row close
          // enough to its bound that the backward's test could keep the tile?
          if (rm) {
            const bool near =
                row_valid && mraw >= bound_raw - kNearSkip * (1.f + fabsf(bound_raw));
            const int store = wg_vote_or(near, bar_id);
            if (store) rm[(size_t)j * T] = mraw;
            kbs.set(j, store != 0);
          }
          continue;
        }
        if (rm) {
          rm[(size_t)j * T] = mraw;
          kbs.set(j, true);
        }
        // ---- kept tile ----------------------------------------------------
        if (n_kept > 0) {  // the previous PV of this block reads V_X and O_X
          mbar_wait(smem_u32(&bars.pv_done[X]), (n_kept - 1) & 1, abort, 0x117);
          tc_fence_after();
        }
        if (r == 0) {
          const uint32_t vb = smem_u32(&bars.v_full[X]);
          mbar_expect_tx(vb, TILE_BYTES);
          tma_load_3d(vdst, &tmV, 0, j * T, z, vb);
          tma_load_3d(vdst + HALF_BYTES, &tmV, 64, j * T, z, vb);
        }
        const float m_new = fmaxf(m_ref, mt);
        const bool first = (n_kept == 0);
        const bool need = !first && (m_new > m_ref + kRescaleLog2);
        if (first) {
          m_ref = m_new;
        } else if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? exp2f(m_ref - m_new) : 1.f;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            float o[32];
            tmem_ld32(t_o + ch * 32, o);
            uint32_t w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(o[e] * alpha);
            tmem_st32(t_o + ch * 32, w);
          }
          if (need) {
            l *= alpha;
            m_ref = m_new;
          }
        }
        // ---- P = exp2(s2 - m_ref) as hi + lo bf16 pairs over the S columns
        float lsum = 0.f;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float s[32];
          tmem_ld32(t_s + ch * 32, s);
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int col = ch * 32 + e;
            const float p0 = (diag && col > r) ? 0.f : exp2f(s[e] * p.scale_log2 - m_ref);
            const float p1 = (diag && col + 1 > r) ? 0.f : exp2f(s[e + 1] * p.scale_log2 - m_ref);
            lsum += p0 + p1;
            const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
            const float2 hf = __bfloat1622float2(h);
            w[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            w[16 + (e >> 1)] = pack_bf16(p0 - hf.x, p1 - hf.y);
          }
          tmem_st32(t_s + ch * 32, w);
        }
        l += lsum;
        ++n_kept;
        bound_raw = (thr + m_ref + __log2f(l)) / p.scale_log2;
        tc_fence_before();
        wg_sync(bar_id);
        if (r == 0) {
          bars.keepflag[X] = 1;
          mbar_arrive(smem_u32(&bars.decision[X]));
        }
      }
      kb.flush();
      kbs.flush();
      // ---- epilogue: O = O_acc / l, LSE = (m + log2 l) ln 2 -------------------
      mbar_wait(smem_u32(&bars.pv_done[X]), (n_kept - 1) & 1, abort, 0x118);
      tc_fence_after();
      const float inv = 1.f / l;
      const size_t orow = ((size_t)z * p.L + (row_valid ? row : 0)) * D;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float o[32];
        tmem_ld32(t_o + ch * 32, o);
        if (row_valid) {
          uint4* d4 = reinterpret_cast<uint4*>(p.O + orow + ch * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
            w.y = pack_bf16(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
            w.z = pack_bf16(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
            w.w = pack_bf16(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
            d4[q] = w;
          }
          if (p.O32) {
            float4* d32 = reinterpret_cast<float4*>(p.O32 + orow + ch * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              d32[q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv,
                                   o[4 * q + 3] * inv);
          }
        }
      }
      if (row_valid) p.LSE[(size_t)z * p.L + row] = (m_ref + __log2f(l)) * kLn2;
      if (r == 0 && p.kept_tiles) p.kept_tiles[(size_t)z * p.nb + iX] = n_kept;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA_A) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
#undef MALA_PART
}

}  // namespace fwd100
}  // namespace mala
