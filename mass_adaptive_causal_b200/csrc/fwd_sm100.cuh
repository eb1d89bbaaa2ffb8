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
// CTA = one query block, 320 threads:
//   warps 0-7  test / softmax: two threads per query row r (TMEM lane r),
//              thread half h owns tile columns [64h, 64h + 64)
//   warp  8    TMA producer: Q_i, then K_i, K_{i-1}, ... through a 4-stage ring
//   warp  9    MMA issuer (one thread)
// TMEM (512 columns): three S buffers [0,128), [128,256), [256,384) and the
// output accumulator O [384,512). The issuer runs up to two tiles ahead of
// the test: while tile t is tested, S of tiles t+1 and t+2 are computed or
// queued, so the tensor pipe never waits for a decision. A buffer is reused
// once the decision on its previous tile is known: right after the vote if
// the tile was skipped, after its P V product has been issued if it was kept.
// A kept tile's P = exp2(s2 - m) is written back over its S columns as bf16
// pairs (each 32-column chunk: 16 columns of P_hi, 16 of P_lo; P = P_hi + P_lo
// to ~16 bits) and PV = P_hi V + P_lo V reads P from TMEM. O is rescaled only
// when the running max grows by more than 2^8; the ratio test is exact for
// any reference max since exp(mt - m) / l is invariant under a common shift.
// V_j is loaded only after the vote says "keep".
//
// Every mbarrier wait is bounded; a wait that runs out records a timeout in
// the device status word and the thread carries on, so no warp is left
// behind at a named barrier and the kernel always terminates.
#pragma once

#include "sm100.cuh"

namespace mala {
namespace fwd100 {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 320;
constexpr int NSOFT = 256;  // test / softmax threads
constexpr int WARP_PRODUCER = 8;
constexpr int WARP_MMA = 9;
constexpr int NSB = 3;  // S buffers in TMEM
constexpr int NSK = 4;  // K stages in shared memory
constexpr int BAR_SOFT = 1;
constexpr uint32_t TILE_BYTES = T * D * 2;   // 32 KB
constexpr uint32_t HALF_BYTES = T * 64 * 2;  // one 64-column swizzled block
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = TILE_BYTES;
constexpr uint32_t OFF_V = OFF_K + NSK * TILE_BYTES;
constexpr uint32_t OFF_X = OFF_V + TILE_BYTES;  // half-row exchange: max[2][128], sum[2][128]
constexpr uint32_t OFF_BAR = OFF_X + 4 * T * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 384;
constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, false, true);
constexpr float kRescaleLog2 = 8.f;  // lazy O rescale threshold (log2 units)

struct Params {
  __nv_bfloat16* O;
  float* O32;  // optional float32 copy of O (nullptr: not written)
  float* LSE;
  int L;
  int nb;
  float scale_log2;
  float log2_tau;
  int never_skip;
  int32_t* kept_tiles;
  uint32_t* keep_bits;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSK];
  uint64_t k_empty[NSK];
  uint64_t s_full[NSB];
  uint64_t decision[NSB];
  uint64_t v_full;
  uint64_t pv_done;
  int keepflag[NSB];
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

__global__ void __launch_bounds__(NT, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(base + OFF_BAR);
  float* xmax = reinterpret_cast<float*>(base + OFF_X);  // [2][128]
  float* xsum = xmax + 2 * T;                            // [2][128]
  volatile int* abort = &bars.abort;
  const uint32_t sbase = smem_u32(base);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int i = p.nb - 1 - (int)blockIdx.x;  // longest query blocks first
  const int z = blockIdx.y;
  const int ntiles = i + 1;  // tile t <-> key block i - t

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 1);
    }
    for (int b = 0; b < NSB; ++b) {
      mbar_init(smem_u32(&bars.s_full[b]), 1);
      mbar_init(smem_u32(&bars.decision[b]), 1);
    }
    mbar_init(smem_u32(&bars.v_full), 1);
    mbar_init(smem_u32(&bars.pv_done), 1);
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint32_t qb = smem_u32(&bars.q_full);
      mbar_expect_tx(qb, TILE_BYTES);
      tma_load_3d(sbase + OFF_Q, &tmQ, 0, i * T, z, qb);
      tma_load_3d(sbase + OFF_Q + HALF_BYTES, &tmQ, 64, i * T, z, qb);
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NSK;
        if (t >= NSK) mbar_wait(smem_u32(&bars.k_empty[s]), ((t / NSK) - 1) & 1, abort, 0x111);
        const uint32_t kb = smem_u32(&bars.k_full[s]);
        const uint32_t dst = sbase + OFF_K + s * TILE_BYTES;
        mbar_expect_tx(kb, TILE_BYTES);
        tma_load_3d(dst, &tmK, 0, (i - t) * T, z, kb);
        tma_load_3d(dst + HALF_BYTES, &tmK, 64, (i - t) * T, z, kb);
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dq = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sbase + OFF_K, 16, 1024);
      const uint64_t dv = sdesc_sw128(sbase + OFF_V, HALF_BYTES, 1024);
      uint32_t v_ph = 0;
      int pv_count = 0;
      mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x112);
      int t_retire = 0;  // oldest tile whose decision is still pending
      // Decision on tile t_retire (buffer t_retire % NSB); P V if it was kept.
      auto retire = [&]() {
        const int b = t_retire % NSB;
        mbar_wait_spin(smem_u32(&bars.decision[b]), (t_retire / NSB) & 1, abort, 0x114);
        if (*reinterpret_cast<volatile int*>(&bars.keepflag[b])) {
          mbar_wait(smem_u32(&bars.v_full), v_ph, abort, 0x115);
          v_ph ^= 1;
          tc_fence_after();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < T / 16; ++kk) {
              const uint32_t a_t = tmem + b * 128 + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half;
              mma_bf16_ts(tmem + TMEM_O, a_t, dv + (uint64_t)((kk * 2048) >> 4), IDESC_PV,
                          (pv_count > 0 || half > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(smem_u32(&bars.pv_done));
          ++pv_count;
        }
        ++t_retire;
      };
      for (int t = 0; t < ntiles; ++t) {
        const int b = t % NSB;
        if (t >= NSB) retire();  // buffer b: tile t - NSB decided (and its PV issued)
        const int s = t % NSK;
        mbar_wait(smem_u32(&bars.k_full[s]), (t / NSK) & 1, abort, 0x113);
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((s * TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16(tmem + b * 128, sdesc_kstep(dq, kk, HALF_BYTES), sdesc_kstep(dk, kk, HALF_BYTES),
                   IDESC_QK, kk > 0);
        mma_commit(smem_u32(&bars.s_full[b]));
        mma_commit(smem_u32(&bars.k_empty[s]));
      }
      while (t_retire < ntiles) retire();
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ test / softmax
    const int h = warp >> 2;  // column half
    const int r = (warp & 3) * 32 + lane;
    const int col0 = 64 * h;
    const int row = i * T + r;
    const bool row_valid = row < p.L;
    const float thr = p.never_skip ? 0.f : (p.log2_tau - __log2f((float)(row + 1)));
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base + TMEM_O + col0;
    float m_ref = kNegInf, l = 0.f;
    float bound_raw = kNegInf;  // keep iff raw row max >= bound_raw
    int n_kept = 0;
    const int nw = (p.nb + 31) >> 5;
    KeepBits kb;
    kb.init(tid == 0 ? p.keep_bits : nullptr, ((size_t)z * p.nb + i) * nw);
    if (tid == 0 && p.keep_bits)
      for (int w = i / 32 + 1; w < nw; ++w) p.keep_bits[((size_t)z * p.nb + i) * nw + w] = 0u;

    for (int t = 0; t < ntiles; ++t) {
      const int b = t % NSB;
      const int j = i - t;
      const bool diag = (t == 0);
      const uint32_t t_s = tmem + lane_base + b * 128 + col0;
      mbar_wait(smem_u32(&bars.s_full[b]), (t / NSB) & 1, abort, 0x116);
      tc_fence_after();
      const float hm = tmem_rowmax64(t_s, diag, r, col0);
      int want = diag || p.never_skip;
      if (!want && row_valid) want = hm >= bound_raw;
      tc_fence_before();
      const int keep = bar_vote_or(want, BAR_SOFT, NSOFT);
      kb.set(j, keep != 0);
      if (!keep) {
        if (tid == 0) {
          bars.keepflag[b] = 0;
          mbar_arrive(smem_u32(&bars.decision[b]));
        }
        continue;
      }
      // ---- kept tile ------------------------------------------------------
      if (n_kept > 0) {  // the previous P V reads V and accumulates into O
        mbar_wait(smem_u32(&bars.pv_done), (n_kept - 1) & 1, abort, 0x117);
        tc_fence_after();
      }
      if (tid == 0) {
        const uint32_t vb = smem_u32(&bars.v_full);
        mbar_expect_tx(vb, TILE_BYTES);
        tma_load_3d(sbase + OFF_V, &tmV, 0, j * T, z, vb);
        tma_load_3d(sbase + OFF_V + HALF_BYTES, &tmV, 64, j * T, z, vb);
      }
      xmax[h * T + r] = hm;
      bar_sync_n(BAR_SOFT, NSOFT);
      const float mt = fmaxf(xmax[r], xmax[T + r]) * p.scale_log2;
      const float m_new = fmaxf(m_ref, mt);
      const bool first = (n_kept == 0);
      const bool need = !first && (m_new > m_ref + kRescaleLog2);
      if (first) {
        m_ref = m_new;
      } else if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? exp2f(m_ref - m_new) : 1.f;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
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
      // P = exp2(s2 - m_ref) over this thread's 64 columns, as hi + lo pairs
      float lsum = 0.f;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float s[32];
        tmem_ld32(t_s + ch * 32, s);
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int col = col0 + ch * 32 + e;
          const float p0 = (diag && col > r) ? 0.f : exp2f(s[e] * p.scale_log2 - m_ref);
          const float p1 = (diag && col + 1 > r) ? 0.f : exp2f(s[e + 1] * p.scale_log2 - m_ref);
          lsum += p0 + p1;
          const __nv_bfloat162 hh = __floats2bfloat162_rn(p0, p1);
          const float2 hf = __bfloat1622float2(hh);
          w[e >> 1] = *reinterpret_cast<const uint32_t*>(&hh);
          w[16 + (e >> 1)] = pack_bf16(p0 - hf.x, p1 - hf.y);
        }
        tmem_st32(t_s + ch * 32, w);
      }
      xsum[h * T + r] = lsum;
      tc_fence_before();
      bar_sync_n(BAR_SOFT, NSOFT);
      l += xsum[r] + xsum[T + r];
      ++n_kept;
      bound_raw = (thr + m_ref + __log2f(l)) / p.scale_log2;
      if (tid == 0) {
        bars.keepflag[b] = 1;
        mbar_arrive(smem_u32(&bars.decision[b]));
      }
    }
    kb.flush();
    // ---- epilogue: O = O_acc / l, LSE = (m + log2 l) ln 2 ---------------------
    mbar_wait(smem_u32(&bars.pv_done), (n_kept - 1) & 1, abort, 0x118);
    tc_fence_after();
    const float inv = 1.f / l;
    const size_t orow = ((size_t)z * p.L + (row_valid ? row : 0)) * D + col0;
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
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
    if (h == 0 && row_valid) p.LSE[(size_t)z * p.L + row] = (m_ref + __log2f(l)) * kLn2;
    if (tid == 0 && p.kept_tiles) p.kept_tiles[(size_t)z * p.nb + i] = n_kept;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fwd100
}  // namespace mala
