// fwd_sm100.cuh -- MALA forward for bf16, d = 128, 128 x 128 tiles on the
// 5th-generation tensor cores (tcgen05 + TMEM), operands staged by TMA.
//
// Rule (MassAlloc Attention; agihunt.info summary, forward paragraph;
// jaehun.me review, "Forward: online sparse softmax"): per query block i the
// key tiles j = i, i-1, ..., 0 are visited from the diagonal back. Every
// tile's scores S = Q_i K_j^T are computed on the tensor cores; the tile is
// skipped iff every valid row r has  mt_r - m_r - ln l_r < ln tau - ln(r+1).
// Only kept tiles load V_j, update (m, l) and accumulate P V_j. The diagonal
// tile is always kept; the final log-normalizer goes to LSE.
//
// Work is in the log2 domain (s2 = s * scale * log2 e) so that every
// exponential is one ex2; the test is the same inequality divided by ln 2.
//
// CTA layout (128 threads, one query block): thread t owns query row t, which
// is TMEM lane t of both accumulators:
//   TMEM cols [  0,128): S = Q_i K_j^T          (fp32)
//   TMEM cols [128,256): PV = P_j V_j of the current kept tile (fp32)
// The output accumulator O lives in the thread's registers (128 floats), so
// rescaling by exp(m_old - m_new) is a register multiply, and a skipped tile
// touches neither TMEM's PV columns nor O.
//
// Shared memory (1024-byte aligned, 128-byte swizzle, 64-column blocks):
//   Q_i (32 KB), K_j (32 KB), V_j (32 KB), P_hi and P_lo (32 KB each).
// P goes to the tensor cores as a bf16 pair hi + lo (PV = P_hi V + P_lo V),
// so the float32 output carries P to ~16 significant bits: the backward's
// row terms D = <dO, O> are computed from that float32 output, and dQ is
// sensitive to their error.
// K_{j-1} is prefetched by TMA as soon as the S MMA of tile j has consumed
// K_j, so its load overlaps the row-max / test of tile j. V_j is requested
// only after the CTA-wide vote says "keep".
#pragma once

#include "sm100.cuh"

namespace mala {
namespace fwd100 {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 128;
constexpr uint32_t TILE_BYTES = T * D * 2;  // 32 KB
constexpr uint32_t HALF_BYTES = T * 64 * 2; // one 64-column swizzled block
constexpr uint32_t SMEM_BYTES = 5 * TILE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, false, true);

struct Params {
  __nv_bfloat16* O;
  float* O32;  // optional float32 copy of O (nullptr: not written)
  float* LSE;
  int L;
  int nb;
  float scale_log2;  // scale * log2(e)
  float log2_tau;    // log2(tau); unused when never_skip
  int never_skip;    // tau == 0
  int32_t* kept_tiles;
  uint32_t* keep_bits;
};

__global__ void __launch_bounds__(NT, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = base;
  unsigned char* k_s = base + TILE_BYTES;
  unsigned char* v_s = base + 2 * TILE_BYTES;
  unsigned char* p_s = base + 3 * TILE_BYTES;
  unsigned char* pl_s = base + 4 * TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + 5 * TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int i = p.nb - 1 - (int)blockIdx.x;  // longest query blocks first
  const int z = blockIdx.y;                  // (b, h) slice
  const uint32_t bar_qk = smem_u32(&bars[0]);
  const uint32_t bar_v = smem_u32(&bars[1]);
  const uint32_t bar_mma = smem_u32(&bars[2]);
  const uint32_t qa = smem_u32(q_s), ka = smem_u32(k_s), va = smem_u32(v_s), pa = smem_u32(p_s);
  const uint32_t pla = smem_u32(pl_s);

  if (tid == 0) {
    mbar_init(bar_qk, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    *abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t t_s = tmem + lane_base;        // this warp's lanes, S columns
  const uint32_t t_pv = tmem + lane_base + 128; // this warp's lanes, PV columns

  if (tid == 0) {
    mbar_expect_tx(bar_qk, 2 * TILE_BYTES);
    tma_load_3d(qa, &tmQ, 0, i * T, z, bar_qk);
    tma_load_3d(qa + HALF_BYTES, &tmQ, 64, i * T, z, bar_qk);
    tma_load_3d(ka, &tmK, 0, i * T, z, bar_qk);
    tma_load_3d(ka + HALF_BYTES, &tmK, 64, i * T, z, bar_qk);
  }

  const int row = i * T + tid;
  const bool row_valid = row < p.L;
  const float thr = p.never_skip ? 0.f : (p.log2_tau - __log2f((float)(row + 1)));
  float m = kNegInf, l = 0.f;
  float o[D];
#pragma unroll
  for (int e = 0; e < D; ++e) o[e] = 0.f;
  uint32_t ph_qk = 0, ph_v = 0, ph_mma = 0;
  int kept_count = 0;
  const int nw = (p.nb + 31) >> 5;
  KeepBits kb;
  kb.init(tid == 0 ? p.keep_bits : nullptr, ((size_t)z * p.nb + i) * nw);
  if (tid == 0 && p.keep_bits)
    for (int w = i / 32 + 1; w < nw; ++w) p.keep_bits[((size_t)z * p.nb + i) * nw + w] = 0u;

  bool ok = true;
  for (int j = i; j >= 0; --j) {
    // ---- S = Q_i K_j^T on the tensor cores --------------------------------
    if (!mbar_wait(bar_qk, ph_qk, abort, 0x101)) ok = false;
    ph_qk ^= 1;
    if (__syncthreads_or(!ok)) { ok = false; break; }
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
        mma_bf16(tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                 IDESC_QK, kk > 0);
      }
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, ph_mma, abort, 0x102)) ok = false;
    ph_mma ^= 1;
    if (__syncthreads_or(!ok)) { ok = false; break; }
    tc_fence_after();
    // K_j consumed: start loading K_{j-1} now
    if (tid == 0 && j > 0) {
      mbar_expect_tx(bar_qk, TILE_BYTES);
      tma_load_3d(ka, &tmK, 0, (j - 1) * T, z, bar_qk);
      tma_load_3d(ka + HALF_BYTES, &tmK, 64, (j - 1) * T, z, bar_qk);
    }
    // ---- row max of the tile and the online test -------------------------
    const bool diag = (j == i);
    float mt = kNegInf;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float s[32];
      tmem_ld32(t_s + c * 32, s);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int col = c * 32 + e;
        const float v = (diag && col > tid) ? kNegInf : s[e] * p.scale_log2;
        mt = fmaxf(mt, v);
      }
    }
    int want = diag || p.never_skip;
    if (!want && row_valid) want = (mt - m - __log2f(l)) >= thr;
    tc_fence_before();
    const int keep = __syncthreads_or(want);
    kb.set(j, keep != 0);
    if (!keep) continue;  // skipped: no V load, no softmax update, no PV
    ++kept_count;
    if (tid == 0) {
      mbar_expect_tx(bar_v, TILE_BYTES);
      tma_load_3d(va, &tmV, 0, j * T, z, bar_v);
      tma_load_3d(va + HALF_BYTES, &tmV, 64, j * T, z, bar_v);
    }
    // ---- retained tile: P = exp2(s2 - m_new), l and m update -------------
    const float mnew = fmaxf(m, mt);
    const float alpha = (m == kNegInf) ? 0.f : exp2f(m - mnew);
    float lsum = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float s[32];
      tmem_ld32(t_s + c * 32, s);
      uint32_t pk[16], pl[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const int col = c * 32 + e;
        const float v0 = (diag && col > tid) ? 0.f : exp2f(s[e] * p.scale_log2 - mnew);
        const float v1 = (diag && col + 1 > tid) ? 0.f : exp2f(s[e + 1] * p.scale_log2 - mnew);
        lsum += v0 + v1;
        const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
        const float2 hf = __bfloat1622float2(h);
        pk[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
        pl[e >> 1] = pack_bf16(v0 - hf.x, v1 - hf.y);
      }
      // P row tid, keys c*32 .. c*32+31: four 16-byte chunks of hi and of lo
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t off = sw128_chunk_off(tid, c * 32 + q * 8, T);
        st_shared_v4(pa + off, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        st_shared_v4(pla + off, pl[4 * q], pl[4 * q + 1], pl[4 * q + 2], pl[4 * q + 3]);
      }
    }
    l = l * alpha + lsum;
    m = mnew;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- PV = P V_j on the tensor cores ------------------------------------
    if (!mbar_wait(bar_v, ph_v, abort, 0x103)) ok = false;
    ph_v ^= 1;
    if (__syncthreads_or(!ok)) { ok = false; break; }
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t src = part == 0 ? pa : pla;
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          const uint32_t boff = kk * 16 * 128;
          mma_bf16(tmem + 128, sdesc_sw128(src + aoff, 16, 1024),
                   sdesc_sw128(va + boff, HALF_BYTES, 1024), IDESC_PV, (part > 0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit(bar_mma);
    }
    if (!mbar_wait(bar_mma, ph_mma, abort, 0x104)) ok = false;
    ph_mma ^= 1;
    if (__syncthreads_or(!ok)) { ok = false; break; }
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float pv[32];
      tmem_ld32(t_pv + c * 32, pv);
#pragma unroll
      for (int e = 0; e < 32; ++e) o[c * 32 + e] = fmaf(o[c * 32 + e], alpha, pv[e]);
    }
    tc_fence_before();
  }
  kb.flush();

  // ---- epilogue: O = acc / l (bf16), LSE = (m + log2 l) ln 2 ----------------
  if (ok && row_valid) {
    const float inv = 1.f / l;
    uint4* dst = reinterpret_cast<uint4*>(p.O + ((size_t)z * p.L + row) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      uint4 w;
      w.x = pack_bf16(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
      w.y = pack_bf16(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
      w.z = pack_bf16(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
      w.w = pack_bf16(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
      dst[c] = w;
    }
    if (p.O32) {
      float4* d32 = reinterpret_cast<float4*>(p.O32 + ((size_t)z * p.L + row) * D);
#pragma unroll
      for (int c = 0; c < D / 4; ++c)
        d32[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv, o[4 * c + 3] * inv);
    }
    p.LSE[(size_t)z * p.L + row] = (m + __log2f(l)) * kLn2;
  }
  if (tid == 0 && p.kept_tiles) p.kept_tiles[(size_t)z * p.nb + i] = kept_count;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fwd100
}  // namespace mala
