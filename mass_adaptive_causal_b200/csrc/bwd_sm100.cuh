// bwd_sm100.cuh -- MALA backward work pass for bf16, d = 128, 128 x 128
// tiles on the 5th-generation tensor cores (tcgen05 + TMEM), operands staged
// by TMA.
//
// Rule (MassAlloc Attention; agihunt.info summary, backward paragraph;
// jaehun.me review, "Backward: offline sparse probabilities"): the backward
// reuses the forward's final log-normalizer LSE; a tile whose every valid row
// has max_c S_rc - LSE_r < ln tau - ln(r+1) is skipped. The test of every
// legal tile runs first (bwd_test_sm100.cuh) and leaves one bit per tile;
// this pass does the post-score work of the kept tiles only:
//   P = exp(S - LSE), dV_j += P^T dO_i, dP = dO_i V_j^T, dS = P o (dP - D),
//   dK_j += scale dS^T Q_i, dQ_i += scale dS K_j.
//
// Persistent CTAs (256 threads, one per SM) take key columns (key block j
// of a key/value head) in turn; a column's K_j, V_j and diagonal block load
// while the previous column writes its dK, dV. Per column a CTA lists the
// kept query blocks i >= j of its column of the bit matrix, then for each:
// S^T = K_j Q_i^T (keys in TMEM lanes) with dP^T = V_j dO_i^T behind it, P,
// dV, dS, then dK and dQ, each stage on its own barrier. Q alternates
// between two buffers and loads two tiles ahead, as each tile's dK product
// frees its buffer; the next tile's S^T is issued right behind the tile's dQ
// product, so the tensor cores compute it while the threads read dQ out; the
// next dO loads once dP^T and dV have read the current one. dK_j, dV_j accumulate in TMEM. Threads t and
// t + 128 own TMEM lane t mod 128 and split the 128 columns of each
// accumulator into halves, so the elementwise work of a tile (P, dS, the dQ
// readout) is spread over 8 warps:
//   TMEM [  0,128): S^T = K_j Q_i^T
//   TMEM [128,256): dP^T = V_j dO_i^T, later reused for dQ_i = dS K_j
//   TMEM [256,384): dK_j accumulator      TMEM [384,512): dV_j accumulator
// Shared memory: K_j, V_j, Q_i (two), dO_i, P^T, dS^T (32 KB each, 128-byte
// swizzle) + per-query LSE and D, and the kept blocks as a bit mask.
// dS goes to the dQ product as a bf16 pair hi + lo (dQ sums rows of dS
// that cancel), to the dK product as hi alone; dQ_i is read back from TMEM
// (query rows in lanes) into a float32 tile in the then free P^T and dS^T
// buffers and added into a float32 workspace by four TMA bulk tensor
// reductions (the adds happen in L2, a 16 KB block per instruction, instead
// of 4096 float4 atomics from the threads), converted afterwards. The next
// tile forms its P while the reductions read the tile and stores P after.
#pragma once

#include "sm100.cuh"

namespace mala {
namespace bwd100 {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 256;
constexpr int NWARP = NT / 32;
// The thread that issues the bulk copies out of shared memory (dQ
// reductions, dK / dV stores) and owns their bulk async-groups; thread 0
// issues the loads and MMAs.
constexpr int BULK_TID = 32;
constexpr uint32_t TILE_BYTES = T * D * 2;
constexpr uint32_t HALF_BYTES = T * 64 * 2;
constexpr int LIST_CHUNK = 1024;  // query blocks listed per round
constexpr int LIST_ROUNDS = LIST_CHUNK / NT;
constexpr int MASK_WORDS = LIST_CHUNK / 32;
static_assert(MASK_WORDS == LIST_ROUNDS * NWARP, "one mask word per warp and listing round");
// K, V, Q (two buffers), dO, P^T, dS^T; LSE and D (two buffers each); the
// barriers; the kept-block masks and their per-warp nonzero-word bits (two)
constexpr uint32_t SMEM_BYTES = 7 * TILE_BYTES + 2048 + 128 + 2 * (MASK_WORDS + NWARP) * 4;
static_assert(SMEM_BYTES <= 227 * 1024, "the work pass must fit one CTA's shared memory");
constexpr uint32_t TMEM_COLS = 512;
// S^T, dP^T: A = K_j or V_j (K-major over d), B = Q_i or dO_i (K-major over d)
constexpr uint32_t IDESC_KQ = idesc_bf16(128, 128, false, false);
// dV, dK: A = P^T or dS^T (K-major over queries), B = dO_i or Q_i (MN-major: d contiguous)
constexpr uint32_t IDESC_ACC = idesc_bf16(128, 128, false, true);
// dQ: A = dS (queries contiguous in dS^T rows: MN-major), B = K_j (MN-major)
constexpr uint32_t IDESC_DQ = idesc_bf16(128, 128, true, true);

struct Params {
  const float* LSE;
  const float* Dterm;
  float* dQacc;
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  int L;
  int nb;
  float scale;       // softmax scale (dS is scaled before the bf16 cast)
  float scale_log2;  // scale * log2(e)
  int never_skip;    // tau == 0: every legal tile is kept (no bits read)
  int32_t* kept_tiles;   // [B * Hq][nb]
  const uint32_t* bits;  // [B * Hq][nb][nw] from the test pass
  int Hq, Hkv, G;        // query heads, key/value heads, G = Hq / Hkv
  int Zkv;               // B * Hkv
  int* item_counter;     // zeroed before the launch: columns handed out past the first
};

// Row `row` of a TMEM accumulator (this thread's lane, 128 columns) -> bf16
// row of a 128 x 128 shared tile in the two 64-column halves and 128-byte
// swizzle of the bf16 tensor maps. Every lane of the warp must call it
// (tcgen05.ld is warp-collective).
__device__ __forceinline__ void stage_row_bf16(uint32_t dst, int row, uint32_t taddr) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      st_shared_v4(dst + sw128_chunk_off(row, c * 32 + q * 8, T), pack_bf16(v[8 * q + 0], v[8 * q + 1]),
                   pack_bf16(v[8 * q + 2], v[8 * q + 3]), pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                   pack_bf16(v[8 * q + 6], v[8 * q + 7]));
  }
}

__global__ void __launch_bounds__(NT, 1)
    bwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmdK,
                    const __grid_constant__ CUtensorMap tmdV, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = smem_raw;
  // 128-byte swizzled tiles need a 1024-byte aligned base
  if (smem_u32(base) & 1023u) {
    if (threadIdx.x == 0) record_layout_error(0x2f2);
    return;
  }
  const uint32_t ka = smem_u32(base);
  const uint32_t va = ka + TILE_BYTES;
  // Q_i of the CTA's tiles alternate between two buffers (tile count parity),
  // so the next tile's Q loads a whole tile ahead
  const uint32_t qa0 = ka + 2 * TILE_BYTES;
  const uint32_t da = ka + 4 * TILE_BYTES;   // dO_i
  const uint32_t pta = ka + 5 * TILE_BYTES;  // P^T
  const uint32_t sta = ka + 6 * TILE_BYTES;  // dS^T
  // per-query LSE * log2(e) and D, two buffers each: the next kept tile's
  // values land in one while the current tile reads the other
  float* lse_s = reinterpret_cast<float*>(base + 7 * TILE_BYTES);  // [2][128]
  float* dd_s = lse_s + 2 * T;                                      // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(dd_s + 2 * T);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* kmask = reinterpret_cast<uint32_t*>(bars + 16);  // [2][MASK_WORDS]
  uint32_t* knz = kmask + 2 * MASK_WORDS;                     // [2][NWARP]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // Warps w and w + 4 share TMEM lanes 32 (w mod 4) .. +31 and split the
  // 128 columns of each accumulator into halves: row = this thread's lane
  // of the tile (a key for S^T / dP^T, a query for dQ), half = which 64.
  const int row = tid & (T - 1);
  const int half = warp >> 2;
  // Columns c = zkv * nb + j (key block j of key/value head zkv), key blocks
  // ascending within a head. The first gridDim.x columns go one to a CTA;
  // after that a CTA takes the next column from a counter, so CTAs that run
  // together work on neighbouring key blocks of one head (their kept query
  // blocks, and the dQ rows they add into, mostly coincide and stay in L2).
  const int n_items = p.nb * p.Zkv;
  int* item_slot = reinterpret_cast<int*>(tmem_slot + 2);
  const uint32_t bar_kv = smem_u32(&bars[0]);
  const uint32_t bar_q0 = smem_u32(&bars[1]);  // Q buffer b: bar_q0 + 8 b
  const uint32_t bar_do = smem_u32(&bars[3]);
  // one completion per tile each: S^T; dP^T and dV; dK; dQ (a commit
  // covers every earlier MMA of the issuing thread)
  const uint32_t bar_s = smem_u32(&bars[4]);
  const uint32_t bar_dv = smem_u32(&bars[5]);
  const uint32_t bar_dk = smem_u32(&bars[6]);
  const uint32_t bar_dq = smem_u32(&bars[7]);
  const uint32_t bar_fin = smem_u32(&bars[8]);  // the exit's wait for every MMA

  if (tid == 0) {
    mbar_init(bar_kv, 1);
    mbar_init(bar_q0, 1);
    mbar_init(bar_q0 + 8, 1);
    mbar_init(bar_do, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_dv, 1);
    mbar_init(bar_dk, 1);
    mbar_init(bar_dq, 1);
    mbar_init(bar_fin, 1);
    *abort = 0;
    fence_mbar_init();
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
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t t_st = tmem + lane_base + half * 64;         // S^T
  const uint32_t t_dpt = tmem + lane_base + 128 + half * 64;  // dP^T, then dQ
  const uint32_t t_dk = tmem + lane_base + 256;
  const uint32_t t_dv = tmem + lane_base + 384;

  // Phases and copies in flight; thread 0 issues every load and MMA, so its
  // own view is the one that the exit path settles (the bulk copies out of
  // shared memory are BULK_TID's). Only thread 0 waits on the Q barriers:
  // bit b of ph_qm / q_pendm is Q buffer b's.
  uint32_t ph_qm = 0, ph_do = 0, ph_s = 0, ph_dv = 0, ph_dk = 0, ph_dq = 0;
  uint32_t q_pendm = 0;
  bool kv_pend = false, do_pend = false;
  int tcount = 0;  // tiles done by this CTA: picks the Q and the LSE / D buffers
  int nlist = 0;   // listings done by this CTA: picks the mask buffer
  uint32_t ph_kv = 0;
  bool ok = true;
  const int nw = (p.nb + 31) >> 5;
  // Loads of column c that need no listing: K_j, V_j and, since the diagonal
  // block (first query head) is nearly always the column's first kept tile,
  // its Q, dO, LSE and D (into buffers tcount & 1). A column whose
  // first kept tile is another block lets these copies land before it fetches
  // its own into the same buffers.
  auto column_row_term = [&](int c) {  // this thread's LSE (half 0) or D of the diagonal block
    const int j = c % p.nb, zkv = c / p.nb;
    const int zq0 = (zkv / p.Hkv) * p.Hq + (zkv % p.Hkv) * p.G;
    const int q = j * T + row;
    if (q >= p.L) return 0.f;
    return half == 0 ? p.LSE[(size_t)zq0 * p.L + q] * kLog2e : p.Dterm[(size_t)zq0 * p.L + q];
  };
  auto store_row_term = [&](float v) {
    if (half == 0)
      lse_s[(tcount & 1) * T + row] = v;
    else
      dd_s[(tcount & 1) * T + row] = v;
  };
  auto issue_column_copies = [&](int c) {
    const int j = c % p.nb, zkv = c / p.nb;
    const int zq0 = (zkv / p.Hkv) * p.Hq + (zkv % p.Hkv) * p.G;
    if (tid == 0) {
      mbar_expect_tx(bar_kv, 2 * TILE_BYTES);
      tma_load_3d(ka, &tmK, 0, j * T, zkv, bar_kv);
      tma_load_3d(ka + HALF_BYTES, &tmK, 64, j * T, zkv, bar_kv);
      tma_load_3d(va, &tmV, 0, j * T, zkv, bar_kv);
      tma_load_3d(va + HALF_BYTES, &tmV, 64, j * T, zkv, bar_kv);
      const int b = tcount & 1;
      const uint32_t qb = qa0 + b * TILE_BYTES, bq = bar_q0 + 8 * b;
      mbar_expect_tx(bq, TILE_BYTES);
      tma_load_3d(qb, &tmQ, 0, j * T, zq0, bq);
      tma_load_3d(qb + HALF_BYTES, &tmQ, 64, j * T, zq0, bq);
      mbar_expect_tx(bar_do, TILE_BYTES);
      tma_load_3d(da, &tmdO, 0, j * T, zq0, bar_do);
      tma_load_3d(da + HALF_BYTES, &tmdO, 64, j * T, zq0, bar_do);
      kv_pend = do_pend = true;
      q_pendm |= 1u << b;
    }
  };
  int col = blockIdx.x;
  if (col < n_items) {
    issue_column_copies(col);
    store_row_term(column_row_term(col));
  }
  while (col < n_items && ok) {
  const int j = col % p.nb;    // key block
  const int zkv = col / p.nb;  // (b, key/value head): K_j, V_j, dK_j, dV_j
  // dK_j and dV_j sum over the G query heads that share this key/value head
  const int zq0 = (zkv / p.Hkv) * p.Hq + (zkv % p.Hkv) * p.G;
  // the next column, taken now so that its loads can start as soon as this
  // column's last products have read the buffers (the value is first needed
  // at the column's end, so the counter's round trip is not waited for here)
  int fetched = 0;
  if (tid == 0) fetched = (int)gridDim.x + atomicAdd(p.item_counter, 1);
  bool kv_ready = false;
  int kept_count = 0;
  bool spec = true;  // the diagonal's copies are still unclaimed

  for (int hg = 0; hg < p.G && ok; ++hg) {
  const int z = zq0 + hg;  // query head: Q_i, dO_i, LSE, D, dQ, the keep bits
  const int kept_before = kept_count;
  for (int i0 = j; i0 < p.nb && ok; i0 += LIST_CHUNK) {
    // ---- the kept query blocks i in [i0, i0 + LIST_CHUNK) as a bit mask,
    // bit b of word m for block i0 + 32 m + b (every bit word is loaded
    // first, then one barrier publishes the mask); every thread walks it in
    // ascending order. Two masks: a thread still walking the previous one
    // is at most one listing behind.
    bool fk[LIST_ROUNDS];
#pragma unroll
    for (int k = 0; k < LIST_ROUNDS; ++k) {
      const int i = i0 + k * NT + tid;
      const bool in = i < p.nb;
      const uint32_t w =
          (in && !p.never_skip) ? p.bits[((size_t)z * p.nb + i) * nw + (j >> 5)] : 0u;
      fk[k] = in && (p.never_skip || ((w >> (j & 31)) & 1u));
    }
    uint32_t* msk = kmask + (nlist & 1) * MASK_WORDS;
    uint32_t* wnz = knz + (nlist & 1) * NWARP;  // bit k: this warp's word of round k is nonzero
    ++nlist;
    uint32_t nzbits = 0u;
#pragma unroll
    for (int k = 0; k < LIST_ROUNDS; ++k) {
      const unsigned bal = __ballot_sync(0xffffffffu, fk[k]);
      if (lane == 0) msk[k * NWARP + warp] = bal;
      nzbits |= (bal != 0u ? 1u : 0u) << k;
    }
    if (lane == 0) wnz[warp] = nzbits;
    __syncthreads();
    // bit m: mask word m is nonzero, so the walk goes from one kept block's
    // word to the next without reading the empty words between them
    uint32_t nzw = 0u;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) {
      const uint32_t b = wnz[w];
#pragma unroll
      for (int k = 0; k < LIST_ROUNDS; ++k) nzw |= ((b >> k) & 1u) << (k * NWARP + w);
    }
    int mw = -1;
    uint32_t rem = 0u;
    auto next_block = [&]() -> int {  // the next kept block, -1 past the last
      while (rem == 0u) {
        const uint32_t ahead = mw >= MASK_WORDS - 1 ? 0u : nzw & (~0u << (mw + 1));
        if (ahead == 0u) {
          mw = MASK_WORDS;
          return -1;
        }
        mw = __ffs(ahead) - 1;
        rem = msk[mw];
      }
      const int bit = __ffs(rem) - 1;
      rem &= rem - 1u;
      return i0 + 32 * mw + bit;
    };
    // Within a list, tile n + 2's Q loads into tile n's Q buffer once tile
    // n's dK product has read it, and tile n + 1's S^T is issued behind tile
    // n's dQ product; tile n + 1's dO loads once tile n's dP / dV products
    // have read the buffer, its LSE and D into the other buffer. Threads
    // 0-127 move the LSE of query `row`, threads 128-255 its D.
    int cur = next_block();
    int nxt = cur >= 0 ? next_block() : -1;
    int nxt2 = nxt >= 0 ? next_block() : -1;
    bool s_ready = false;  // thread 0: this tile's S^T was issued by the previous tile
    bool first = true;     // the list's first tile
    bool prefetched = false;
    for (; cur >= 0 && ok; cur = nxt, nxt = nxt2, nxt2 = nxt2 >= 0 ? next_block() : -1) {
    const int i = cur;
    const bool has_next = nxt >= 0;
    const int inext = has_next ? nxt : 0;
    const int qb = tcount & 1;  // this tile's Q buffer; the next tile's is qb ^ 1
    const uint32_t qc = qa0 + qb * TILE_BYTES, qn = qa0 + (qb ^ 1) * TILE_BYTES;
    const uint32_t bar_qc = bar_q0 + 8 * qb, bar_qn = bar_q0 + 8 * (qb ^ 1);
    float* lse_c = lse_s + qb * T;
    float* dd_c = dd_s + qb * T;
    if (spec) {
      spec = false;
      if (hg == 0 && i == j) {
        prefetched = true;  // the diagonal's copies (and LSE, D) are this tile's
      } else if (tid == 0) {  // they land before this block's go into the buffers
        if (mbar_wait(bar_qc, (ph_qm >> qb) & 1u, abort, 0x208)) {
          ph_qm ^= 1u << qb;
          q_pendm &= ~(1u << qb);
        } else {
          ok = false;
        }
        if (mbar_wait(bar_do, ph_do, abort, 0x209)) {
          ph_do ^= 1;
          do_pend = false;
        } else {
          ok = false;
        }
      }
    }
    if (!prefetched) {
      const int q = i * T + row;
      const bool qv = q < p.L;
      if (half == 0)
        lse_c[row] = qv ? p.LSE[(size_t)z * p.L + q] * kLog2e : 0.f;
      else
        dd_c[row] = qv ? p.Dterm[(size_t)z * p.L + q] : 0.f;
      if (tid == 0) {
        mbar_expect_tx(bar_qc, TILE_BYTES);
        tma_load_3d(qc, &tmQ, 0, i * T, z, bar_qc);
        tma_load_3d(qc + HALF_BYTES, &tmQ, 64, i * T, z, bar_qc);
        mbar_expect_tx(bar_do, TILE_BYTES);
        tma_load_3d(da, &tmdO, 0, i * T, z, bar_do);
        tma_load_3d(da + HALF_BYTES, &tmdO, 64, i * T, z, bar_do);
        q_pendm |= 1u << qb;
        do_pend = true;
      }
    }
    // the list's second tile's Q into the other buffer, whose last readers
    // (the previous tile's S^T and dK products) have completed; later tiles'
    // Q load two tiles ahead, as each tile's dK product frees its buffer
    if (tid == 0 && first && has_next) {
      mbar_expect_tx(bar_qn, TILE_BYTES);
      tma_load_3d(qn, &tmQ, 0, inext * T, z, bar_qn);
      tma_load_3d(qn + HALF_BYTES, &tmQ, 64, inext * T, z, bar_qn);
      q_pendm |= 1u << (qb ^ 1);
    }
    first = false;
    // next tile's LSE or D: loaded now, stored once this tile is done
    float next_val = 0.f;
    if (has_next) {
      const int q = inext * T + row;
      if (q < p.L) next_val = (half == 0 ? p.LSE : p.Dterm)[(size_t)z * p.L + q];
    }
    if (!kv_ready) {
      if (mbar_wait(bar_kv, ph_kv, abort, 0x201)) {
        kv_pend = false;
      } else {
        ok = false;
      }
      kv_ready = true;
    }
    // ---- S^T = K_j Q_i^T, unless the previous tile issued it; then
    // dP^T = V_j dO_i^T, which needs no P and runs while the threads form P
    // (the previous tile has read its dQ out of these columns)
    if (tid == 0) {
      if (!s_ready) {
        if (mbar_wait(bar_qc, (ph_qm >> qb) & 1u, abort, 0x202)) {
          ph_qm ^= 1u << qb;
          q_pendm &= ~(1u << qb);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            mma_bf16(tmem, sdesc_sw128(ka + off, 16, 1024), sdesc_sw128(qc + off, 16, 1024),
                     IDESC_KQ, kk > 0);
          }
          mma_commit(bar_s);
        } else {
          ok = false;
        }
      }
      if (mbar_wait(bar_do, ph_do, abort, 0x204)) {
        ph_do ^= 1;
        do_pend = false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          mma_bf16(tmem + 128, sdesc_sw128(va + off, 16, 1024), sdesc_sw128(da + off, 16, 1024),
                   IDESC_KQ, kk > 0);
        }
      } else {
        ok = false;
      }
    }
    if (mbar_wait(bar_s, ph_s, abort, 0x203)) {
      ph_s ^= 1;
    } else {
      ok = false;
    }
    if (__syncthreads_or(!ok)) { ok = false; break; }
    tc_fence_after();
    const bool diag = (i == j);
    {
      // P^T row (key `row`) over this thread's 64 queries, fp32 kept for dS
      float pr[T / 2];
      // an interior tile (below the diagonal, every query row < L) masks nothing
      const bool interior = !diag && (i + 1) * T <= p.L;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float s[32];
        tmem_ld32(t_st + c * 32, s);
        const float4* l4 = reinterpret_cast<const float4*>(lse_c + half * 64 + c * 32);
        if (interior) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 lv = l4[e4];
            pr[c * 32 + 4 * e4 + 0] = ex2_approx(s[4 * e4 + 0] * p.scale_log2 - lv.x);
            pr[c * 32 + 4 * e4 + 1] = ex2_approx(s[4 * e4 + 1] * p.scale_log2 - lv.y);
            pr[c * 32 + 4 * e4 + 2] = ex2_approx(s[4 * e4 + 2] * p.scale_log2 - lv.z);
            pr[c * 32 + 4 * e4 + 3] = ex2_approx(s[4 * e4 + 3] * p.scale_log2 - lv.w);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int qc = half * 64 + c * 32 + e;
            const bool legal = (!diag || qc >= row) && (i * T + qc) < p.L;
            pr[c * 32 + e] = legal ? ex2_approx(s[e] * p.scale_log2 - lse_c[qc]) : 0.f;
          }
        }
      }
      // P is formed while the previous tile's dQ reductions read their
      // staging tile (the P^T and dS^T buffers); it is stored once they have
      if (tid == BULK_TID) bulk_wait_read_all();
      __syncthreads();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int q0 = q * 8;
        st_shared_v4(pta + sw128_chunk_off(row, half * 64 + q0, T),
                     pack_bf16(pr[q0], pr[q0 + 1]), pack_bf16(pr[q0 + 2], pr[q0 + 3]),
                     pack_bf16(pr[q0 + 4], pr[q0 + 5]), pack_bf16(pr[q0 + 6], pr[q0 + 7]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // ---- dV += P^T dO_i --------------------------------------------------------
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          mma_bf16(tmem + 384, sdesc_sw128(pta + aoff, 16, 1024),
                   sdesc_sw128(da + kk * 2048, HALF_BYTES, 1024), IDESC_ACC,
                   (kept_count > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_dv);
      }
      if (mbar_wait(bar_dv, ph_dv, abort, 0x205)) {  // dP^T and dV done
        ph_dv ^= 1;
      } else {
        ok = false;
      }
      if (__syncthreads_or(!ok)) { ok = false; break; }
      tc_fence_after();
      // dO_i has been read: the next tile's dO goes into its buffer now
      if (tid == 0 && has_next) {
        mbar_expect_tx(bar_do, TILE_BYTES);
        tma_load_3d(da, &tmdO, 0, inext * T, z, bar_do);
        tma_load_3d(da + HALF_BYTES, &tmdO, 64, inext * T, z, bar_do);
        do_pend = true;
      }
      // ---- dS^T = P^T o (dP^T - D) * scale as a bf16 pair hi + lo --------------
      // dQ sums dS K over keys whose rows of dS cancel (each full row of dS
      // sums to zero), so a single bf16 rounding of dS costs several percent
      // of dQ; hi + lo carries ~16 significant bits. lo goes into the P^T
      // buffer, free now that the dV product has completed.
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float dp[32];
        tmem_ld32(t_dpt + c * 32, dp);
        // D of the tile's query columns half * 64 + c * 32 + ..., four at a time
        const float4* d4 = reinterpret_cast<const float4*>(dd_c + half * 64 + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t whi[4], wlo[4];
          const float4 da = d4[2 * q], db = d4[2 * q + 1];
          const float dv[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int lc = c * 32 + q * 8 + e;  // this thread's column
            const float a = pr[lc] * (dp[q * 8 + e] - dv[e]) * p.scale;
            const float b = pr[lc + 1] * (dp[q * 8 + e + 1] - dv[e + 1]) * p.scale;
            const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
            const float2 hf = __bfloat1622float2(h);
            whi[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            wlo[e >> 1] = pack_bf16(a - hf.x, b - hf.y);
          }
          const uint32_t off = sw128_chunk_off(row, half * 64 + c * 32 + q * 8, T);
          st_shared_v4(sta + off, whi[0], whi[1], whi[2], whi[3]);
          st_shared_v4(pta + off, wlo[0], wlo[1], wlo[2], wlo[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      // ---- dK += hi^T Q_i, then dQ_i = (hi + lo) K_j into the dP^T columns
      // (read into the threads by now), then the next tile's S^T into the
      // S^T columns (P has been formed), its Q having landed meanwhile. dK
      // sums over queries, where dS has no cancelling structure: the single
      // rounding of hi leaves it within ~2e-3 (rel-L2).
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          mma_bf16(tmem + 256, sdesc_sw128(sta + aoff, 16, 1024),
                   sdesc_sw128(qc + kk * 2048, HALF_BYTES, 1024), IDESC_ACC,
                   (kept_count > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_dk);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t src = part == 0 ? sta : pta;
#pragma unroll
          for (int kk = 0; kk < T / 16; ++kk) {
            mma_bf16(tmem + 128, sdesc_sw128(src + kk * 2048, HALF_BYTES, 1024),
                     sdesc_sw128(ka + kk * 2048, HALF_BYTES, 1024), IDESC_DQ,
                     (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(bar_dq);
        s_ready = false;
        if (has_next) {
          if (mbar_wait(bar_qn, (ph_qm >> (qb ^ 1)) & 1u, abort, 0x20d)) {
            ph_qm ^= 1u << (qb ^ 1);
            q_pendm &= ~(1u << (qb ^ 1));
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
              mma_bf16(tmem, sdesc_sw128(ka + off, 16, 1024), sdesc_sw128(qn + off, 16, 1024),
                       IDESC_KQ, kk > 0);
            }
            mma_commit(bar_s);
            s_ready = true;
          } else {
            ok = false;
          }
        }
        // the dK product has read Q_i: the tile after next loads into qc
        if (mbar_wait(bar_dk, ph_dk, abort, 0x207)) {
          ph_dk ^= 1;
          if (nxt2 >= 0) {
            mbar_expect_tx(bar_qc, TILE_BYTES);
            tma_load_3d(qc, &tmQ, 0, nxt2 * T, z, bar_qc);
            tma_load_3d(qc + HALF_BYTES, &tmQ, 64, nxt2 * T, z, bar_qc);
            q_pendm |= 1u << qb;
          }
        } else {
          ok = false;
        }
      }
      if (mbar_wait(bar_dq, ph_dq, abort, 0x206)) {
        ph_dq ^= 1;
      } else {
        ok = false;
      }
      if (__syncthreads_or(!ok)) { ok = false; break; }
      tc_fence_after();
      ++kept_count;
      // ---- dQ_i (lane = query `row`, this thread's 64 of d) into a float32
      // staging tile in the P^T and dS^T buffers (free now, 64 KB
      // contiguous): four blocks of 32 columns, 128 rows of 128 bytes with
      // the 128-byte swizzle of the reduction's tensor map. Thread 0 adds it
      // into the workspace with one bulk reduction per block after the
      // tile's last barrier; rows past L are not written.
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float v[32];
        tmem_ld32(t_dpt + c * 32, v);
        const uint32_t blk = pta + (uint32_t)(2 * half + c) * 16384u + (uint32_t)row * 128u;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          st_shared_v4(blk + ((uint32_t)(q ^ (row & 7)) << 4), __float_as_uint(v[4 * q]),
                       __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]),
                       __float_as_uint(v[4 * q + 3]));
      }
      fence_proxy_async_smem();  // the staging tile visible to the bulk copy
    }
    if (has_next) {
      if (half == 0)
        lse_s[((tcount + 1) & 1) * T + row] = next_val * kLog2e;
      else
        dd_s[((tcount + 1) & 1) * T + row] = next_val;
    }
    prefetched = has_next;
    ++tcount;
    // the TMEM columns (and the LSE / D buffer just filled) are ready for
    // the next tile once every thread is here
    tc_fence_before();
    __syncthreads();
    if (tid == BULK_TID) {
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) tma_reduce_add_3d(&tmdQ, pta + cb * 16384u, cb * 32, i * T, z);
      bulk_commit_group();
    }
    }
  }
  if (tid == 0 && p.kept_tiles) p.kept_tiles[(size_t)z * p.nb + j] = kept_count - kept_before;
  }
  // The column's buffers are free: its last products have completed (or it
  // kept no tile). Copies still unclaimed -- K_j, V_j and the diagonal's
  // when no tile was kept -- land first; then the next column's loads start
  // while this one writes dK_j, dV_j.
  if (!kv_ready) {
    if (!mbar_wait(bar_kv, ph_kv, abort, 0x20a)) ok = false;
  }
  ph_kv ^= 1;
  if (spec && tid == 0) {
    const int b = tcount & 1;
    if (!mbar_wait(bar_q0 + 8 * b, (ph_qm >> b) & 1u, abort, 0x20b)) ok = false;
    ph_qm ^= 1u << b;
    if (!mbar_wait(bar_do, ph_do, abort, 0x20c)) ok = false;
    ph_do ^= 1;
  }
  if (tid == 0) {
    // with every wait met nothing is in flight: the column's last tile loads
    // no next Q, and the diagonal's copies were claimed or waited for
    if (ok) {
      kv_pend = do_pend = false;
      q_pendm = 0u;
    }
    *item_slot = fetched;
  }
  // the epilogue stages dK_j, dV_j in the P^T and dS^T buffers once the last
  // tile's dQ reductions have read them
  if (tid == BULK_TID) bulk_wait_read_all();
  // item_slot written; every thread past its column's loads
  if (__syncthreads_or(!ok)) ok = false;
  const int next = *item_slot;
  const bool more = ok && next < n_items;
  // the next column's copies start now; its LSE / D are loaded now and stored
  // after the epilogue, which does not wait for them
  float next_term = 0.f;
  if (more) {
    issue_column_copies(next);
    next_term = column_row_term(next);
  }

  // ---- epilogue: dK_j (warps 0-3) into the P^T buffer, dV_j (warps 4-7)
  // into the dS^T buffer as bf16 tiles, written out by four bulk tensor
  // stores (rows past L are not written) that run under the next column's
  // first products; the next tile stores its P once they have read the
  // buffers. A column that kept no tile writes zero rows directly.
  const int key = j * T + row;
  if (ok) {
    if (kept_count > 0) {
      tc_fence_after();
      stage_row_bf16(half == 0 ? pta : sta, row, half == 0 ? t_dk : t_dv);
      fence_proxy_async_smem();  // the staged tiles visible to the bulk stores
    } else if (key < p.L) {
      __nv_bfloat16* dst = (half == 0 ? p.dK : p.dV) + ((size_t)zkv * p.L + key) * D;
      uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(dst)[c] = zero;
    }
  }
  if (more) store_row_term(next_term);
  // dK, dV read out of TMEM before the next column's products overwrite them
  tc_fence_before();
  if (__syncthreads_or(!ok)) ok = false;
  tc_fence_after();
  if (ok && kept_count > 0 && tid == BULK_TID) {
    tma_store_3d(&tmdK, pta, 0, j * T, zkv);
    tma_store_3d(&tmdK, pta + HALF_BYTES, 64, j * T, zkv);
    tma_store_3d(&tmdV, sta, 0, j * T, zkv);
    tma_store_3d(&tmdV, sta + HALF_BYTES, 64, j * T, zkv);
    bulk_commit_group();
  }
  col = next;
  }
  // thread 0's copies and MMAs still in flight (anything on the error path)
  // land before the CTA releases its shared memory and TMEM: one last commit
  // covers every MMA it issued
  if (tid == BULK_TID) bulk_wait_all();  // every dQ reduction and dK / dV store has landed
  if (tid == 0) {
    if (kv_pend) mbar_settle(bar_kv, ph_kv);
    if (q_pendm & 1u) mbar_settle(bar_q0, ph_qm & 1u);
    if (q_pendm & 2u) mbar_settle(bar_q0 + 8, (ph_qm >> 1) & 1u);
    if (do_pend) mbar_settle(bar_do, ph_do);
    mma_commit(bar_fin);
    mbar_settle(bar_fin, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace bwd100
}  // namespace mala
