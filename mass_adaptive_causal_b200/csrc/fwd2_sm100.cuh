// fwd2_sm100.cuh -- MALA forward for bf16, d = 128, 128 x 128 tiles, on CTA
// pairs: each MMA spans two SMs (tcgen05 cta_group::2).
//
// Rule (MassAlloc Attention; agihunt.info summary, forward paragraph;
// jaehun.me review, "Forward: online sparse softmax"): per query block i the
// key tiles j = i, i-1, ..., 0 are visited from the diagonal back. Every
// tile's scores S = Q_i K_j^T are computed on the tensor cores; the tile is
// skipped iff every valid row r has  mt_r - m_r - ln l_r < ln tau - ln(r+1),
// i.e. exp(mt - m) / l < tau / Lq. Only kept tiles read V_j, update (m, l) and
// accumulate P V_j. The diagonal tile is always kept; the final
// log-normalizer goes to LSE. Work is in log2 units (s2 = s * scale * log2 e).
//
// Cluster = two CTAs on two SMs, one query block each: rank 0 has block
// i0 = 2c, rank 1 block i1 = 2c + 1 (same (b, h)). They visit the same key
// tiles K_{i1}, K_{i0}, ..., K_0. Every QK is one M = 256 MMA issued by rank 0
// (the leader): A is each CTA's own Q block, B (the key tile) is split by
// rows, 64 keys in each CTA's shared memory, so each SM loads half of every
// K tile; each CTA's TMEM receives its own 128 x 128 block of S. A kept
// tile's PV is one M = 256 MMA as well (A = each CTA's P from its TMEM, B = V
// split by columns, 64 of d in each CTA); the rows of a CTA that did not
// keep the tile are masked out of D, so its O is untouched.
//
// TMEM (512 columns per SM): a ring of three S buffers [0, 384) and O
// [384, 512). The ring lets the leader issue the next two tiles' QKs while a
// tile is being tested, so the test's latency is off the tensor pipe's path.
//
// Warp roles (288 threads per CTA):
//   warps 0-3  softmax / test of this CTA's block (thread r owns row r = TMEM lane r)
//   warp  4    K producer: this CTA's Q block, then its half of each K tile (6 stages)
//   warp  5    V producer: this CTA's half (64 columns of d) of each V tile a PV needs
//   warps 6, 7 (leader) QK issuers for even / odd tiles. An issuing thread's own
//              shared-memory polls wait until its queued MMAs are dispatched, so
//              two issuers keep the pipe fed while either one waits.
//   warp  8    (leader) decisions: gathers both CTAs' votes per tile, requests V,
//              issues PV, frees the S buffer for the QK four tiles later
//
// Every mbarrier wait is bounded; a wait that runs out records a timeout in
// the device status word and the thread carries on, so every thread reaches
// the final cluster barrier: the kernel always terminates.
#pragma once

#include "sm100.cuh"

namespace mala {
namespace fwd2 {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 288;
constexpr int WARP_KPROD = 4;
constexpr int WARP_VPROD = 5;
constexpr int WARP_QK0 = 6;  // also allocates TMEM (the same warp in both CTAs)
constexpr int WARP_QK1 = 7;
constexpr int WARP_DEC = 8;
constexpr int NSK = 6;    // K half stages (even, so one stage's tiles share an issuer)
constexpr int NSV = 2;    // V half stages
constexpr int NSLOT = 3;  // S buffers
constexpr uint32_t Q_BYTES = T * D * 2;     // 32 KB: this CTA's query block
constexpr uint32_t QH_BYTES = T * 64 * 2;   // one 64-column swizzled block of Q
constexpr uint32_t KH_BYTES = 64 * D * 2;   // 16 KB: 64 keys x 128 d
constexpr uint32_t KH_BLK = 64 * 64 * 2;    // 8 KB: one 64-column block of a K half
constexpr uint32_t VH_BYTES = T * 64 * 2;   // 16 KB: 128 keys x 64 columns of d
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_V = OFF_K + NSK * KH_BYTES;
constexpr uint32_t OFF_BAR = OFF_V + NSV * VH_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 384;
constexpr uint32_t IDESC_QK = idesc_bf16(256, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(256, 128, false, true);
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
  int Hq, G;  // query heads; G query heads share each key/value head
  // Chunks appended to a KV cache, packed (the VARLEN instantiation):
  // sequence b's queries are tokens [cu_q[b], cu_q[b+1]) of Q [total_q][Hq][d],
  // its keys / values tokens [cu_k[b], cu_k[b+1]) of K, V [total_k][Hkv][d];
  // its query r sits at position off + r, off = Lk - Lq. Key tiles are
  // aligned to the chunk's query blocks: tile k starts at position
  // off + T (k - koff), koff = ceil(off / T); positions below 0 are masked.
  const int* cu_q;
  const int* cu_k;
  int total_q;
  int nbq_max;  // trace rows per (b, h)
  int nw;       // trace words per row
};

struct Bars {
  uint64_t q_full;            // leader: both CTAs' Q blocks
  uint64_t k_full[NSK];       // leader: both halves of a K tile
  uint64_t k_empty[NSK];      // each CTA: stage free again
  uint64_t s_full[NSLOT];     // each CTA: S of the slot's tile is in TMEM
  // leader: a CTA's decision for a slot's tile arrives on exactly one of
  // these two (per slot and rank), so the signal carries no data
  uint64_t dec_keep[NSLOT][2];
  uint64_t dec_skip[NSLOT][2];
  uint64_t slot_free[NSLOT];  // leader: the slot may take the next QK
  uint64_t v_req[NSV];        // each CTA: a V half to load (tile in req_j)
  uint64_t v_full[NSV];       // leader: both V halves loaded
  uint64_t v_empty[NSV];      // each CTA: V stage free again
  uint64_t pv_done;           // each CTA: one arrival per PV that updated its O
  int req_j[NSV];             // each CTA: key block of a V request, -1 = stop
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier block");
static_assert(NSK % 2 == 0, "a K stage's tiles must all belong to one issuer");

// OR-vote over the 128 softmax threads on named barrier 1.
__device__ __forceinline__ int vote_or(int pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.cta.red.or.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(out)
      : "r"(pred)
      : "memory");
  return (int)out;
}
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <bool VARLEN>
__global__ void __launch_bounds__(NT, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
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
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  const int z = blockIdx.y;  // (b, query head)
  // this (b, head)'s sequence: query rows, cache offset, TMA coordinates
  int Lq, off, zq, zkv, yq0, yk0;
  if (VARLEN) {
    const int b = z / p.Hq, h = z % p.Hq;
    yq0 = p.cu_q[b];
    yk0 = p.cu_k[b];
    Lq = p.cu_q[b + 1] - yq0;
    off = (p.cu_k[b + 1] - yk0) - Lq;
    zq = h;
    zkv = h / p.G;
  } else {
    Lq = p.L;
    off = 0;
    zq = z;
    zkv = (z / p.Hq) * (p.Hq / p.G) + (z % p.Hq) / p.G;  // its key/value head
    yq0 = yk0 = 0;
  }
  const int nb = (Lq + T - 1) / T;
  const int npairs = (nb + 1) / 2;
  const int koff = (off + T - 1) / T;
  // a cluster beyond this sequence's pairs, or of a sequence with fewer
  // keys than queries (not a cache append), has nothing to do: both CTAs
  // leave together, before any barrier
  if ((int)(blockIdx.x >> 1) >= npairs || off < 0) return;
  // a sequence longer than the stated maxima would overrun the trace rows
  if (VARLEN && (nb > p.nbq_max || nb + koff > 32 * p.nw)) return;
  const int c = npairs - 1 - (int)(blockIdx.x >> 1);  // longest pairs first
  const int i0 = 2 * c, i1 = 2 * c + 1;
  const bool hasB = i1 < nb;
  const bool mine = leader || hasB;  // this CTA has a query block
  const int iX = i0 + (int)rank;
  const int ktop = (hasB ? i1 : i0) + koff;
  const int ntiles = ktop + 1;  // tile t <-> key tile ktop - t
  // first key position of key tile k (below 0 for the oldest tile of a
  // chunk whose cache is not a whole number of tiles)
  auto kpos = [&](int k) { return off + T * (k - koff); };
  // the CTA's block takes part in tile t iff the tile is not past its diagonal
  auto part = [&](int t) { return mine && ktop - t <= iX + koff; };
  // PVs whose V the producers load without a request: the diagonal tiles,
  // always kept (t = 0 for rank 1's block, t = 1 for rank 0's), or every
  // tile when nothing is skipped.
  const int npre = p.never_skip ? ntiles : (hasB ? 2 : 1);

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 1);
    }
    for (int u = 0; u < NSLOT; ++u) {
      mbar_init(smem_u32(&bars.s_full[u]), 1);
      for (int r = 0; r < 2; ++r) {
        mbar_init(smem_u32(&bars.dec_keep[u][r]), 1);
        mbar_init(smem_u32(&bars.dec_skip[u][r]), 1);
      }
      mbar_init(smem_u32(&bars.slot_free[u]), 1);
    }
    for (int v = 0; v < NSV; ++v) {
      mbar_init(smem_u32(&bars.v_req[v]), 1);
      mbar_init(smem_u32(&bars.v_full[v]), 1);
      mbar_init(smem_u32(&bars.v_empty[v]), 1);
    }
    mbar_init(smem_u32(&bars.pv_done), 1);
    bars.abort = 0;
    fence_mbar_init_cluster();
  }
  if (warp == WARP_QK0) {
    tmem_alloc_pair(smem_u32(&bars.tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_slot;
  auto lead = [&](const void* x) { return mapa_rank(smem_u32(x), 0); };

  if (warp == WARP_KPROD) {
    // -------------------------------------------------------------- K producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      if (leader) mbar_expect_tx(smem_u32(&bars.q_full), 2 * Q_BYTES);
      tma_load_3d_pair(sbase + OFF_Q, &tmQ, 0, yq0 + iX * T, zq, lead(&bars.q_full));
      tma_load_3d_pair(sbase + OFF_Q + QH_BYTES, &tmQ, 64, yq0 + iX * T, zq, lead(&bars.q_full));
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % NSK;
        if (t >= NSK && !mbar_wait(smem_u32(&bars.k_empty[s]), ((t / NSK) - 1) & 1, abort, 0x211))
          break;
        if (leader) mbar_expect_tx(smem_u32(&bars.k_full[s]), 2 * KH_BYTES);
        const int row = yk0 + kpos(ktop - t) + 64 * (int)rank;
        const uint32_t dst = sbase + OFF_K + s * KH_BYTES;
        tma_load_3d_pair(dst, &tmK, 0, row, zkv, lead(&bars.k_full[s]));
        tma_load_3d_pair(dst + KH_BLK, &tmK, 64, row, zkv, lead(&bars.k_full[s]));
      }
    }
    __syncwarp();
  } else if (warp == WARP_VPROD) {
    // -------------------------------------------------------------- V producer
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      for (int n = 0;; ++n) {
        const int vs = n % NSV;
        int j;
        if (n < npre) {
          j = ktop - n;  // PV n is tile n
        } else {
          if (!mbar_wait_cluster(smem_u32(&bars.v_req[vs]), ((n - npre) / NSV) & 1, abort, 0x212))
            break;
          j = *reinterpret_cast<volatile int*>(&bars.req_j[vs]);
          if (j < 0) break;
        }
        if (n >= NSV && !mbar_wait(smem_u32(&bars.v_empty[vs]), ((n / NSV) - 1) & 1, abort, 0x213))
          break;
        if (leader) mbar_expect_tx(smem_u32(&bars.v_full[vs]), 2 * VH_BYTES);
        tma_load_3d_pair(sbase + OFF_V + vs * VH_BYTES, &tmV, 64 * (int)rank, yk0 + kpos(j), zkv,
                         lead(&bars.v_full[vs]));
      }
    }
    __syncwarp();
  } else if (warp == WARP_QK0 || warp == WARP_QK1) {
    // ------------------------------------------------- QK issuers (leader only)
    if (leader && lane == 0) {
      const int par = warp - WARP_QK0;
      const uint64_t dq = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      uint64_t dks[NSK];
#pragma unroll
      for (int s = 0; s < NSK; ++s) dks[s] = sdesc_sw128(sbase + OFF_K + s * KH_BYTES, 16, 1024);
      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x214);
      tc_fence_after();
      for (int t = par; ok && t < ntiles; t += 2) {
        const int u = t % NSLOT, s = t % NSK;
        if (t >= NSLOT) {
          ok = mbar_wait_spin(smem_u32(&bars.slot_free[u]), ((t - NSLOT) / NSLOT) & 1, abort, 0x215);
          if (!ok) break;
        }
        ok = mbar_wait(smem_u32(&bars.k_full[s]), (t / NSK) & 1, abort, 0x216);
        if (!ok) break;
        tc_fence_after();
        uint64_t dk = dks[0];
#pragma unroll
        for (int q = 1; q < NSK; ++q)
          if (s == q) dk = dks[q];
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_pair(tmem + u * 128, sdesc_kstep(dq, kk, QH_BYTES), sdesc_kstep(dk, kk, KH_BLK),
                   IDESC_QK, kk > 0, 0u, 0u);
        commit_pair(smem_u32(&bars.s_full[u]), 3);
        commit_pair(smem_u32(&bars.k_empty[s]), 3);
      }
    }
    __syncwarp();
  } else if (warp == WARP_DEC) {
    // ------------------------------------------- decisions and PV (leader only)
    if (leader && lane == 0) {
      uint64_t dvs[NSV];
#pragma unroll
      for (int v = 0; v < NSV; ++v) dvs[v] = sdesc_sw128(sbase + OFF_V + v * VH_BYTES, VH_BYTES, 1024);
      int vcount = 0;
      bool ok = true;
      // parity of the completed phases of dec_keep / dec_skip per slot and
      // rank (bit 8 * rank)
      uint32_t nkeep[NSLOT] = {0, 0, 0}, nskip[NSLOT] = {0, 0, 0};
      for (int t = 0; ok && t < ntiles; ++t) {
        const int u = t % NSLOT;
        int kr[2];
        for (int r = 0; r < 2 && ok; ++r) {
          const uint32_t bk = smem_u32(&bars.dec_keep[u][r]), bs = smem_u32(&bars.dec_skip[u][r]);
          const uint32_t pk = (nkeep[u] >> (8 * r)) & 1u, ps = (nskip[u] >> (8 * r)) & 1u;
          const unsigned long long t0 = globaltimer_ns();
          while (true) {
            if (mbar_test(bk, pk & 1)) { kr[r] = 1; nkeep[u] ^= 1u << (8 * r); break; }
            if (mbar_test(bs, ps & 1)) { kr[r] = 0; nskip[u] ^= 1u << (8 * r); break; }
            if (*abort || globaltimer_ns() - t0 > kWaitLimitNs) {
              if (atomicExch((int*)abort, 1) == 0) record_timeout(0x217);
              ok = false;
              break;
            }
          }
        }
        if (!ok) break;
        const int k0 = kr[0], k1 = kr[1];
        if (k0 | k1) {
          const int vs = vcount % NSV;
          if (vcount >= npre) {  // ask both V producers for tile t
            for (uint32_t r = 0; r < 2; ++r) {
              st_cluster_u32(mapa_rank(smem_u32(&bars.req_j[vs]), r), (uint32_t)(ktop - t));
              mbar_arrive_cluster(mapa_rank(smem_u32(&bars.v_req[vs]), r));
            }
          }
          ok = mbar_wait_spin(smem_u32(&bars.v_full[vs]), (vcount / NSV) & 1, abort, 0x218);
          if (!ok) break;
          tc_fence_after();
          const uint32_t m0 = k0 ? 0u : 0xffffffffu, m1 = k1 ? 0u : 0xffffffffu;
          uint64_t dv = dvs[0];
#pragma unroll
          for (int q = 1; q < NSV; ++q)
            if (vs == q) dv = dvs[q];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < T / 16; ++kk) {
              const uint32_t a_t = tmem + u * 128 + 32 * (kk >> 1) + 8 * (kk & 1) + 16 * half;
              mma_pair_ts(tmem + TMEM_O, a_t, dv + (uint64_t)((kk * 2048) >> 4), IDESC_PV, 1u, m0,
                          m1);
            }
          }
          commit_pair(smem_u32(&bars.v_empty[vs]), 3);
          commit_pair(smem_u32(&bars.pv_done), (uint16_t)((k0 ? 1 : 0) | (k1 ? 2 : 0)));
          commit_pair(smem_u32(&bars.slot_free[u]), 1);
          ++vcount;
        } else {
          mbar_arrive(smem_u32(&bars.slot_free[u]));
        }
      }
      // no further V requests: stop both V producers (a request for key block -1)
      if (vcount >= npre) {
        const int vs = vcount % NSV;
        for (uint32_t r = 0; r < 2; ++r) {
          st_cluster_u32(mapa_rank(smem_u32(&bars.req_j[vs]), r), 0xffffffffu);
          mbar_arrive_cluster(mapa_rank(smem_u32(&bars.v_req[vs]), r));
        }
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------- softmax / test (4 warps)
    const int r = tid;  // 0..127
    const int row = iX * T + r;  // row of the chunk; position off + row
    // (packed chunks: a row past the packed tensor is never written, whatever
    // the offsets say)
    const bool row_valid = mine && row < Lq && (!VARLEN || yq0 + row < p.total_q);
    const float thr = p.never_skip ? 0.f : (p.log2_tau - __log2f((float)(off + row + 1)));
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t t_o = tmem + lane_base + TMEM_O;
    auto signal = [&](int u, int keep) {  // thread 0: this CTA's decision for slot u
      mbar_arrive_remote(keep ? lead(&bars.dec_keep[u][rank]) : lead(&bars.dec_skip[u][rank]));
    };
    // O starts at zero: every PV accumulates (a CTA's first PV may follow
    // PVs of the peer's tiles).
    {
      uint32_t zero[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) zero[e] = 0u;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_st32(t_o + ch * 32, zero);
      tc_fence_before();
    }
    float m_ref = kNegInf, l = 0.f;
    // keep iff mraw * scale_log2 - m_ref - log2 l >= thr; cached as a raw
    // score bound, refreshed whenever (m_ref, l) change
    float bound_raw = kNegInf;
    int n_kept = 0;
    // trace row of this block: bit k of word k / 32 = key tile k kept
    const int nw = VARLEN ? p.nw : (nb + 31) >> 5;
    const size_t brow = (size_t)z * (VARLEN ? p.nbq_max : nb) + iX;
    KeepBits kb;
    kb.init(r == 0 && mine ? p.keep_bits : nullptr, brow * nw);
    if (r == 0 && mine && p.keep_bits)
      for (int w = (iX + koff) / 32 + 1; w < nw; ++w) p.keep_bits[brow * nw + w] = 0u;
    softmax_sync();  // O zeroed by every thread before any decision leaves

    for (int t = 0; t < ntiles; ++t) {
      const int u = t % NSLOT;
      // Wait for the tile's QK even when not taking part: the decision for
      // slot u must not run ahead of the slot's previous use.
      mbar_wait(smem_u32(&bars.s_full[u]), (t / NSLOT) & 1, abort, 0x219);
      tc_fence_after();
      if (!part(t)) {
        if (r == 0) signal(u, 0);
        continue;
      }
      const int j = ktop - t;  // key tile
      const bool diag = (j == iX + koff);
      const int lo = VARLEN ? max(0, -kpos(j)) : 0;  // columns below lo: no key
      const uint32_t t_s = tmem + lane_base + u * 128;
      // ---- row max of the tile (raw scores: the positive scale commutes)
      const float mraw = (VARLEN && lo > 0) ? tmem_rowmax128_from(t_s, lo)
                                            : tmem_rowmax128(t_s, diag, r);
      const float mt = mraw * p.scale_log2;
      int want = diag || p.never_skip;
      if (!want && row_valid) want = mraw >= bound_raw;
      tc_fence_before();
      const int keep = vote_or(want);
      kb.set(j, keep != 0);
      if (!keep) {
        if (r == 0) signal(u, 0);
        continue;
      }
      // ---- kept tile ------------------------------------------------------
      if (n_kept > 0) {  // this CTA's previous PV reads O
        mbar_wait(smem_u32(&bars.pv_done), (n_kept - 1) & 1, abort, 0x21a);
        tc_fence_after();
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
      // ---- P = exp2(s2 - m_ref) as hi + lo bf16 pairs over the S columns:
      // each 32-column chunk holds 16 columns of P_hi and 16 of P_lo
      float lsum = 0.f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float sv[32];
        tmem_ld32(t_s + ch * 32, sv);
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int col = ch * 32 + e;
          const float p0 = ((diag && col > r) || col < lo) ? 0.f
                                                           : exp2f(sv[e] * p.scale_log2 - m_ref);
          const float p1 = ((diag && col + 1 > r) || col + 1 < lo)
                               ? 0.f
                               : exp2f(sv[e + 1] * p.scale_log2 - m_ref);
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
      softmax_sync();  // every row's P and O rescale are in TMEM
      if (r == 0) signal(u, 1);
    }
    kb.flush();
    if (mine && n_kept > 0) {
      // ---- epilogue: O = O_acc / l, LSE = (m + log2 l) ln 2 -----------------
      mbar_wait(smem_u32(&bars.pv_done), (n_kept - 1) & 1, abort, 0x21b);
      tc_fence_after();
      const float inv = 1.f / l;
      const size_t orow = VARLEN ? ((size_t)(yq0 + (row_valid ? row : 0)) * p.Hq + zq) * D
                                 : ((size_t)z * p.L + (row_valid ? row : 0)) * D;
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
      if (row_valid) {
        const size_t li = VARLEN ? (size_t)zq * p.total_q + yq0 + row : (size_t)z * p.L + row;
        p.LSE[li] = (m_ref + __log2f(l)) * kLn2;
      }
      if (r == 0 && p.kept_tiles) p.kept_tiles[brow] = n_kept;
    }
  }
  // both CTAs finish every access to the other's shared memory and TMEM
  // before either frees TMEM or exits
  tc_fence_before();
  cluster_sync_all();
  if (warp == WARP_QK0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace fwd2
}  // namespace mala
