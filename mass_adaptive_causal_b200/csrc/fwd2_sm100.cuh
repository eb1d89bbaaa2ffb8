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
// tile's PV is one M = 256 MMA as well (A = each CTA's P in its shared
// memory, B = V split by columns, 64 of d in each CTA); the rows of a CTA
// that did not keep the tile are masked out of D, so its O is untouched.
//
// With skipping, nearly every tile is a QK followed by a row-max test: per
// tile a test thread waits for S, reads its row from TMEM, reduces it and
// votes, a chain of dependent latencies longer than the tile's MMA. Two
// warpgroups therefore take alternate key tiles of the block, so each has
// two tiles' MMA time for its chain. Skipping stays exact although a group
// tests against the running state it last saw: the bound
// ln tau - ln Lq + m + ln l only grows as tiles are kept, so a tile below an
// old bound is below the current one. A group that wants to keep a tile
// first waits until every earlier tile is final, reloads the state if the
// other group has kept a tile since it last looked, tests again, and only
// then updates the state, so the kept tiles are exactly those of the
// sequential rule. A skipped tile is marked final with one plain store that
// also carries its group's keep count; only a kept tile publishes state, with
// a release store of that count, so no fence sits on the skip path, which
// nearly every tile takes. Each thread holds
// its whole S row in registers and releases the S buffer right after the
// TMEM load. At tau = 0 every tile is kept and the state is sequential, so
// there the eight test warps instead split each row into two column halves.
//
// The QK issuers wait for a tile's K and for the decision ring before they
// wait for its S buffer, so the buffer's release is the last event before
// the MMAs. Rank 1 sends buffer releases and decisions to the leader with
// st.async (a store into the leader's shared memory counted on a leader
// mbarrier), which does not hold up the sending warp.
//
// TMEM (512 columns per SM): three S buffers [0, 384) and O [384, 512).
// Shared memory: Q, K-half stages, two V-half stages, P (hi, lo) buffers.
//
// Warp roles (384 threads per CTA, three warps per scheduler, so a thread
// may use up to 168 registers):
//   warps 0-7  softmax / test (thread t: row t % 128 = TMEM lane, group t / 128)
//   warp  8    producer: this CTA's Q block, its half of each K tile, and its
//              half (64 columns of d) of each V tile a PV needs
//   warps 9, 10 (leader) QK issuers for even / odd tiles. An issuing thread's own
//              shared-memory polls wait until its queued MMAs are dispatched, so
//              two issuers keep the pipe fed while either one waits.
//   warp  11   (leader) decisions: reads both CTAs' decisions per tile, requests V,
//              issues the PVs
//
// Every wait is bounded; a wait that runs out records a timeout in the
// device status word and the thread carries on, so every thread reaches the
// final cluster barrier: the kernel always terminates.
#pragma once

#include "sm100.cuh"

namespace mala {
namespace fwd2 {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 384;
constexpr int NSOFT = 256;  // softmax / test threads
constexpr int WARP_PROD = 8;
constexpr int WARP_QK0 = 9;  // also allocates TMEM (the same warp in both CTAs)
constexpr int WARP_QK1 = 10;
constexpr int WARP_DEC = 11;
constexpr int NSV = 2;    // V half stages
constexpr int NSLOT = 3;  // S buffers
constexpr int RD = 16;    // decision ring: tiles the PV issuer may fall behind the QKs
constexpr int NFIN = 8;   // ring of "tile final" marks between the two test groups
constexpr uint32_t Q_BYTES = T * D * 2;     // 32 KB: this CTA's query block
constexpr uint32_t QH_BYTES = T * 64 * 2;   // one 64-column swizzled block of Q (or P)
constexpr uint32_t KH_BYTES = 64 * D * 2;   // 16 KB: 64 keys x 128 d
constexpr uint32_t KH_BLK = 64 * 64 * 2;    // 8 KB: one 64-column block of a K half
constexpr uint32_t VH_BYTES = T * 64 * 2;   // 16 KB: 128 keys x 64 columns of d
constexpr uint32_t P_BYTES = T * T * 2;     // 32 KB: P_hi (then P_lo), 128 rows x 128 keys
constexpr uint32_t BAR_BYTES = 3072;
constexpr int NSK_MAX = 6;

// Shared-memory plan. With skipping (DENSE = false) nearly every tile is a
// 512-cycle QK, so six K stages cover the L2 latency and one P buffer
// serves the kept tiles, which are rare and finalized in order. At tau = 0
// every tile is kept and costs about three times as long, so two K stages
// suffice and two P buffers let tile t + 1's P be written while tile t's PV
// still reads its own.
template <bool DENSE>
struct Plan {
  static constexpr int NSK = DENSE ? 2 : 6;  // even: one stage's tiles share an issuer
  static constexpr int NPB = DENSE ? 2 : 1;  // P buffers, tile t uses t % NPB
  // S buffer u's full / free barriers come in pairs: tile t uses pair member
  // t % 2, so each barrier serves every sixth tile. Then one test group
  // (DENSE: every test warp) consumes its phases, and one QK issuer (even or
  // odd tiles) arms, waits for or commits them, in order; with one barrier
  // per buffer the two issuers would take alternate phases, and one could
  // arm a phase while the other's earlier phase was still pending.
  static constexpr int SGRP_MASK = 1;
  static constexpr int SPER = 6;                        // tiles between uses of one barrier
  static constexpr uint32_t REL_LOCAL = DENSE ? 8 : 4;  // releasing warps per CTA and tile
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NSK * KH_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + NSV * VH_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + NPB * 2 * P_BYTES;
  // no alignment slack: the kernel requires (and checks) a 1024-byte
  // aligned start, which dynamic shared memory has when a kernel declares
  // no static shared memory
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(NSK % 2 == 0 && NSK <= NSK_MAX, "K stages");
};
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
  uint64_t q_full;                 // leader: both CTAs' Q blocks
  uint64_t k_full[NSK_MAX];        // leader: both halves of a K tile
  uint64_t k_empty[NSK_MAX];       // each CTA: stage free again
  uint64_t s_full[NSLOT][2];       // each CTA: S of a tile is in TMEM (see Plan::SGRP_MASK)
  // leader: S read by both CTAs -- REL_LOCAL arrivals of its own test warps,
  // and one of the QK issuer that arms 4 bytes for each of rank 1's stores
  uint64_t slot_free[NSLOT][2];
  // leader: rank r's decision for tile t is in dec_word[t % RD][r]; rank 0
  // arrives on dec_full[][0] after writing it, rank 1's st.async completes
  // 4 bytes on dec_full[][1], armed by the PV issuer
  uint64_t dec_full[RD][2];
  uint64_t v_req[NSV];             // each CTA: a V half to load (tile in req_j)
  uint64_t v_full[NSV];            // leader: both V halves loaded
  uint64_t v_empty[NSV];           // each CTA: V stage free again
  uint64_t pv_done[2];             // each CTA: one arrival per PV that read P buffer b
  int req_j[NSV];                  // each CTA: key block of a V request, -1 = stop
  int dec_word[RD][2];             // leader: 1 = keep, 0 = skip
  int sink;                        // leader: target of rank 1's buffer-release stores
  int dec_done;                    // leader: tiles whose decisions the PV issuer has read
  // each CTA, between its two test groups. fin[t % NFIN]: tile t is final,
  // written in one 8-byte store as (t + 1) | (kept tiles of its group so
  // far) << 32; kcount[g]: group g's kept tiles, a release store after the
  // group wrote the running (m, l) per row of its latest kept tile
  unsigned long long fin[NFIN];
  int kcount[2];
  union {
    struct {
      float m[T];
      float l[T];
    } st;
    struct {  // tau = 0: a kept tile's half-row maxima and sums
      float max[2][T];
      float sum[2][T];
    } half;
  } x;
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(Bars) <= BAR_BYTES, "barrier block");

// OR-vote over 128 threads on named barrier ID (a compile-time constant).
template <int ID>
__device__ __forceinline__ int vote_or_128(int pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.cta.red.or.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(out)
      : "r"(pred), "n"(ID)
      : "memory");
  return (int)out;
}
template <int ID>
__device__ __forceinline__ void sync_128() {
  asm volatile("barrier.cta.sync %0, 128;" ::"n"(ID) : "memory");
}
__device__ __forceinline__ void sync_256() { asm volatile("barrier.cta.sync 3, 256;" ::: "memory"); }

// The same over a 64-column half row whose tile columns are c0 + e.
__device__ __forceinline__ float half_row_max(const float (&v)[64], int c0, int hi, int lo) {
  const float ninf = -__builtin_huge_valf();
  float a[8];
  if (c0 + 63 <= hi && c0 >= lo) {
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = v[k];
#pragma unroll
    for (int e = 8; e < 56; e += 16) {
#pragma unroll
      for (int k = 0; k < 8; ++k) a[k] = fmax3f(a[k], v[e + k], v[e + 8 + k]);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], v[56 + k]);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = ninf;
#pragma unroll
    for (int e = 0; e < 64; e += 8) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int c = c0 + e + k;
        a[k] = fmaxf(a[k], (c > hi || c < lo) ? ninf : v[e + k]);
      }
    }
  }
  return fmaxf(fmaxf(fmax3f(a[0], a[1], a[2]), fmax3f(a[3], a[4], a[5])), fmaxf(a[6], a[7]));
}

// P = exp2(s * scale_log2 - m) for 8 keys (tile columns col0 .. col0 + 7,
// masked ones 0; MASKED = false: the tile has no masked column) as a bf16
// pair hi + lo, stored into row r of the swizzled P buffers; returns the 8
// values' float sum.
template <bool MASKED>
__device__ __forceinline__ float p_chunk8(const float* s, int col0, int hi, int lo, float scale_log2,
                                          float m, uint32_t p_hi, uint32_t p_lo, int r) {
  uint32_t hw[4], lw[4];
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const int col = col0 + e;
    const bool x0 = MASKED && (col > hi || col < lo);
    const bool x1 = MASKED && (col + 1 > hi || col + 1 < lo);
    const float p0 = x0 ? 0.f : ex2_approx(s[e] * scale_log2 - m);
    const float p1 = x1 ? 0.f : ex2_approx(s[e + 1] * scale_log2 - m);
    sum += p0 + p1;
    const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
    const float2 hf = __bfloat1622float2(hb);
    hw[e >> 1] = *reinterpret_cast<const uint32_t*>(&hb);
    lw[e >> 1] = pack_bf16(p0 - hf.x, p1 - hf.y);
  }
  const uint32_t o = sw128_chunk_off(r, col0, T);
  st_shared_v4(p_hi + o, hw[0], hw[1], hw[2], hw[3]);
  st_shared_v4(p_lo + o, lw[0], lw[1], lw[2], lw[3]);
  return sum;
}

// Scales `ncols` (a multiple of 32) TMEM columns of this thread's lane by a.
__device__ __forceinline__ void tmem_scale(uint32_t taddr, int ncols, float a) {
  for (int ch = 0; ch < ncols; ch += 32) {
    float o[32];
    tmem_ld32(taddr + ch, o);
    uint32_t w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(o[e] * a);
    tmem_st32(taddr + ch, w);
  }
}

// O / l of this thread's row, columns c0 .. c0 + ncols - 1, to bf16 (and
// float32) global memory.
__device__ __forceinline__ void store_o(uint32_t t_o, int c0, int ncols, float inv, bool valid,
                                        __nv_bfloat16* O, float* O32, size_t orow) {
  for (int ch = 0; ch < ncols; ch += 32) {
    float o[32];
    tmem_ld32(t_o + c0 + ch, o);
    if (!valid) continue;
    uint4* d4 = reinterpret_cast<uint4*>(O + orow + c0 + ch);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack_bf16(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
      w.y = pack_bf16(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
      w.z = pack_bf16(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
      w.w = pack_bf16(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
      d4[q] = w;
    }
    if (O32) {
      float4* d32 = reinterpret_cast<float4*>(O32 + orow + c0 + ch);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        d32[q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv,
                             o[4 * q + 3] * inv);
    }
  }
}

// Keep bits of one block's row, set from two test groups: each accumulates
// the bits of its own tiles a word at a time and ORs whole words into the
// (zeroed) row.
struct KeepBitsOr {
  uint32_t* row;
  uint32_t word;
  int cur;
  __device__ __forceinline__ void init(uint32_t* bits, size_t row_off) {
    row = bits ? bits + row_off : nullptr;
    word = 0;
    cur = -1;
  }
  __device__ __forceinline__ void set(int j, bool kept) {
    if (!row) return;
    const int w = j >> 5;
    if (w != cur) {
      if (cur >= 0 && word) atomicOr(&row[cur], word);
      cur = w;
      word = 0;
    }
    if (kept) word |= 1u << (j & 31);
  }
  __device__ __forceinline__ void flush() {
    if (row && cur >= 0 && word) atomicOr(&row[cur], word);
    cur = -1;
  }
};

template <bool VARLEN, bool DENSE>
__global__ void __launch_bounds__(NT, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p) {
  using PL = Plan<DENSE>;
  constexpr int NSK = PL::NSK, NPB = PL::NPB, SPER = PL::SPER;
  constexpr uint32_t OFF_Q = PL::OFF_Q, OFF_K = PL::OFF_K, OFF_V = PL::OFF_V, OFF_P = PL::OFF_P,
                     OFF_BAR = PL::OFF_BAR;
  constexpr uint32_t REL_TX = 4 * PL::REL_LOCAL;  // bytes of rank 1's releases per tile
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = smem_raw;
  // 128-byte swizzled operands need 1024-byte aligned stages; both CTAs of a
  // cluster have the same offset, so both leave here together if it is not
  if (smem_u32(base) & 1023u) {
    if (threadIdx.x == 0) record_layout_error(0x2f0);
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
  // PVs whose V the producer loads without a request: the diagonal tiles,
  // always kept and the first PVs (t = 0 for rank 1's block, t = 1 for rank
  // 0's), or every tile when nothing is skipped.
  const int npre = p.never_skip ? ntiles : (hasB ? 2 : 1);
  // S buffer barrier pair member of tile t
  auto sg = [&](int t) { return t & PL::SGRP_MASK; };

  if (tid == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.k_empty[s]), 1);
    }
    for (int u = 0; u < NSLOT; ++u)
      for (int g = 0; g < 2; ++g) {
        mbar_init(smem_u32(&bars.s_full[u][g]), 1);
        mbar_init(smem_u32(&bars.slot_free[u][g]), PL::REL_LOCAL + 1);
      }
    for (int u = 0; u < RD; ++u)
      for (int r = 0; r < 2; ++r) mbar_init(smem_u32(&bars.dec_full[u][r]), 1);
    for (int v = 0; v < NSV; ++v) {
      mbar_init(smem_u32(&bars.v_req[v]), 1);
      mbar_init(smem_u32(&bars.v_full[v]), 1);
      mbar_init(smem_u32(&bars.v_empty[v]), 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&bars.pv_done[b]), 1);
    bars.dec_done = 0;
    for (int f = 0; f < NFIN; ++f) bars.fin[f] = 0ull;
    bars.kcount[0] = bars.kcount[1] = 0;
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

  if (warp == WARP_PROD) {
    // ----------------------------------------------------------- producer
    // One thread serves two queues in one polling loop: the K halves of
    // tiles 0, 1, ... as stages free up, and the V halves of the PVs in order
    // (preloaded, or requested by the leader's PV issuer).
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (leader) mbar_expect_tx(smem_u32(&bars.q_full), 2 * Q_BYTES);
      tma_load_3d_pair(sbase + OFF_Q, &tmQ, 0, yq0 + iX * T, zq, lead(&bars.q_full));
      tma_load_3d_pair(sbase + OFF_Q + QH_BYTES, &tmQ, 64, yq0 + iX * T, zq, lead(&bars.q_full));
      int tk = 0;   // next K tile
      int nv = 0;   // next V load (PV number)
      int vj = -2;  // key block of V load nv once known (-1: stop, -2: not yet)
      bool vdone = false;
      unsigned long long t0 = globaltimer_ns();
      while ((tk < ntiles || !vdone) && !*abort) {
        bool progress = false;
        if (tk < ntiles) {
          const int s = tk % NSK;
          if (tk < NSK || mbar_test(smem_u32(&bars.k_empty[s]), ((tk / NSK) - 1) & 1)) {
            if (leader) mbar_expect_tx(smem_u32(&bars.k_full[s]), 2 * KH_BYTES);
            const int row = yk0 + kpos(ktop - tk) + 64 * (int)rank;
            const uint32_t dst = sbase + OFF_K + s * KH_BYTES;
            tma_load_3d_pair(dst, &tmK, 0, row, zkv, lead(&bars.k_full[s]));
            tma_load_3d_pair(dst + KH_BLK, &tmK, 64, row, zkv, lead(&bars.k_full[s]));
            ++tk;
            progress = true;
          }
        }
        if (!vdone) {
          const int vs = nv % NSV;
          if (vj == -2) {
            if (nv < npre) {
              vj = ktop - nv;  // PV nv is tile nv
            } else if (mbar_test_cluster(smem_u32(&bars.v_req[vs]), ((nv - npre) / NSV) & 1)) {
              vj = *reinterpret_cast<volatile int*>(&bars.req_j[vs]);
              if (vj < 0) vdone = true;
              progress = true;
            }
          }
          if (vj >= 0 &&
              (nv < NSV || mbar_test(smem_u32(&bars.v_empty[vs]), ((nv / NSV) - 1) & 1))) {
            if (leader) mbar_expect_tx(smem_u32(&bars.v_full[vs]), 2 * VH_BYTES);
            tma_load_3d_pair(sbase + OFF_V + vs * VH_BYTES, &tmV, 64 * (int)rank, yk0 + kpos(vj),
                             zkv, lead(&bars.v_full[vs]));
            ++nv;
            vj = -2;
            progress = true;
          }
        }
        if (progress) {
          t0 = globaltimer_ns();
        } else {
          __nanosleep(32);  // idle: leave the scheduler to the test warps
        }
        if (!progress && globaltimer_ns() - t0 > kWaitLimitNs) {
          if (atomicExch((int*)abort, 1) == 0) record_timeout(0x212);
          break;
        }
      }
    }
    __syncwarp();
  } else if (warp == WARP_QK0 || warp == WARP_QK1) {
    // ------------------------------------------------- QK issuers (leader only)
    if (leader && lane == 0) {
      const int par = warp - WARP_QK0;
      const uint64_t dq = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sbase + OFF_K, 16, 1024);
      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort, 0x214);
      tc_fence_after();
      for (int t = par; ok && t < ntiles; t += 2) {
        const int u = t % NSLOT, s = t % NSK;
        // the tile's K and the decision ring usually are ready long before
        // the S buffer: wait for them first, so that the buffer's release is
        // the last event before the MMAs
        ok = mbar_wait(smem_u32(&bars.k_full[s]), (t / NSK) & 1, abort, 0x216);
        if (!ok) break;
        // tile t's decisions go to ring entry t % RD: the PV issuer must have
        // read that entry's previous tile (t - RD) first
        if (t >= RD) {
          ok = wait_counter(&bars.dec_done, t - RD + 1, abort, 0x21c);
          if (!ok) break;
        }
        if (t >= NSLOT) {  // S of tile t - NSLOT read by both CTAs
          const int tp = t - NSLOT;
          const uint32_t fb = smem_u32(&bars.slot_free[u][sg(tp)]);
          mbar_expect_tx(fb, REL_TX);
          ok = mbar_wait_spin(fb, (tp / SPER) & 1, abort, 0x215);
          if (!ok) break;
        }
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((s * KH_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_pair(tmem + u * 128, sdesc_kstep(dq, kk, QH_BYTES), sdesc_kstep(dk, kk, KH_BLK),
                   IDESC_QK, kk > 0, 0u, 0u);
        commit_pair(smem_u32(&bars.s_full[u][sg(t)]), 3);
        commit_pair(smem_u32(&bars.k_empty[s]), 3);
      }
      // the last NSLOT tiles' buffer releases have no later QK to wait for
      // them: wait here, so that no store of rank 1 is still on its way to
      // this CTA's shared memory when the kernel ends
      for (int t = par; ok && t < ntiles; t += 2) {
        if (t + NSLOT < ntiles) continue;
        const uint32_t fb = smem_u32(&bars.slot_free[t % NSLOT][sg(t)]);
        mbar_expect_tx(fb, REL_TX);
        ok = mbar_wait(fb, (t / SPER) & 1, abort, 0x21d);
      }
    }
    __syncwarp();
  } else if (warp == WARP_DEC) {
    // ------------------------------------------- decisions and PV (leader only)
    if (leader && lane == 0) {
      uint64_t dvs[NSV];
#pragma unroll
      for (int v = 0; v < NSV; ++v) dvs[v] = sdesc_sw128(sbase + OFF_V + v * VH_BYTES, VH_BYTES, 1024);
      const uint64_t dp0 = sdesc_sw128(sbase + OFF_P, 16, 1024);
      int vcount = 0;
      bool ok = true;
      for (int t = 0; ok && t < ntiles; ++t) {
        const int u = t % RD;
        const uint32_t ph = (t / RD) & 1;
        mbar_expect_tx(smem_u32(&bars.dec_full[u][1]), 4);  // rank 1's decision word
        ok = mbar_wait(smem_u32(&bars.dec_full[u][0]), ph, abort, 0x217) &&
             mbar_wait(smem_u32(&bars.dec_full[u][1]), ph, abort, 0x21e);
        if (!ok) break;
        const volatile int* dw = &bars.dec_word[u][0];
        const int k0 = dw[0], k1 = dw[1];
        // entry u is read: its next tile (t + RD) may be issued
        *reinterpret_cast<volatile int*>(&bars.dec_done) = t + 1;
        if (!(k0 | k1)) continue;
        const int vs = vcount % NSV;
        if (vcount >= npre) {  // ask both producers for tile t's V
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
        // O += P_hi V + P_lo V over the pair (rows of a CTA that skipped
        // masked); tile t's P is in buffer t % NPB
        const int pb = t % NPB;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint64_t dp = dp0 + (uint64_t)(((pb * 2 + half) * P_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < T / 16; ++kk)
            mma_pair(tmem + TMEM_O, sdesc_kstep(dp, kk, QH_BYTES), dv + (uint64_t)((kk * 2048) >> 4),
                     IDESC_PV, 1u, m0, m1);
        }
        commit_pair(smem_u32(&bars.v_empty[vs]), 3);
        commit_pair(smem_u32(&bars.pv_done[pb]), (uint16_t)((k0 ? 1 : 0) | (k1 ? 2 : 0)));
        ++vcount;
      }
      // no further V requests: stop both producers (a request for key block -1)
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
    // ------------------------------------------------ softmax / test (8 warps)
    const int r = tid & (T - 1);  // row of the block = TMEM lane
    const int g = tid >> 7;       // test group (tau > 0) or column half (tau = 0)
    const int row = iX * T + r;   // row of the chunk; position off + row
    // (packed chunks: a row past the packed tensor is never written, whatever
    // the offsets say)
    const bool row_valid = mine && row < Lq && (!VARLEN || yq0 + row < p.total_q);
    const float thr = p.never_skip ? 0.f : (p.log2_tau - __log2f((float)(off + row + 1)));
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base + TMEM_O;
    auto signal = [&](int t, int keep) {  // one thread: this CTA's decision for tile t
      const int u = t % RD;
      if (leader) {
        *reinterpret_cast<volatile int*>(&bars.dec_word[u][0]) = keep;
        mbar_arrive(smem_u32(&bars.dec_full[u][0]));
      } else {
        st_async_u32(lead(&bars.dec_word[u][1]), (uint32_t)keep, lead(&bars.dec_full[u][1]));
      }
    };
    auto release = [&](int t) {  // lane 0 of each warp: this warp has read tile t's S
      const uint32_t b = smem_u32(&bars.slot_free[t % NSLOT][sg(t)]);
      if (leader)
        mbar_arrive_relaxed(b);
      else
        st_async_u32(lead(&bars.sink), 0u, mapa_rank(b, 0));
    };
    // trace row of this block: bit k of word k / 32 = key tile k kept
    const int nw = VARLEN ? p.nw : (nb + 31) >> 5;
    const size_t brow = (size_t)z * (VARLEN ? p.nbq_max : nb) + iX;
    if (tid == 0 && mine && p.keep_bits)
      for (int w = 0; w < nw; ++w) p.keep_bits[brow * nw + w] = 0u;
    // O starts at zero: every PV accumulates (a CTA's first PV may follow
    // PVs of the peer's tiles)
    if (g == 0) {
      uint32_t zero[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) zero[e] = 0u;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_st32(t_o + ch * 32, zero);
      tc_fence_before();
    }
    sync_256();  // O and the trace row zeroed before any decision leaves

    float m_ref = kNegInf, l = 0.f;
    // keep iff mraw * scale_log2 - m_ref - log2 l >= thr; cached as a raw
    // score bound, refreshed whenever (m_ref, l) change
    float bound_raw = kNegInf;

    if constexpr (!DENSE) {
      // ---- two groups, alternate tiles (group g: tiles t = g, g + 2, ...)
      KeepBitsOr kb;
      kb.init(r == 64 && mine ? p.keep_bits : nullptr, brow * nw);
      auto vote = [&](int pred) { return g == 0 ? vote_or_128<1>(pred) : vote_or_128<2>(pred); };
      auto gsync = [&]() {
        if (g == 0)
          sync_128<1>();
        else
          sync_128<2>();
      };
      // kept tiles of this group, and of the other group as of the state
      // held in (m_ref, l): the state is the latest unless the other group
      // has kept a tile since
      int k_own = 0, k_peer = 0;
      // A tile's bookkeeping is spread over three warps of the group, since
      // the group's next vote waits for its slowest warp: row 0 publishes
      // the state, row 32 sends the decision, row 64 marks the tile final
      // and keeps the trace bits.
      auto finalize = [&](int t) {  // one thread, after the group's decision for tile t
        *reinterpret_cast<volatile unsigned long long*>(&bars.fin[t % NFIN]) =
            ((unsigned long long)(uint32_t)k_own << 32) | (uint32_t)(t + 1);
      };
      const uint32_t p_hi = sbase + OFF_P, p_lo = p_hi + P_BYTES;
      for (int t = g; t < ntiles; t += 2) {
        const int u = t % NSLOT;
        // Wait for the tile's QK even when not taking part: this CTA's
        // release of the slot must not run ahead of the slot's previous use.
        mbar_wait(smem_u32(&bars.s_full[u][sg(t)]), (t / SPER) & 1, abort, 0x219);
        tc_fence_after();
        if (!part(t)) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release(t);
          if (r == 32) signal(t, 0);
          if (r == 64) finalize(t);
          continue;
        }
        // ---- this thread's S row into registers; the S buffer is free again
        uint32_t v[128];
        tmem_ld128(tmem + lane_base + u * 128, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release(t);
        const int j = ktop - t;  // key tile
        const bool diag = (j == iX + koff);
        const int lo = VARLEN ? max(0, -kpos(j)) : 0;  // columns below lo: no key
        const int hi = diag ? r : T - 1;                // columns past hi: masked
        // ---- row max of the tile (raw scores: the positive scale commutes)
        const float mraw = row_max128(v, hi, lo);
        int keep = vote(diag || (row_valid && mraw >= bound_raw));
        if (__builtin_expect(keep, 0)) {
          // Every earlier tile must be final: this group's are, and the other
          // group's are once its tile t - 1 is (it finalizes in order). If it
          // kept a tile since this group's state was current, its state is
          // the latest: load it (acquire) and test again.
          if (t > 0) {
            const unsigned long long fw = wait_word64_lo(&bars.fin[(t - 1) % NFIN], t, abort, 0x21f);
            const int kp = (int)(fw >> 32);
            if (kp != k_peer) {
              wait_acquire(&bars.kcount[g ^ 1], kp, abort, 0x220);
              m_ref = bars.x.st.m[r];
              l = bars.x.st.l[r];
              bound_raw = (thr + m_ref + __log2f(l)) / p.scale_log2;
              k_peer = kp;
            }
            // outside the branch, so that every thread of the group meets
            // the barrier even if a timed-out wait left them disagreeing
            keep = vote(diag || (row_valid && mraw >= bound_raw));
          }
          if (keep) {
            const int nk = k_own + k_peer;  // kept tiles before tile t
            const float mt = mraw * p.scale_log2;
            const float m_new = fmaxf(m_ref, mt);
            const bool need = nk > 0 && (m_new > m_ref + kRescaleLog2);
            float alpha = 1.f;
            if (nk == 0) {
              m_ref = m_new;
            } else if (need) {
              alpha = exp2f(m_ref - m_new);
              m_ref = m_new;
            }
            // the previous kept tile's PV has read P and updated O
            if (nk > 0) {
              mbar_wait(smem_u32(&bars.pv_done[0]), (nk - 1) & 1, abort, 0x21a);
              tc_fence_after();
            }
            // P = exp2(s2 - m_ref) as a bf16 pair hi + lo, 8 keys per store
            float lsum = 0.f;
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {
              float s8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) s8[e] = __uint_as_float(v[ch * 8 + e]);
              lsum += p_chunk8<true>(s8, ch * 8, hi, lo, p.scale_log2, m_ref, p_hi, p_lo, r);
            }
            if (__any_sync(0xffffffffu, need)) tmem_scale(t_o, 128, alpha);  // warp-collective
            l = l * alpha + lsum;
            bound_raw = (thr + m_ref + __log2f(l)) / p.scale_log2;
            bars.x.st.m[r] = m_ref;
            bars.x.st.l[r] = l;
            fence_proxy_async_smem();  // P visible to the tensor cores
            tc_fence_before();
            gsync();  // every row's P, O rescale and state are in place
            ++k_own;
            if (r == 0) st_release_cta(&bars.kcount[g], k_own);  // publishes the state
            if (r == 32) signal(t, 1);
            if (r == 64) finalize(t);
            kb.set(j, true);
            continue;
          }
        }
        kb.set(j, false);
        if (r == 32) signal(t, 0);
        if (r == 64) finalize(t);
      }
      kb.flush();
      sync_256();  // both groups are done: the state is the final one
      const int nk = *reinterpret_cast<volatile int*>(&bars.kcount[0]) +
                     *reinterpret_cast<volatile int*>(&bars.kcount[1]);
      if (mine && nk > 0) {
        // ---- epilogue: O = O_acc / l, LSE = (m + log2 l) ln 2 -------------
        mbar_wait(smem_u32(&bars.pv_done[0]), (nk - 1) & 1, abort, 0x21b);
        tc_fence_after();
        m_ref = bars.x.st.m[r];
        l = bars.x.st.l[r];
        const size_t orow = VARLEN ? ((size_t)(yq0 + (row_valid ? row : 0)) * p.Hq + zq) * D
                                   : ((size_t)z * p.L + (row_valid ? row : 0)) * D;
        store_o(t_o, 64 * g, 64, 1.f / l, row_valid, p.O, p.O32, orow);
        if (row_valid && g == 0) {
          const size_t li = VARLEN ? (size_t)zq * p.total_q + yq0 + row : (size_t)z * p.L + row;
          p.LSE[li] = (m_ref + __log2f(l)) * kLn2;
        }
        if (tid == 0 && p.kept_tiles) p.kept_tiles[brow] = nk;
      }
    } else {
      // ---- tau = 0: every warp reads every tile, thread t holds columns
      // 64 (t / 128) .. + 63 of its row; the halves meet through shared
      // memory (row max before P, row sum after)
      const int c0 = 64 * g;
      const uint32_t t_oh = t_o + c0;
      KeepBitsOr kb;
      kb.init(tid == 0 && mine ? p.keep_bits : nullptr, brow * nw);
      int pcnt[2] = {0, 0};  // this CTA's PVs per P buffer so far
      auto wait_pbuf = [&](int b) {
        if (pcnt[b] > 0) {
          mbar_wait(smem_u32(&bars.pv_done[b]), (pcnt[b] - 1) & 1, abort, 0x21a);
          tc_fence_after();
        }
      };
      int n_kept = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int u = t % NSLOT;
        mbar_wait(smem_u32(&bars.s_full[u][sg(t)]), (t / SPER) & 1, abort, 0x219);
        tc_fence_after();
        if (!part(t)) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release(t);
          if (tid == 0) signal(t, 0);
          continue;
        }
        float v[64];
        tmem_ld64(tmem + lane_base + u * 128 + c0, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release(t);
        const int j = ktop - t;
        const bool diag = (j == iX + koff);
        const int lo = VARLEN ? max(0, -kpos(j)) : 0;
        const int hi = diag ? r : T - 1;
        const float pmax = half_row_max(v, c0, hi, lo);
        // this instantiation runs only with tau = 0: every legal tile is
        // kept, so there is nothing to vote on
        kb.set(j, true);
        bars.x.half.max[g][r] = pmax;
        sync_256();
        const float mt = fmaxf(bars.x.half.max[0][r], bars.x.half.max[1][r]) * p.scale_log2;
        const float m_new = fmaxf(m_ref, mt);
        const bool first = (n_kept == 0);
        const bool need = !first && (m_new > m_ref + kRescaleLog2);
        float alpha = 1.f;
        if (first) {
          m_ref = m_new;
        } else if (need) {
          alpha = exp2f(m_ref - m_new);
          m_ref = m_new;
        }
        // P buffer t % NPB is free once this CTA's last PV that read it is done
        const int pb = t % NPB;
        wait_pbuf(pb);
        const uint32_t p_hi = sbase + OFF_P + pb * 2 * P_BYTES, p_lo = p_hi + P_BYTES;
        float lsum = 0.f;
        if (diag || lo > 0) {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            lsum += p_chunk8<true>(&v[ch * 8], c0 + ch * 8, hi, lo, p.scale_log2, m_ref, p_hi,
                                   p_lo, r);
        } else {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            lsum += p_chunk8<false>(&v[ch * 8], c0 + ch * 8, hi, lo, p.scale_log2, m_ref, p_hi,
                                    p_lo, r);
        }
        if (__any_sync(0xffffffffu, need)) {  // tcgen05.ld/st are warp-collective
          // every earlier PV of this CTA has updated O before it is rescaled
          if (NPB > 1) wait_pbuf(pb ^ 1);
          tmem_scale(t_oh, 64, alpha);
        }
        ++pcnt[pb];
        bars.x.half.sum[g][r] = lsum;
        fence_proxy_async_smem();  // P visible to the tensor cores
        tc_fence_before();
        sync_256();  // every row's P, O rescale and half sums are in place
        if (tid == 0) signal(t, 1);
        l = l * alpha + (bars.x.half.sum[0][r] + bars.x.half.sum[1][r]);
        ++n_kept;
      }
      kb.flush();
      if (mine && n_kept > 0) {
        for (int b = 0; b < NPB; ++b) wait_pbuf(b);
        const size_t orow = VARLEN ? ((size_t)(yq0 + (row_valid ? row : 0)) * p.Hq + zq) * D
                                   : ((size_t)z * p.L + (row_valid ? row : 0)) * D;
        store_o(t_o, c0, 64, 1.f / l, row_valid, p.O, p.O32, orow);
        if (row_valid && g == 0) {
          const size_t li = VARLEN ? (size_t)zq * p.total_q + yq0 + row : (size_t)z * p.L + row;
          p.LSE[li] = (m_ref + __log2f(l)) * kLn2;
        }
        if (tid == 0 && p.kept_tiles) p.kept_tiles[brow] = n_kept;
      }
    }
  }
  // A CTA that gave up on a wait may still have copies or MMAs in flight:
  // give them time to land before the CTA's shared memory and TMEM go.
  if (*abort) drain_in_flight();
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
