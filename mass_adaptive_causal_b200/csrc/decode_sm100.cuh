// decode_sm100.cuh -- one MALA decode step over a bf16 KV cache (d = 128).
//
// The pages use one rule for prefill and decode and keep the cache whole
// (MassAlloc Attention; agihunt.info summary, rule and limits paragraphs).
// For one new token per sequence, the cache of (b, kv head g) is cut into
// 128-key tiles aligned from position 0 and visited newest first; the rows of
// a tile are the G query heads sharing g; the newest tile is always kept and
// a later tile is skipped iff every head has  mt - m - ln l < ln tau - ln Lc.
//
// The sequential rule is split so that the HBM stream is parallel:
//  A  stats:  every CTA streams a contiguous run of K tiles (TMA ring, no
//             multicast) and computes, per tile and head, the row max m_t and
//             l_t = sum exp(s - m_t) (mma.sync m16n8k16: 16 keys x 8 heads).
//             This pass reads all of K once: it is the HBM-bound part.
//  B  scan:   one CTA per (b, g) replays the exact online test on (m_t, l_t)
//             newest first -- a kept tile's update needs only those two
//             numbers per head -- a warp testing 32 tiles per step against the
//             current state; emits the kept-tile list and the final (m, l).
//  C  values: kept tiles only: re-read K and V, p = exp(s - m_final),
//             o += p V (float32 atomics), then o / l -> bf16.
// Everything is in the log2 domain (s2 = s * scale * log2 e).
#pragma once

#include "sm100.cuh"

namespace mala {
namespace dec {

using namespace sm100;

constexpr int T = 128;
constexpr int D = 128;
constexpr int NT = 128;  // 4 warps x 32 keys
constexpr int GMAX = 8;  // heads per KV group (the mma N dimension)
constexpr uint32_t TILE_BYTES = T * D * 2;
constexpr uint32_t HALF_BYTES = T * 64 * 2;
constexpr uint32_t PV_SMEM = 2 * TILE_BYTES + 1024 + GMAX * T * 4 + 4096 * 4 + 256;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& a0, uint32_t& a1, uint32_t& a2,
                                        uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// B fragments of the group's query heads: B[k][n] = q[head n][d = 16 ks + k].
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16* q, int grp, int G,
                                             uint32_t (&bq)[8][2]) {
  const int lane = threadIdx.x & 31;
  const int n = lane >> 2;
  const int kq = (lane & 3) * 2;
  const __nv_bfloat16* qh = q + ((size_t)grp * G + n) * D;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    if (n < G) {
      bq[ks][0] = *reinterpret_cast<const uint32_t*>(qh + ks * 16 + kq);
      bq[ks][1] = *reinterpret_cast<const uint32_t*>(qh + ks * 16 + kq + 8);
    } else {
      bq[ks][0] = bq[ks][1] = 0u;
    }
  }
}

// Scores of this warp's 32 keys against the group's heads:
// acc[mb][0..3] = S[key 32w + 16mb + lane/4 (+8)][head 2(lane%4) (+1)].
__device__ __forceinline__ void warp_scores(uint32_t tile, const uint32_t (&bq)[8][2],
                                            float (&acc)[2][4]) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[mb][e] = 0.f;
  // two independent accumulation chains (mb = 0, 1) interleaved over ks
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int mb = 0; mb < 2; ++mb) {
      const int r = warp * 32 + mb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int c = ks * 16 + (lane >> 4) * 8;
      uint32_t a0, a1, a2, a3;
      ldsm_x4(tile + sw128_chunk_off(r, c, T), a0, a1, a2, a3);
      mma16816(acc[mb], a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
    }
  }
}

struct StatsParams {
  const __nv_bfloat16* q;
  float2* stats;  // [n_groups][G][nt] (m2_t, l_t)
  int G, Lc, nt, n_groups;
  long long total_tiles;
  long long tiles_per_cta;
  float scale_log2;
};

// One consumer warp per ring stage: warp w reads stage w only (tiles w,
// w + 6, ...), so it never waits on a stage more than one phase ahead.
constexpr int STATS_NST = 6;                          // TMA ring depth
constexpr int STATS_CONSUMERS = STATS_NST;            // warps, one whole tile each
constexpr int STATS_NT = 32 * (STATS_CONSUMERS + 1);  // + one TMA producer warp
constexpr uint32_t STATS_RING_SMEM = STATS_NST * TILE_BYTES + 1024 + 256;

// Phase A: one CTA per SM streams a contiguous run of tiles. The last warp
// keeps a 6-stage TMA ring full; consumer warp w handles tiles w, w+6, ... of
// the run entirely by itself (8 m16 blocks x 8 k-steps of mma.sync against
// the group's query heads), so no CTA-wide barrier sits on the stream.
__global__ void __launch_bounds__(STATS_NT) stats_kernel(const __grid_constant__ CUtensorMap tmK,
                                                         const StatsParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring = smem_u32(base);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + STATS_NST * TILE_BYTES);
  uint64_t* empty = full + STATS_NST;
  volatile int* abort = reinterpret_cast<volatile int*>(empty + STATS_NST);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const long long begin = (long long)blockIdx.x * p.tiles_per_cta;
  long long end = begin + p.tiles_per_cta;
  if (end > p.total_tiles) end = p.total_tiles;
  if (begin >= end) return;
  const int count = (int)(end - begin);

  if (tid == 0) {
    for (int s = 0; s < STATS_NST; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == STATS_CONSUMERS) {
    if (lane == 0) {
      for (int k = 0; k < count; ++k) {
        const int s = k % STATS_NST;
        if (k >= STATS_NST)
          mbar_wait(smem_u32(&empty[s]), ((k / STATS_NST) - 1) & 1, abort, 0x300);
        const long long flat = begin + k;
        const int grp = (int)(flat / p.nt), t = (int)(flat % p.nt);
        const uint32_t bar = smem_u32(&full[s]);
        mbar_expect_tx(bar, TILE_BYTES);
        tma_load_3d(ring + s * TILE_BYTES, &tmK, 0, t * T, grp, bar);
        tma_load_3d(ring + s * TILE_BYTES + HALF_BYTES, &tmK, 64, t * T, grp, bar);
      }
    }
    return;
  }

  uint32_t bq[8][2];
  int cur_grp = -1;
  const int n0 = (lane & 3) * 2;
  for (int k = warp; k < count; k += STATS_CONSUMERS) {
    const long long flat = begin + k;
    const int grp = (int)(flat / p.nt), t = (int)(flat % p.nt);
    if (grp != cur_grp) {
      load_q_frags(p.q, grp, p.G, bq);
      cur_grp = grp;
    }
    const int s = k % STATS_NST;
    mbar_wait(smem_u32(&full[s]), (k / STATS_NST) & 1, abort, 0x301);
    const uint32_t tile = ring + s * TILE_BYTES;
    // S[key][head] for all 128 keys: 8 m16 blocks, two blocks per chain
    float acc[8][4];
#pragma unroll
    for (int mb = 0; mb < 8; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mb][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int mb = 0; mb < 8; ++mb) {
        const int r = mb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = ks * 16 + (lane >> 4) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(tile + sw128_chunk_off(r, c, T), a0, a1, a2, a3);
        mma16816(acc[mb], a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[s]));  // scores are in registers
    float mx0 = kNegInf, mx1 = kNegInf;
#pragma unroll
    for (int mb = 0; mb < 8; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = t * T + mb * 16 + (lane >> 2) + (e >> 1) * 8;
        const float v = key < p.Lc ? acc[mb][e] * p.scale_log2 : kNegInf;
        acc[mb][e] = v;
        if (e & 1) mx1 = fmaxf(mx1, v); else mx0 = fmaxf(mx0, v);
      }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int mb = 0; mb < 8; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (e & 1) s1 += exp2f(acc[mb][e] - mx1); else s0 += exp2f(acc[mb][e] - mx0);
      }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, o);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if (lane < 4) {
      if (n0 < p.G) p.stats[((size_t)grp * p.G + n0) * p.nt + t] = make_float2(mx0, s0);
      if (n0 + 1 < p.G) p.stats[((size_t)grp * p.G + n0 + 1) * p.nt + t] = make_float2(mx1, s1);
    }
  }
}

struct ScanParams {
  const float2* stats;
  int* kept;       // [n_groups][nt] kept tile indices, newest first
  int* counts;     // [n_groups]
  float* mfin;     // [n_groups][G] final running max (log2 units)
  float* lfin;     // [n_groups][G] final retained mass
  float* oacc;     // [n_groups][G][D] zeroed here
  int G, nt, n_groups;
  float thr;       // log2(tau) - log2(Lc)
  int never_skip;
  int32_t* kept_tiles;   // [n_groups] (per_head: [n_groups][G])
  uint32_t* keep_bits;   // [n_groups][nw] (per_head: [n_groups][G][nw])
  // per_head: every query head decides alone (its own ratio test); the list
  // holds the tiles any head kept, head_mask[list entry] which heads did
  int per_head;
  uint8_t* head_mask;    // [n_groups][nt]
};

// Per-head rows: head h keeps tile t iff  m_t,h - m_h - log2 l_h >= thr  with
// its own running (m_h, l_h); the newest tile is every head's first. Warp 0
// looks 32 tiles ahead: lane k tests tile next - k for every head; the first
// tile some head wants is taken by exactly the heads that want it (no head's
// state changed on the tiles before it, so their tests there stand).
__device__ __forceinline__ void scan_per_head(const ScanParams& p, const float2* st, int grp) {
  const int lane = threadIdx.x & 31;
  const int G = p.G, nt = p.nt, nw = (nt + 31) >> 5;
  float m[GMAX], l[GMAX];
  int cnt[GMAX];
  int count = 0;
  int* kept = p.kept + (size_t)grp * nt;
  uint8_t* mask = p.head_mask + (size_t)grp * nt;
  uint32_t* bits = p.keep_bits ? p.keep_bits + (size_t)grp * G * nw : nullptr;
  auto take = [&](int t, uint32_t hm) {
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G && ((hm >> h) & 1u)) {
        const float2 s = st[h * nt + t];
        if (cnt[h] == 0) {
          m[h] = s.x;
          l[h] = s.y;
        } else {
          const float mn = fmaxf(m[h], s.x);
          l[h] = l[h] * exp2f(m[h] - mn) + s.y * exp2f(s.x - mn);
          m[h] = mn;
        }
        ++cnt[h];
        if (bits && lane == 0) bits[(size_t)h * nw + (t >> 5)] |= 1u << (t & 31);
      }
    }
    if (lane == 0) {
      kept[count] = t;
      mask[count] = (uint8_t)hm;
    }
    ++count;
  };
#pragma unroll
  for (int h = 0; h < GMAX; ++h) cnt[h] = 0;
  take(nt - 1, (1u << G) - 1u);
  int next = nt - 2;
  while (next >= 0) {
    const int tt = next - lane;
    uint32_t want = 0;
    if (tt >= 0) {
#pragma unroll
      for (int h = 0; h < GMAX; ++h)
        if (h < G && (p.never_skip || (st[h * nt + tt].x - m[h] - __log2f(l[h])) >= p.thr))
          want |= 1u << h;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, want != 0u);
    if (bal == 0u) {
      next -= 32;
      continue;
    }
    const int src = __ffs(bal) - 1;
    const uint32_t hm = __shfl_sync(0xffffffffu, want, src);
    take(next - src, hm);
    __syncwarp();
    next = next - src - 1;
  }
  if (lane == 0) p.counts[grp] = count;
#pragma unroll
  for (int h = 0; h < GMAX; ++h)
    if (h < G && lane == h) {
      p.mfin[(size_t)grp * G + h] = m[h];
      p.lfin[(size_t)grp * G + h] = l[h];
      if (p.kept_tiles) p.kept_tiles[(size_t)grp * G + h] = cnt[h];
    }
}

// One CTA (128 threads) per group: stage the group's stats in shared memory
// (when they fit; otherwise they are read from global memory), then warp 0
// replays the online test.
__global__ void __launch_bounds__(NT) scan_kernel(const ScanParams p, int stage_in_smem) {
  extern __shared__ float2 st_smem[];  // [G][nt]
  const int grp = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int G = p.G, nt = p.nt;
  const float2* src = p.stats + (size_t)grp * G * nt;
  const float2* st = src;
  if (stage_in_smem) {
    for (int e = tid; e < G * nt; e += NT) st_smem[e] = src[e];
    st = st_smem;
  }
  float* oz = p.oacc + (size_t)grp * G * D;
  for (int e = tid; e < G * D; e += NT) oz[e] = 0.f;
  const int nw = (nt + 31) >> 5;
  const int nbits = p.per_head ? G * nw : nw;
  if (p.keep_bits)
    for (int e = tid; e < nbits; e += NT) p.keep_bits[(size_t)grp * nbits + e] = 0u;
  __syncthreads();
  if (tid >= 32) return;
  if (p.per_head) {
    scan_per_head(p, st, grp);
    return;
  }

  float m[GMAX], l[GMAX];
  int count = 0;
  int* kept = p.kept + (size_t)grp * nt;
  uint32_t* bits = p.keep_bits ? p.keep_bits + (size_t)grp * nw : nullptr;
  auto take = [&](int t) {
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        const float2 s = st[h * nt + t];
        if (count == 0) {
          m[h] = s.x;
          l[h] = s.y;
        } else {
          const float mn = fmaxf(m[h], s.x);
          l[h] = l[h] * exp2f(m[h] - mn) + s.y * exp2f(s.x - mn);
          m[h] = mn;
        }
      }
    }
    if (lane == 0) {
      kept[count] = t;
      if (bits) bits[t >> 5] |= 1u << (t & 31);
    }
    ++count;
  };
  take(nt - 1);  // the newest tile is always kept
  int next = nt - 2;
  while (next >= 0) {
    const int tt = next - lane;
    int want = 0;
    if (tt >= 0) {
      if (p.never_skip) {
        want = 1;
      } else {
#pragma unroll
        for (int h = 0; h < GMAX; ++h)
          if (h < G) want |= (st[h * nt + tt].x - m[h] - __log2f(l[h])) >= p.thr;
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, want);
    if (bal == 0u) {
      next -= 32;
      continue;
    }
    const int t = next - (__ffs(bal) - 1);
    take(t);
    __syncwarp();
    next = t - 1;
  }
  if (lane == 0) {
    p.counts[grp] = count;
    if (p.kept_tiles) p.kept_tiles[grp] = count;
  }
#pragma unroll
  for (int h = 0; h < GMAX; ++h)
    if (h < G && lane == h) {
      p.mfin[(size_t)grp * G + h] = m[h];
      p.lfin[(size_t)grp * G + h] = l[h];
    }
}

struct PVParams {
  const __nv_bfloat16* q;
  const int* kept;
  const int* counts;
  const float* mfin;
  float* oacc;
  int G, Lc, nt, n_groups;
  float scale_log2;
  const uint8_t* head_mask;  // per-head rows: heads that kept each list entry (else null)
};

// Persistent CTAs over the flattened list of kept tiles of all groups.
__global__ void __launch_bounds__(NT) pv_kernel(const __grid_constant__ CUtensorMap tmK,
                                                const __grid_constant__ CUtensorMap tmV,
                                                const PVParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ka = smem_u32(base);
  const uint32_t va = ka + TILE_BYTES;
  const unsigned char* vbytes = base + TILE_BYTES;
  float* ps = reinterpret_cast<float*>(base + 2 * TILE_BYTES);  // [GMAX][T]
  int* prefix = reinterpret_cast<int*>(ps + GMAX * T);          // [n_groups + 1] (<= 4096)
  uint64_t* bar = reinterpret_cast<uint64_t*>(prefix + 4096);
  volatile int* abort = reinterpret_cast<volatile int*>(bar + 1);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;

  if (tid == 0) {
    mbar_init(smem_u32(bar), 1);
    *abort = 0;
    fence_mbar_init();
    int acc = 0;
    for (int g = 0; g < p.n_groups; ++g) {
      prefix[g] = acc;
      acc += p.counts[g];
    }
    prefix[p.n_groups] = acc;
  }
  __syncthreads();
  const int total = prefix[p.n_groups];
  uint32_t bq[8][2];
  int cur_grp = -1;
  uint32_t phase = 0;
  const int n0 = (lane & 3) * 2;
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    int lo = 0, hi = p.n_groups;  // largest g with prefix[g] <= item
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= item) lo = mid; else hi = mid;
    }
    const int grp = lo;
    const int t = p.kept[(size_t)grp * p.nt + (item - prefix[grp])];
    const uint32_t hm = p.head_mask ? p.head_mask[(size_t)grp * p.nt + (item - prefix[grp])] : 0xffu;
    if (tid == 0) {
      const uint32_t b = smem_u32(bar);
      mbar_expect_tx(b, 2 * TILE_BYTES);
      tma_load_3d(ka, &tmK, 0, t * T, grp, b);
      tma_load_3d(ka + HALF_BYTES, &tmK, 64, t * T, grp, b);
      tma_load_3d(va, &tmV, 0, t * T, grp, b);
      tma_load_3d(va + HALF_BYTES, &tmV, 64, t * T, grp, b);
    }
    if (grp != cur_grp) {
      load_q_frags(p.q, grp, G, bq);
      cur_grp = grp;
    }
    const bool ok = mbar_wait(smem_u32(bar), phase, abort, 0x302);
    phase ^= 1;
    if (__syncthreads_or(!ok)) break;
    float acc[2][4];
    warp_scores(ka, bq, acc);
    const float mf0 = (n0 < G) ? p.mfin[(size_t)grp * G + n0] : 0.f;
    const float mf1 = (n0 + 1 < G) ? p.mfin[(size_t)grp * G + n0 + 1] : 0.f;
#pragma unroll
    for (int mb = 0; mb < 2; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kl = warp * 32 + mb * 16 + (lane >> 2) + (e >> 1) * 8;
        const int n = n0 + (e & 1);
        if (n < G) {
          const bool valid = t * T + kl < p.Lc && ((hm >> n) & 1u);
          ps[n * T + kl] =
              valid ? exp2f(acc[mb][e] * p.scale_log2 - ((e & 1) ? mf1 : mf0)) : 0.f;
        }
      }
    __syncthreads();
    // o[h][n] += sum_key p[h][key] V[key][n], thread = column n
    float o[GMAX];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) o[h] = 0.f;
    for (int key = 0; key < T; ++key) {
      const uint32_t off = sw128_chunk_off(key, tid, T) + (tid & 7) * 2;
      const float v = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vbytes + off));
#pragma unroll
      for (int h = 0; h < GMAX; ++h)
        if (h < G) o[h] = fmaf(ps[h * T + key], v, o[h]);
    }
#pragma unroll
    for (int h = 0; h < GMAX; ++h)
      if (h < G) atomicAdd(&p.oacc[((size_t)grp * G + h) * D + tid], o[h]);
    __syncthreads();  // K, V, ps free for the next item
  }
}

// o = oacc / l -> bf16, one thread per element.
__global__ void finalize_kernel(const float* __restrict__ oacc, const float* __restrict__ lfin,
                                __nv_bfloat16* __restrict__ o, size_t heads) {
  const size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (e >= heads * D) return;
  o[e] = __float2bfloat16_rn(oacc[e] / lfin[e / D]);
}

}  // namespace dec
}  // namespace mala
