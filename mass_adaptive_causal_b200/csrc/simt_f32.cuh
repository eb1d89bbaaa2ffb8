// simt_f32.cuh -- float32 MALA forward / backward on the CUDA cores.
//
// tcgen05 has no float32 operand type (tf32 only), so float32 inputs are
// handled with plain FFMA: 64 x 64 tiles, 256 threads, every product read
// from padded row-major shared-memory tiles (stride D + 1 floats keeps each
// warp's accesses conflict-free). The method is the same as the bf16 tensor
// core kernels: MassAlloc Attention, agihunt.info summary (rule, forward and
// backward paragraphs), jaehun.me review "Forward: online sparse softmax" and
// "Backward: offline sparse probabilities".
#pragma once

#include "common.cuh"

namespace mala {
namespace simt {

constexpr int T = 64;
constexpr int NT = 256;

template <int D>
struct FwdSmem {
  float q[T][D + 1];
  float k[T][D + 1];
  float v[T][D + 1];
  float s[T][T + 1];
  float m[T], l[T], alpha[T];
};

template <int D>
__device__ __forceinline__ void load_tile(float (*dst)[D + 1], const float* src, int row0, int L) {
  for (int e = threadIdx.x; e < T * D; e += NT) {
    const int r = e / D, c = e % D;
    dst[r][c] = (row0 + r < L) ? src[(size_t)(row0 + r) * D + c] : 0.f;
  }
}

// One CTA per (slice z, query block i); query blocks are launched longest
// first. Thread t owns output elements e = t + NT * u of the 64 x D block.
template <int D>
__global__ void __launch_bounds__(NT) fwd_f32_kernel(const float* __restrict__ Q,
                                                     const float* __restrict__ K,
                                                     const float* __restrict__ V,
                                                     float* __restrict__ O, float* __restrict__ LSE,
                                                     int L, int nb, float scale, float log_tau,
                                                     int never_skip, int32_t* kept_tiles,
                                                     uint32_t* keep_bits) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>(smem_raw);
  constexpr int PER = T * D / NT;
  const int i = nb - 1 - blockIdx.x;
  const size_t z = blockIdx.y;
  const float* Qz = Q + z * L * D;
  const float* Kz = K + z * L * D;
  const float* Vz = V + z * L * D;
  const int tid = threadIdx.x;
  const int nw = (nb + 31) / 32;
  KeepBits kb;
  kb.init(tid == 0 ? keep_bits : nullptr, (z * nb + i) * nw);
  if (tid == 0 && keep_bits)
    for (int w = i / 32 + 1; w < nw; ++w) keep_bits[(z * nb + i) * nw + w] = 0u;

  load_tile<D>(sm.q, Qz, i * T, L);
  if (tid < T) {
    sm.m[tid] = kNegInf;
    sm.l[tid] = 0.f;
  }
  float acc[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) acc[u] = 0.f;
  int kept_count = 0;

  for (int j = i; j >= 0; --j) {
    __syncthreads();
    load_tile<D>(sm.k, Kz, j * T, L);
    __syncthreads();
    // scores of the tile; the diagonal tile masks keys after the query
    for (int e = tid; e < T * T; e += NT) {
      const int r = e / T, c = e % T;
      float a = 0.f;
#pragma unroll 8
      for (int x = 0; x < D; ++x) a = fmaf(sm.q[r][x], sm.k[c][x], a);
      const bool legal = (j < i) || (c <= r);
      sm.s[r][c] = legal ? a * scale : kNegInf;
    }
    __syncthreads();
    // per-row test: keep if (mt - m - ln l) >= ln tau - ln(r + 1)
    int want = 0;
    float mt = kNegInf;
    if (tid < T) {
      for (int c = 0; c < T; ++c) mt = fmaxf(mt, sm.s[tid][c]);
      const int row = i * T + tid;
      if (j == i || never_skip) {
        want = 1;
      } else if (row < L) {
        const float lhs = mt - sm.m[tid] - logf(sm.l[tid]);
        want = lhs >= (log_tau - logf((float)(row + 1)));
      }
    }
    const int keep = __syncthreads_or(want);
    kb.set(j, keep != 0);
    if (!keep) continue;  // skipped: V never loaded, state untouched
    ++kept_count;
    load_tile<D>(sm.v, Vz, j * T, L);
    if (tid < T) {
      const float m_old = sm.m[tid];
      const float mnew = fmaxf(m_old, mt);
      const float alpha = (m_old == kNegInf) ? 0.f : expf(m_old - mnew);
      float lsum = 0.f;
      for (int c = 0; c < T; ++c) {
        const float p = expf(sm.s[tid][c] - mnew);
        sm.s[tid][c] = p;
        lsum += p;
      }
      sm.l[tid] = sm.l[tid] * alpha + lsum;
      sm.m[tid] = mnew;
      sm.alpha[tid] = alpha;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + NT * u;
      const int r = e / D, n = e % D;
      float a = acc[u] * sm.alpha[r];
#pragma unroll 8
      for (int c = 0; c < T; ++c) a = fmaf(sm.s[r][c], sm.v[c][n], a);
      acc[u] = a;
    }
  }
  kb.flush();
  __syncthreads();
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int e = tid + NT * u;
    const int r = e / D, n = e % D;
    const int row = i * T + r;
    if (row < L) O[(z * L + row) * D + n] = acc[u] / sm.l[r];
  }
  if (tid < T) {
    const int row = i * T + tid;
    if (row < L) LSE[z * L + row] = sm.m[tid] + logf(sm.l[tid]);
  }
  if (tid == 0 && kept_tiles) kept_tiles[z * nb + i] = kept_count;
}

template <int D>
struct BwdSmem {
  float k[T][D + 1];
  float v[T][D + 1];
  float q[T][D + 1];
  float dO[T][D + 1];
  float p[T][T + 1];
  float ds[T][T + 1];
  float lse[T], dd[T];
};

// One CTA per (slice z, key block j); loops over query blocks i >= j.
// dK, dV accumulate in registers; dQ is added atomically into a float32
// workspace (converted afterwards).
template <int D>
__global__ void __launch_bounds__(NT) bwd_f32_kernel(
    const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
    const float* __restrict__ dO, const float* __restrict__ LSE, const float* __restrict__ Dterm,
    float* __restrict__ dQacc, float* __restrict__ dK, float* __restrict__ dV, int L, int nb,
    float scale, float log_tau, int never_skip, int32_t* kept_tiles, uint32_t* keep_bits) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem_raw);
  constexpr int PER = T * D / NT;
  const int j = blockIdx.x;  // key block 0 has the most query blocks: launched first
  const size_t z = blockIdx.y;
  const int tid = threadIdx.x;
  const int nw = (nb + 31) / 32;
  const float* Qz = Q + z * L * D;
  const float* dOz = dO + z * L * D;
  load_tile<D>(sm.k, K + z * L * D, j * T, L);
  load_tile<D>(sm.v, V + z * L * D, j * T, L);
  float gk[PER], gv[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) gk[u] = gv[u] = 0.f;
  int kept_count = 0;

  for (int i = j; i < nb; ++i) {
    __syncthreads();
    load_tile<D>(sm.q, Qz, i * T, L);
    if (tid < T) {
      const int row = i * T + tid;
      sm.lse[tid] = row < L ? LSE[z * L + row] : 0.f;
      sm.dd[tid] = row < L ? Dterm[z * L + row] : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < T * T; e += NT) {
      const int r = e / T, c = e % T;
      float a = 0.f;
#pragma unroll 8
      for (int x = 0; x < D; ++x) a = fmaf(sm.q[r][x], sm.k[c][x], a);
      const bool legal = (i > j) || (c <= r);
      sm.p[r][c] = legal ? a * scale : kNegInf;
    }
    __syncthreads();
    // offline test with the final normalizer: keep if max_c S - LSE >= ln tau - ln(r+1)
    int want = 0;
    if (tid < T) {
      const int row = i * T + tid;
      if (never_skip) {
        want = 1;
      } else if (row < L) {
        float mx = kNegInf;
        for (int c = 0; c < T; ++c) mx = fmaxf(mx, sm.p[tid][c]);
        want = (mx - sm.lse[tid]) >= (log_tau - logf((float)(row + 1)));
      }
    }
    const int keep = __syncthreads_or(want);
    if (tid == 0 && keep_bits) {
      uint32_t* w = keep_bits + (z * nb + i) * nw + (j >> 5);
      if (keep) atomicOr(w, 1u << (j & 31));
    }
    if (!keep) continue;
    ++kept_count;
    load_tile<D>(sm.dO, dOz, i * T, L);
    // P = exp(S - LSE) (rows beyond L contribute nothing)
    for (int e = tid; e < T * T; e += NT) {
      const int r = e / T, c = e % T;
      const bool valid = (i * T + r) < L;
      sm.p[r][c] = valid ? expf(sm.p[r][c] - sm.lse[r]) : 0.f;
    }
    __syncthreads();
    // dS = P * (dP - D), dP = dO V^T
    for (int e = tid; e < T * T; e += NT) {
      const int r = e / T, c = e % T;
      float a = 0.f;
#pragma unroll 8
      for (int x = 0; x < D; ++x) a = fmaf(sm.dO[r][x], sm.v[c][x], a);
      sm.ds[r][c] = sm.p[r][c] * (a - sm.dd[r]);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + NT * u;
      const int c = e / D, n = e % D;
      float av = gv[u], ak = 0.f;
#pragma unroll 8
      for (int r = 0; r < T; ++r) {
        av = fmaf(sm.p[r][c], sm.dO[r][n], av);
        ak = fmaf(sm.ds[r][c], sm.q[r][n], ak);
      }
      gv[u] = av;
      gk[u] += scale * ak;
    }
    // dQ_i += scale * dS K_j
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + NT * u;
      const int r = e / D, n = e % D;
      const int row = i * T + r;
      float a = 0.f;
#pragma unroll 8
      for (int c = 0; c < T; ++c) a = fmaf(sm.ds[r][c], sm.k[c][n], a);
      if (row < L) atomicAdd(&dQacc[(z * L + row) * D + n], scale * a);
    }
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int e = tid + NT * u;
    const int c = e / D, n = e % D;
    const int col = j * T + c;
    if (col < L) {
      dK[(z * L + col) * D + n] = gk[u];
      dV[(z * L + col) * D + n] = gv[u];
    }
  }
  if (tid == 0 && kept_tiles) kept_tiles[z * nb + j] = kept_count;
}

}  // namespace simt
}  // namespace mala
