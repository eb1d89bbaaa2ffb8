// aux.cuh -- small bandwidth-bound kernels around the backward pass:
// the row terms D_r = <dO_r, O_r> (the "standard attention state" the
// backward uses next to the forward's log-normalizer; agihunt.info summary,
// backward paragraph) and the conversion of the float32 dQ accumulator.
#pragma once

#include "common.cuh"

namespace mala {
namespace aux {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float& d, float x) { d = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16& d, float x) { d = __float2bfloat16_rn(x); }

// One warp per row: D[row] = sum_c dO[row][c] * O[row][c] (float32 sum).
template <typename TIn>
__global__ void row_dot_kernel(const TIn* __restrict__ dO, const TIn* __restrict__ O,
                               float* __restrict__ D, size_t rows, int d) {
  const size_t warp = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const TIn* a = dO + warp * d;
  const TIn* b = O + warp * d;
  float s = 0.f;
  for (int c = lane; c < d; c += 32) s = fmaf(to_f(a[c]), to_f(b[c]), s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) D[warp] = s;
}

// Vectorised bf16 variant for d % 8 == 0: 16-byte loads, one warp per row.
__global__ void row_dot_bf16_v8_kernel(const __nv_bfloat16* __restrict__ dO,
                                       const __nv_bfloat16* __restrict__ O, float* __restrict__ D,
                                       size_t rows, int d) {
  const size_t warp = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const uint4* a = reinterpret_cast<const uint4*>(dO + warp * d);
  const uint4* b = reinterpret_cast<const uint4*>(O + warp * d);
  float s = 0.f;
  for (int c = lane; c < d / 8; c += 32) {
    const uint4 x = a[c], y = b[c];
    const __nv_bfloat162* xa = reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162* ya = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fx = __bfloat1622float2(xa[e]), fy = __bfloat1622float2(ya[e]);
      s = fmaf(fx.x, fy.x, s);
      s = fmaf(fx.y, fy.y, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) D[warp] = s;
}

// D from the float32 output and a bf16 dO (one warp per row, d % 4 == 0).
__global__ void row_dot_mixed_kernel(const __nv_bfloat16* __restrict__ dO,
                                     const float* __restrict__ O32, float* __restrict__ D,
                                     size_t rows, int d) {
  const size_t warp = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const uint2* a = reinterpret_cast<const uint2*>(dO + warp * d);
  const float4* b = reinterpret_cast<const float4*>(O32 + warp * d);
  float s = 0.f;
  for (int c = lane; c < d / 4; c += 32) {
    const uint2 x = a[c];
    const float4 y = b[c];
    const float2 x0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.x));
    const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.y));
    s = fmaf(x0.x, y.x, s);
    s = fmaf(x0.y, y.y, s);
    s = fmaf(x1.x, y.z, s);
    s = fmaf(x1.y, y.w, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) D[warp] = s;
}

template <typename TOut>
__global__ void convert_kernel(const float* __restrict__ src, TOut* __restrict__ dst, size_t n) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x)
    from_f(dst[e], src[e]);
}

__global__ void convert_bf16_v4_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                       size_t n4) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4;
       e += (size_t)gridDim.x * blockDim.x) {
    const float4 v = src[e];
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&lo);
    o.y = *reinterpret_cast<uint32_t*>(&hi);
    dst[e] = o;
  }
}

__global__ void zero_kernel(float4* __restrict__ p, size_t n4) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n4;
       e += (size_t)gridDim.x * blockDim.x)
    p[e] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Keep bits when every legal tile is kept: row i has bits j = 0..i set.
__global__ void lower_bits_kernel(uint32_t* __restrict__ bits, int nb, size_t nwords) {
  const int nw = (nb + 31) / 32;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < nwords;
       e += (size_t)gridDim.x * blockDim.x) {
    const int w = (int)(e % nw);
    const int i = (int)((e / nw) % nb);
    const int lo = w * 32;
    uint32_t v = 0u;
    if (i >= lo + 31) v = 0xffffffffu;
    else if (i >= lo) v = (uint32_t)((1ull << (i - lo + 1)) - 1ull);
    bits[e] = v;
  }
}

__global__ void zero_u32_kernel(uint32_t* __restrict__ p, size_t n) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x)
    p[e] = 0u;
}

}  // namespace aux
}  // namespace mala
