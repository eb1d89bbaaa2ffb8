// common.cuh -- shared device helpers of the MALA CUDA library (sm_100a).
//
// The library is compiled as one translation unit (mala_lib.cu includes
// every kernel header), so the device status word below exists once per GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mala {

// ---------------------------------------------------------------------------
// Device status word. A kernel that gives up on a wait ORs a code in here
// (kernels never trap); mala_check() reads and clears it.
// ---------------------------------------------------------------------------
__device__ unsigned int g_status = 0;
__device__ unsigned int g_status_where = 0;

enum : unsigned int {
  kStatusTimeout = 1u,
  kStatusLayout = 2u,  // a kernel found its dynamic shared memory misaligned
};

// Wait limit for every device-side spin: about two seconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_timeout(unsigned int where) {
  atomicOr(&g_status, kStatusTimeout);
  atomicExch(&g_status_where, where);
}
__device__ __forceinline__ void record_layout_error(unsigned int where) {
  atomicOr(&g_status, kStatusLayout);
  atomicExch(&g_status_where, where);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegInf = -__builtin_huge_valf();

// Keep-bit bookkeeping shared by the prefill kernels: row `rowblk` of the
// [nb][nw] bit matrix of slice z. Thread 0 of a CTA accumulates 32 decisions
// at a time and stores whole words, so no atomics are needed.
// The backward's offline test for one query row, as a bound on the raw
// (unscaled) score: the row keeps a tile iff its largest raw score in that
// tile is >= this value. LSE is the forward's final natural log-normalizer;
// rows past L never keep (+inf).
__device__ __forceinline__ float bwd_keep_bound_raw(const float* LSE, size_t row_off, int row,
                                                    int L, float log2_tau, float scale_log2) {
  if (row >= L) return __int_as_float(0x7f800000);
  const float c2 = LSE[row_off + row] * kLog2e + log2_tau - __log2f((float)(row + 1));
  return c2 / scale_log2;
}

struct KeepBits {
  uint32_t* row;  // nullptr when not requested
  uint32_t word;
  int cur;        // word index being accumulated, -1 = none
  __device__ __forceinline__ void init(uint32_t* bits, size_t row_off) {
    row = bits ? bits + row_off : nullptr;
    word = 0;
    cur = -1;
  }
  __device__ __forceinline__ void set(int j, bool kept) {
    if (!row) return;
    const int w = j >> 5;
    if (w != cur) {
      if (cur >= 0) row[cur] = word;
      cur = w;
      word = 0;
    }
    if (kept) word |= 1u << (j & 31);
  }
  __device__ __forceinline__ void flush() {
    if (row && cur >= 0) row[cur] = word;
    cur = -1;
  }
};

}  // namespace mala
