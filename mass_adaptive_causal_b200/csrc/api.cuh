// api.cuh -- the C ABI declared in include/mala.h: argument checks, TMA
// tensor maps, launch configuration. No device memory is allocated here;
// every buffer is the caller's.
#pragma once

#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include "aux.cuh"
#include "bwd_sm100.cuh"
#include "bwd_test_sm100.cuh"
#include "decode_sm100.cuh"
#include "fwd2_sm100.cuh"
#include "mala.h"
#include "simt_f32.cuh"

namespace mala {
namespace host {

#define MALA_CUDA_TRY(expr)                   \
  do {                                        \
    cudaError_t e_ = (expr);                  \
    if (e_ != cudaSuccess) return MALA_ERR_CUDA; \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool tau_ok(float tau) { return isfinite(tau) && tau >= 0.f; }

inline float resolve_scale(float scale, int d) {
  return scale > 0.f ? scale : 1.f / sqrtf((float)d);
}

inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda at build time).
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// bf16 tensor [Z][rows][128] seen as 3-D (x = d, y = row, z = slice), box
// 64 x box_rows x 1 with 128-byte swizzle; rows past `rows` read as zero.
inline bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t Z,
                     uint32_t box_rows = 128) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, rows, Z};
  cuuint64_t strides[2] = {128 * 2, rows * 128 * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  memset(m, 0, sizeof(*m));
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Float32 tensor [Z][rows][128] seen as 3-D (x = d, y = row, z = Z), box
// 32 x 128 x 1 (128-byte rows), 128-byte swizzle: the backward's dQ
// accumulator, target of bulk tensor reductions; rows past `rows` are not
// written.
inline bool make_map_f32_acc(CUtensorMap* m, void* base, uint64_t rows, uint64_t Z) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, rows, Z};
  cuuint64_t strides[2] = {128 * 4, rows * 128 * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  memset(m, 0, sizeof(*m));
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed bf16 tensor [tokens][heads][128] seen as 3-D (x = d, y = token,
// z = head), box 64 x box_rows x 1, 128-byte swizzle; tokens outside
// [0, tokens) read as zero.
inline bool make_map_packed(CUtensorMap* m, const void* base, uint64_t tokens, uint64_t heads,
                            uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, tokens, heads};
  cuuint64_t strides[2] = {heads * 128 * 2, 128 * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  memset(m, 0, sizeof(*m));
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

inline mala_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

// ----------------------------------------------------------------- forward
inline mala_status fwd_f32(const float* Q, const float* K, const float* V, float* O, float* LSE,
                           int Z, int L, int d, float scale, float tau, int32_t* kept,
                           uint32_t* bits, cudaStream_t s) {
  const int nb = (L + simt::T - 1) / simt::T;
  const dim3 grid(nb, Z);
  const float log_tau = tau > 0.f ? logf(tau) : 0.f;
  const int never = tau == 0.f;
#define MALA_FWD_F32(DD)                                                                      \
  {                                                                                           \
    const size_t sm = sizeof(simt::FwdSmem<DD>);                                              \
    MALA_CUDA_TRY(cudaFuncSetAttribute(simt::fwd_f32_kernel<DD>,                              \
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)); \
    simt::fwd_f32_kernel<DD><<<grid, simt::NT, sm, s>>>(Q, K, V, O, LSE, L, nb, scale,        \
                                                         log_tau, never, kept, bits);         \
  }
  if (d == 32) MALA_FWD_F32(32)
  else if (d == 64) MALA_FWD_F32(64)
  else MALA_FWD_F32(128)
#undef MALA_FWD_F32
  return launch_status();
}

template <bool VARLEN, bool DENSE>
inline mala_status launch_pair(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                               const fwd2::Params& p, int npairs, int Z, cudaStream_t s);

// Trace words per query block of a chunk: key tiles k < nbq + ceil(off / 128).
inline int varlen_trace_words(int max_q, int max_k) {
  const int nkt = (max_q + 127) / 128 + (max_k + 127) / 128;
  return (nkt + 31) / 32;
}

inline mala_status fwd_bf16(const void* Q, const void* K, const void* V, void* O, float* LSE,
                            float* O32, int B, int Hq, int Hkv, int L, float scale, float tau,
                            int32_t* kept, uint32_t* bits, cudaStream_t s) {
  const int Z = B * Hq, Zkv = B * Hkv;
  // Q and V in 128-row boxes; K in 64-row boxes (each CTA of a pair loads
  // half of every key tile)
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, L, Z) || !make_map(&mk, K, L, Zkv, 64) || !make_map(&mv, V, L, Zkv))
    return MALA_ERR_CUDA;
  fwd2::Params p;
  p.O = reinterpret_cast<__nv_bfloat16*>(O);
  p.O32 = O32;
  p.LSE = LSE;
  p.L = L;
  p.nb = (L + fwd2::T - 1) / fwd2::T;
  p.npairs = (p.nb + 1) / 2;
  p.scale_log2 = scale * kLog2e;
  p.never_skip = tau == 0.f;
  p.log2_tau = tau > 0.f ? log2f(tau) : 0.f;
  p.kept_tiles = kept;
  p.keep_bits = bits;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  // tau = 0 keeps every tile: the instantiation with two P buffers
  return p.never_skip ? launch_pair<false, true>(mq, mk, mv, p, p.npairs, Z, s)
                      : launch_pair<false, false>(mq, mk, mv, p, p.npairs, Z, s);
}

template <bool VARLEN, bool DENSE>
inline mala_status launch_pair(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                               const fwd2::Params& p, int npairs, int Z, cudaStream_t s) {
  constexpr uint32_t smem = fwd2::Plan<DENSE>::SMEM_BYTES;
  MALA_CUDA_TRY(cudaFuncSetAttribute(fwd2::fwd_pair_kernel<VARLEN, DENSE>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * npairs, Z, 1);
  cfg.blockDim = dim3(fwd2::NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  MALA_CUDA_TRY(cudaLaunchKernelEx(&cfg, fwd2::fwd_pair_kernel<VARLEN, DENSE>, mq, mk, mv, p));
  return launch_status();
}

// Chunks appended to KV caches, packed tokens (see mala_fwd_varlen).
inline mala_status fwd_varlen_bf16(const void* Q, const void* K, const void* V, void* O,
                                   float* LSE, const int32_t* cu_q, const int32_t* cu_k,
                                   int batch, int max_q, int max_k, int total_q, int total_k,
                                   int Hq, int Hkv, float scale, float tau, int32_t* kept,
                                   uint32_t* bits, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  if (!make_map_packed(&mq, Q, total_q, Hq, 128) || !make_map_packed(&mk, K, total_k, Hkv, 64) ||
      !make_map_packed(&mv, V, total_k, Hkv, 128))
    return MALA_ERR_CUDA;
  fwd2::Params p;
  memset(&p, 0, sizeof(p));
  p.O = reinterpret_cast<__nv_bfloat16*>(O);
  p.LSE = LSE;
  p.scale_log2 = scale * kLog2e;
  p.never_skip = tau == 0.f;
  p.log2_tau = tau > 0.f ? log2f(tau) : 0.f;
  p.kept_tiles = kept;
  p.keep_bits = bits;
  p.Hq = Hq;
  p.G = Hq / Hkv;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.total_q = total_q;
  p.nbq_max = (max_q + fwd2::T - 1) / fwd2::T;
  p.nw = varlen_trace_words(max_q, max_k);
  return launch_pair<true, false>(mq, mk, mv, p, (p.nbq_max + 1) / 2, batch * Hq, s);
}

// ---------------------------------------------------------------- backward
struct BwdWorkspace {
  float* D;
  float* dQacc;
  uint32_t* bits;  // per-tile keep bits of the test pass (sized for 64-row tiles)
  int* counter;    // the work pass's column counter
};
inline size_t bwd_bits_words(size_t Z, size_t L) {
  const size_t nb = (L + 63) / 64;
  return Z * nb * ((nb + 31) / 32);
}
inline size_t bwd_ws_bytes(size_t Z, size_t L, size_t d) {
  return round256(Z * L * sizeof(float)) + round256(Z * L * d * sizeof(float)) +
         round256(bwd_bits_words(Z, L) * sizeof(uint32_t)) + 256;
}
inline BwdWorkspace bwd_ws_carve(void* ws, size_t Z, size_t L, size_t d) {
  BwdWorkspace w;
  char* c = reinterpret_cast<char*>(ws);
  w.D = reinterpret_cast<float*>(c);
  c += round256(Z * L * sizeof(float));
  w.dQacc = reinterpret_cast<float*>(c);
  c += round256(Z * L * d * sizeof(float));
  w.bits = reinterpret_cast<uint32_t*>(c);
  c += round256(bwd_bits_words(Z, L) * sizeof(uint32_t));
  w.counter = reinterpret_cast<int*>(c);
  return w;
}

inline int blocks_for(size_t n, int per_block, int cap) {
  size_t b = (n + per_block - 1) / per_block;
  return (int)(b > (size_t)cap ? cap : (b == 0 ? 1 : b));
}

inline mala_status bwd_common_pre(const void* O, const float* O32, const void* dO, mala_dtype dt,
                                  BwdWorkspace w, size_t Z, int L, int d, uint32_t* bits, int nb,
                                  cudaStream_t s) {
  const size_t rows = Z * (size_t)L;
  const int blocks = blocks_for(rows, 8, 1 << 20);
  if (O32 && dt == MALA_BF16)
    aux::row_dot_mixed_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(dO),
                                                      O32, w.D, rows, d);
  else if (O32)
    aux::row_dot_kernel<float><<<blocks, 256, 0, s>>>(reinterpret_cast<const float*>(dO), O32,
                                                      w.D, rows, d);
  else if (dt == MALA_BF16)
    aux::row_dot_bf16_v8_kernel<<<blocks, 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(dO), reinterpret_cast<const __nv_bfloat16*>(O),
        w.D, rows, d);
  else
    aux::row_dot_kernel<float><<<blocks, 256, 0, s>>>(reinterpret_cast<const float*>(dO),
                                                      reinterpret_cast<const float*>(O), w.D,
                                                      rows, d);
  const size_t n4 = rows * d / 4;
  aux::zero_kernel<<<blocks_for(n4, 256, 4 * sm_count()), 256, 0, s>>>(
      reinterpret_cast<float4*>(w.dQacc), n4);
  if (bits) {
    const size_t nbits = Z * (size_t)nb * ((nb + 31) / 32);
    aux::zero_u32_kernel<<<blocks_for(nbits, 256, 4 * sm_count()), 256, 0, s>>>(bits, nbits);
  }
  return launch_status();
}

inline mala_status bwd_f32(const float* Q, const float* K, const float* V, const float* dO,
                           const float* LSE, BwdWorkspace w, float* dQ, float* dK, float* dV,
                           int Z, int L, int d, float scale, float tau, int32_t* kept,
                           uint32_t* bits, cudaStream_t s) {
  const int nb = (L + simt::T - 1) / simt::T;
  const dim3 grid(nb, Z);
  const float log_tau = tau > 0.f ? logf(tau) : 0.f;
  const int never = tau == 0.f;
#define MALA_BWD_F32(DD)                                                                      \
  {                                                                                           \
    const size_t sm = sizeof(simt::BwdSmem<DD>);                                              \
    MALA_CUDA_TRY(cudaFuncSetAttribute(simt::bwd_f32_kernel<DD>,                              \
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)); \
    simt::bwd_f32_kernel<DD><<<grid, simt::NT, sm, s>>>(Q, K, V, dO, LSE, w.D, w.dQacc, dK,   \
                                                         dV, L, nb, scale, log_tau, never,    \
                                                         kept, bits);                         \
  }
  if (d == 32) MALA_BWD_F32(32)
  else if (d == 64) MALA_BWD_F32(64)
  else MALA_BWD_F32(128)
#undef MALA_BWD_F32
  const size_t n = (size_t)Z * L * d;
  aux::convert_kernel<float><<<blocks_for(n, 256, 4 * sm_count()), 256, 0, s>>>(w.dQacc, dQ, n);
  return launch_status();
}

inline mala_status bwd_bf16(const void* Q, const void* K, const void* V, const void* dO,
                            const float* LSE, BwdWorkspace w, void* dQ,
                            void* dK, void* dV, int B, int Hq, int Hkv, int L, float scale,
                            float tau,
                            int32_t* kept, uint32_t* bits, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mdo, mk64, mdq, mdk, mdv;
  const int Z = B * Hq, Zkv = B * Hkv;
  if (!make_map(&mq, Q, L, Z) || !make_map(&mk, K, L, Zkv) || !make_map(&mv, V, L, Zkv) ||
      !make_map(&mdo, dO, L, Z) || !make_map(&mk64, K, L, Zkv, 64) ||
      !make_map_f32_acc(&mdq, w.dQacc, L, Z) || !make_map(&mdk, dK, L, Zkv) ||
      !make_map(&mdv, dV, L, Zkv))
    return MALA_ERR_CUDA;
  const int nb = (L + bwd100::T - 1) / bwd100::T;
  const int never = tau == 0.f;
  uint32_t* tile_bits = bits ? bits : w.bits;
  if (!never) {
    // pass 1: the offline test of every legal tile -> one bit per tile
    bwdtest::Params tp;
    tp.LSE = LSE;
    tp.L = L;
    tp.nb = nb;
    tp.nclus = (nb + 3) / 4;
    tp.Hq = Hq;
    tp.G = Hq / Hkv;
    tp.scale_log2 = scale * kLog2e;
    tp.log2_tau = log2f(tau);
    tp.bits = tile_bits;
    // every legal tile's scores are recomputed against the final LSE, on
    // CTA pairs of four query blocks (each CTA loads half of every key tile)
    MALA_CUDA_TRY(cudaFuncSetAttribute(bwdtest::test_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bwdtest::SMEM_BYTES));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * tp.nclus, Z, 1);
    cfg.blockDim = dim3(bwdtest::NT, 1, 1);
    cfg.dynamicSmemBytes = bwdtest::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    MALA_CUDA_TRY(cudaLaunchKernelEx(&cfg, bwdtest::test_kernel, mq, mk64, tp));
  } else if (bits) {
    const size_t nwords = (size_t)Z * nb * ((nb + 31) / 32);
    aux::lower_bits_kernel<<<blocks_for(nwords, 256, 4 * sm_count()), 256, 0, s>>>(bits, nb,
                                                                                 nwords);
  }
  // pass 2: post-score work of the kept tiles, one CTA per key block
  bwd100::Params p;
  p.LSE = LSE;
  p.Dterm = w.D;
  p.dQacc = w.dQacc;
  p.dK = reinterpret_cast<__nv_bfloat16*>(dK);
  p.dV = reinterpret_cast<__nv_bfloat16*>(dV);
  p.L = L;
  p.nb = nb;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.never_skip = never;
  p.kept_tiles = kept;
  p.bits = tile_bits;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.Zkv = Zkv;
  p.item_counter = w.counter;
  aux::zero_u32_kernel<<<1, 32, 0, s>>>(reinterpret_cast<uint32_t*>(w.counter), 1);
  MALA_CUDA_TRY(cudaFuncSetAttribute(bwd100::bwd_bf16_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)bwd100::SMEM_BYTES));
  // persistent: one CTA per SM takes (key block, key/value head) columns in
  // turn; dK_j, dV_j sum over the column's query heads
  const int ncols = p.nb * Zkv;
  const int nsm = sm_count();
  bwd100::bwd_bf16_kernel<<<ncols < nsm ? ncols : nsm, bwd100::NT, bwd100::SMEM_BYTES, s>>>(
      mq, mk, mv, mdo, mdq, mdk, mdv, p);
  const size_t n4 = (size_t)Z * L * 128 / 4;
  aux::convert_bf16_v4_kernel<<<blocks_for(n4, 256, 4 * sm_count()), 256, 0, s>>>(
      reinterpret_cast<const float4*>(w.dQacc), reinterpret_cast<uint2*>(dQ), n4);
  return launch_status();
}

// ------------------------------------------------------------------ decode
struct DecWorkspace {
  float2* stats;
  int* kept;
  int* counts;
  float* mfin;
  float* lfin;
  float* oacc;
  uint8_t* head_mask;
};
inline size_t dec_ws_bytes(size_t B, size_t Hq, size_t Hkv, size_t Lc, size_t d) {
  const size_t groups = B * Hkv;
  const size_t nt = (Lc + 127) / 128;
  return round256(B * Hq * nt * sizeof(float2)) + round256(groups * nt * sizeof(int)) +
         round256(groups * sizeof(int)) + 2 * round256(B * Hq * sizeof(float)) +
         round256(B * Hq * d * sizeof(float)) + round256(groups * nt);
}
inline DecWorkspace dec_ws_carve(void* ws, size_t B, size_t Hq, size_t Hkv, size_t Lc, size_t d) {
  const size_t groups = B * Hkv;
  const size_t nt = (Lc + 127) / 128;
  char* p = reinterpret_cast<char*>(ws);
  DecWorkspace w;
  w.stats = reinterpret_cast<float2*>(p);
  p += round256(B * Hq * nt * sizeof(float2));
  w.kept = reinterpret_cast<int*>(p);
  p += round256(groups * nt * sizeof(int));
  w.counts = reinterpret_cast<int*>(p);
  p += round256(groups * sizeof(int));
  w.mfin = reinterpret_cast<float*>(p);
  p += round256(B * Hq * sizeof(float));
  w.lfin = reinterpret_cast<float*>(p);
  p += round256(B * Hq * sizeof(float));
  w.oacc = reinterpret_cast<float*>(p);
  p += round256(B * Hq * d * sizeof(float));
  w.head_mask = reinterpret_cast<uint8_t*>(p);
  return w;
}

inline mala_status decode_bf16(const void* q, const void* Kc, const void* Vc, void* o, int B,
                               int Hq, int Hkv, int Lc, float scale, float tau, int per_head,
                               DecWorkspace w, int32_t* kept_tiles, uint32_t* bits,
                               cudaStream_t s) {
  const int G = Hq / Hkv;
  const int groups = B * Hkv;
  const int nt = (Lc + dec::T - 1) / dec::T;
  CUtensorMap mk, mv;
  if (!make_map(&mk, Kc, Lc, groups) || !make_map(&mv, Vc, Lc, groups)) return MALA_ERR_CUDA;
  const int nsm = sm_count();
  const float scale_log2 = scale * kLog2e;

  dec::StatsParams sp;
  sp.q = reinterpret_cast<const __nv_bfloat16*>(q);
  sp.stats = w.stats;
  sp.G = G;
  sp.Lc = Lc;
  sp.nt = nt;
  sp.n_groups = groups;
  sp.total_tiles = (long long)groups * nt;
  const long long ctas = sp.total_tiles < nsm ? sp.total_tiles : nsm;
  sp.tiles_per_cta = (sp.total_tiles + ctas - 1) / ctas;
  sp.scale_log2 = scale_log2;
  const int grid_a = (int)((sp.total_tiles + sp.tiles_per_cta - 1) / sp.tiles_per_cta);
  MALA_CUDA_TRY(cudaFuncSetAttribute(dec::stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)dec::STATS_RING_SMEM));
  dec::stats_kernel<<<grid_a, dec::STATS_NT, dec::STATS_RING_SMEM, s>>>(mk, sp);

  dec::ScanParams cp;
  cp.stats = w.stats;
  cp.kept = w.kept;
  cp.counts = w.counts;
  cp.mfin = w.mfin;
  cp.lfin = w.lfin;
  cp.oacc = w.oacc;
  cp.G = G;
  cp.nt = nt;
  cp.n_groups = groups;
  cp.never_skip = tau == 0.f;
  cp.thr = tau > 0.f ? log2f(tau) - log2f((float)Lc) : 0.f;
  cp.kept_tiles = kept_tiles;
  cp.keep_bits = bits;
  cp.per_head = per_head;
  cp.head_mask = w.head_mask;
  const size_t scan_smem = (size_t)G * nt * sizeof(float2);
  const int stage = scan_smem <= 200 * 1024;
  MALA_CUDA_TRY(cudaFuncSetAttribute(dec::scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     stage ? (int)scan_smem : 0));
  dec::scan_kernel<<<groups, dec::NT, stage ? scan_smem : 0, s>>>(cp, stage);

  dec::PVParams pp;
  pp.q = sp.q;
  pp.kept = w.kept;
  pp.counts = w.counts;
  pp.mfin = w.mfin;
  pp.oacc = w.oacc;
  pp.G = G;
  pp.Lc = Lc;
  pp.nt = nt;
  pp.n_groups = groups;
  pp.scale_log2 = scale_log2;
  pp.head_mask = per_head ? w.head_mask : nullptr;
  MALA_CUDA_TRY(cudaFuncSetAttribute(dec::pv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)dec::PV_SMEM));
  dec::pv_kernel<<<2 * nsm, dec::NT, dec::PV_SMEM, s>>>(mk, mv, pp);

  const size_t heads = (size_t)B * Hq;
  dec::finalize_kernel<<<(int)((heads * 128 + 255) / 256), 256, 0, s>>>(
      w.oacc, w.lfin, reinterpret_cast<__nv_bfloat16*>(o), heads);
  return launch_status();
}

}  // namespace host
}  // namespace mala

// =========================================================================
// extern "C" entry points
// =========================================================================
using namespace mala::host;

extern "C" {

const char* mala_status_string(mala_status s) {
  switch (s) {
    case MALA_OK: return "MALA_OK";
    case MALA_ERR_INVALID_ARG: return "MALA_ERR_INVALID_ARG";
    case MALA_ERR_UNSUPPORTED: return "MALA_ERR_UNSUPPORTED";
    case MALA_ERR_CUDA: return "MALA_ERR_CUDA";
    case MALA_ERR_TIMEOUT: return "MALA_ERR_TIMEOUT";
    case MALA_ERR_TOO_LARGE: return "MALA_ERR_TOO_LARGE";
  }
  return "MALA_ERR_UNKNOWN";
}

int mala_version(void) { return 100; }

static mala_status check_prefill_shape(int B, int H, int Hkv, int L, int d, mala_dtype dt,
                                       float tau, int tile) {
  if (B < 1 || H < 1 || Hkv < 1 || L < 0 || d < 1) return MALA_ERR_INVALID_ARG;
  if (H % Hkv != 0) return MALA_ERR_INVALID_ARG;
  if (dt == MALA_F32 && Hkv != H) return MALA_ERR_UNSUPPORTED;  // grouped heads: bf16 only
  if ((long long)B * H > 65535) return MALA_ERR_INVALID_ARG;
  if (!tau_ok(tau)) return MALA_ERR_INVALID_ARG;
  if (dt == MALA_BF16) {
    if (d != 128 || tile != 128) return MALA_ERR_UNSUPPORTED;
  } else if (dt == MALA_F32) {
    if ((d != 32 && d != 64 && d != 128) || tile != 64) return MALA_ERR_UNSUPPORTED;
  } else {
    return MALA_ERR_UNSUPPORTED;
  }
  return MALA_OK;
}

mala_status mala_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE,
                     float* O_f32, int B, int H, int Hkv, int L, int d, mala_dtype dt, float tau,
                     int tile, float scale, int32_t* kept_tiles, uint32_t* keep_bits,
                     void* stream) {
  mala_status st = check_prefill_shape(B, H, Hkv, L, d, dt, tau, tile);
  if (st != MALA_OK) return st;
  if (L == 0) return MALA_OK;
  if (!Q || !K || !V || !O || !LSE) return MALA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) ||
      !aligned16(O_f32))
    return MALA_ERR_INVALID_ARG;
  const int Z = B * H;
  const float sc = resolve_scale(scale, d);
  cudaStream_t s = as_stream(stream);
  if (dt == MALA_F32) {
    mala_status st = fwd_f32(reinterpret_cast<const float*>(Q), reinterpret_cast<const float*>(K),
                             reinterpret_cast<const float*>(V), reinterpret_cast<float*>(O), LSE,
                             Z, L, d, sc, tau, kept_tiles, keep_bits, s);
    if (st == MALA_OK && O_f32 && O_f32 != O)
      MALA_CUDA_TRY(cudaMemcpyAsync(O_f32, O, (size_t)Z * L * d * sizeof(float),
                                    cudaMemcpyDeviceToDevice, s));
    return st;
  }
  return fwd_bf16(Q, K, V, O, LSE, O_f32, B, H, Hkv, L, sc, tau, kept_tiles, keep_bits, s);
}

mala_status mala_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                            int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int H,
                            int Hkv, int d, float tau, int tile, float scale,
                            int32_t* kept_tiles, uint32_t* keep_bits, void* stream) {
  if (batch < 1 || H < 1 || Hkv < 1 || d < 1 || total_q < 0 || total_k < 0 ||
      max_seqlen_q < 0 || max_seqlen_k < 0)
    return MALA_ERR_INVALID_ARG;
  if (H % Hkv != 0 || !tau_ok(tau)) return MALA_ERR_INVALID_ARG;
  if (d != 128 || tile != 128) return MALA_ERR_UNSUPPORTED;
  if ((long long)batch * H > 65535) return MALA_ERR_INVALID_ARG;
  if (total_q == 0 || max_seqlen_q == 0) return MALA_OK;
  if (!Q || !K || !V || !O || !LSE || !cu_seqlens_q || !cu_seqlens_k) return MALA_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, O, LSE};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MALA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return MALA_ERR_INVALID_ARG;
  return fwd_varlen_bf16(Q, K, V, O, LSE, cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q,
                         max_seqlen_k, total_q, total_k, H, Hkv, resolve_scale(scale, d), tau,
                         kept_tiles, keep_bits, as_stream(stream));
}

int mala_varlen_trace_words(int max_seqlen_q, int max_seqlen_k) {
  if (max_seqlen_q < 0 || max_seqlen_k < 0) return 0;
  return varlen_trace_words(max_seqlen_q, max_seqlen_k);
}

size_t mala_bwd_workspace_bytes(int B, int H, int L, int d) {
  if (B < 1 || H < 1 || L < 0 || d < 1) return 0;
  return bwd_ws_bytes((size_t)B * H, (size_t)L, (size_t)d);
}

mala_status mala_bwd(const void* Q, const void* K, const void* V, const void* O,
                     const float* O_f32, const void* dO, const float* LSE, void* dQ, void* dK,
                     void* dV, void* workspace, size_t workspace_bytes, int B, int H, int Hkv,
                     int L, int d, mala_dtype dt, float tau, int tile, float scale,
                     int32_t* kept_tiles, uint32_t* keep_bits, void* stream) {
  mala_status st = check_prefill_shape(B, H, Hkv, L, d, dt, tau, tile);
  if (st != MALA_OK) return st;
  if (L == 0) return MALA_OK;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace)
    return MALA_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MALA_ERR_INVALID_ARG;
  if (!aligned16(O_f32)) return MALA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MALA_ERR_INVALID_ARG;
  if (workspace_bytes < mala_bwd_workspace_bytes(B, H, L, d)) return MALA_ERR_INVALID_ARG;
  const int Z = B * H;
  const float sc = resolve_scale(scale, d);
  cudaStream_t s = as_stream(stream);
  BwdWorkspace w = bwd_ws_carve(workspace, Z, L, d);
  const int nb = (L + tile - 1) / tile;
  st = bwd_common_pre(O, O_f32, dO, dt, w, Z, L, d, keep_bits, nb, s);
  if (st != MALA_OK) return st;
  if (dt == MALA_F32)
    return bwd_f32(reinterpret_cast<const float*>(Q), reinterpret_cast<const float*>(K),
                   reinterpret_cast<const float*>(V), reinterpret_cast<const float*>(dO), LSE, w,
                   reinterpret_cast<float*>(dQ), reinterpret_cast<float*>(dK),
                   reinterpret_cast<float*>(dV), Z, L, d, sc, tau, kept_tiles, keep_bits, s);
  return bwd_bf16(Q, K, V, dO, LSE, w, dQ, dK, dV, B, H, Hkv, L, sc, tau, kept_tiles, keep_bits,
                  s);
}

size_t mala_decode_workspace_bytes(int B, int Hq, int Hkv, int Lc, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lc < 1 || d < 1) return 0;
  return dec_ws_bytes((size_t)B, (size_t)Hq, (size_t)Hkv, (size_t)Lc, (size_t)d);
}

mala_status mala_decode(const void* q, const void* Kcache, const void* Vcache, void* o, int B,
                        int Hq, int Hkv, int Lc, int d, float tau, float scale, int per_head,
                        void* workspace, size_t workspace_bytes, int32_t* kept_tiles,
                        uint32_t* keep_bits, void* stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lc < 1 || d < 1) return MALA_ERR_INVALID_ARG;
  if (per_head != 0 && per_head != 1) return MALA_ERR_INVALID_ARG;
  if (!tau_ok(tau)) return MALA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return MALA_ERR_INVALID_ARG;
  if (d != 128 || Hq / Hkv > mala::dec::GMAX) return MALA_ERR_UNSUPPORTED;
  if ((long long)B * Hkv > 4095) return MALA_ERR_UNSUPPORTED;
  if (!q || !Kcache || !Vcache || !o || !workspace) return MALA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, Kcache, Vcache, o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MALA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MALA_ERR_INVALID_ARG;
  if (workspace_bytes < mala_decode_workspace_bytes(B, Hq, Hkv, Lc, d)) return MALA_ERR_INVALID_ARG;
  DecWorkspace w = dec_ws_carve(workspace, B, Hq, Hkv, Lc, d);
  return decode_bf16(q, Kcache, Vcache, o, B, Hq, Hkv, Lc, resolve_scale(scale, d), tau, per_head,
                     w, kept_tiles, keep_bits, as_stream(stream));
}

mala_status mala_check(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MALA_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return MALA_ERR_CUDA;
  unsigned int st = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&st, mala::g_status, sizeof(st)) != cudaSuccess) return MALA_ERR_CUDA;
  if (st != 0) {
    if (cudaMemcpyToSymbol(mala::g_status, &zero, sizeof(zero)) != cudaSuccess)
      return MALA_ERR_CUDA;
    return (st & mala::kStatusTimeout) ? MALA_ERR_TIMEOUT : MALA_ERR_CUDA;
  }
  return MALA_OK;
}

}  // extern "C"
