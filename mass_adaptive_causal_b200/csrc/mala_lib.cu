// mala_lib.cu -- the whole CUDA library as one translation unit, so that the
// device status word (common.cuh) exists once per GPU and every kernel can
// set it without relocatable device code.
#include "api.cuh"

// -------------------------------------------------------------------------
// mala_decode_noalloc: the decode step with its workspace in a static device
// array, for callers that cannot allocate device memory (their host program
// owns all of it). The array is part of this library's module, so every GPU
// that loads the library holds MALA_DECODE_NOALLOC_SCRATCH_BYTES until exit.
// -------------------------------------------------------------------------
#include <mutex>

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[MALA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
// Per device: the array's device address and the unique ID of the context it
// belongs to. A context destroyed and created again (cudaDeviceReset, or a
// driver-API user replacing the current context) gets a new ID, so an address
// from an earlier context is never reused.
struct ScratchSlot {
  unsigned long long ctx_id;
  unsigned char* ptr;
};
ScratchSlot g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(ptr);
}

// The unique ID of the context current on this thread (0 if none yet).
bool current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  return !ctx || get_id(ctx, id) == CUDA_SUCCESS;
}

// In host code `g_decode_scratch` only names the array; its address on the
// current device comes from the runtime, once per device and context, and is
// cached.
mala_status scratch_on_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MALA_ERR_CUDA;
  unsigned long long id = 0;
  if (!current_context_id(&id)) return MALA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot& slot = g_scratch[dev];
  if (id == 0 || slot.ptr == nullptr || slot.ctx_id != id) {
    // the lookup makes the device's primary context current when none is
    unsigned char* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_decode_scratch) != cudaSuccess || !ptr)
      return MALA_ERR_CUDA;
    if (id == 0 && (!current_context_id(&id) || id == 0)) return MALA_ERR_CUDA;
    slot.ptr = ptr;
    slot.ctx_id = id;
  }
  *out = slot.ptr;
  return MALA_OK;
}

}  // namespace

extern "C" mala_status mala_decode_noalloc(const void* q, const void* Kcache, const void* Vcache,
                                           void* o, int B, int Hq, int Hkv, int Lc, int d,
                                           float tau, float scale, int32_t* kept_tiles,
                                           uint32_t* keep_bits, void* stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lc < 1 || d < 1) return MALA_ERR_INVALID_ARG;
  if (!tau_ok(tau)) return MALA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return MALA_ERR_INVALID_ARG;
  if (d != 128 || Hq / Hkv > mala::dec::GMAX) return MALA_ERR_UNSUPPORTED;
  if ((long long)B * Hkv > 4095) return MALA_ERR_UNSUPPORTED;
  if (!q || !Kcache || !Vcache || !o) return MALA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, Kcache, Vcache, o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MALA_ERR_INVALID_ARG;
  if (mala_decode_workspace_bytes(B, Hq, Hkv, Lc, d) > MALA_DECODE_NOALLOC_SCRATCH_BYTES)
    return MALA_ERR_TOO_LARGE;
  unsigned char* scratch = nullptr;
  const mala_status st = scratch_on_current_device(&scratch);
  if (st != MALA_OK) return st;
  // Every region is written before it is read within the call; the scan
  // kernel zeroes the float32 output accumulator, the one region that must
  // start at zero.
  DecWorkspace w = dec_ws_carve(scratch, B, Hq, Hkv, Lc, d);
  return decode_bf16(q, Kcache, Vcache, o, B, Hq, Hkv, Lc, resolve_scale(scale, d), tau, 0, w,
                     kept_tiles, keep_bits, as_stream(stream));
}

// -------------------------------------------------------------------------
// mala_selftest_wait: a wait that runs out on purpose, through the same
// bounded mbarrier wait as every kernel, so that the status path
// (record_timeout -> mala_check) can be tested without a fault.
// -------------------------------------------------------------------------
namespace {

__global__ void selftest_wait_kernel() {
  using namespace mala::sm100;
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // phase 0 never completes: nothing arrives on `bar`
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort, 0x7f0);
}

}  // namespace

extern "C" mala_status mala_selftest_wait(void* stream) {
  selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>();
  return launch_status();
}
