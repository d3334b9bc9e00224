// noalloc.cu -- prefill entry point that needs no caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they run the
// prefill: a plugin inside a host framework that owns every device allocation
// and hands plugins no allocator, a serving loop that reserved all device
// memory up front, or a latency-critical path that must not take the implicit
// device synchronisation of cudaMalloc/cudaFree.  For them the prefill's
// scratch lives in one fixed array in this library's device image.  Every GPU
// that loads the library holds that array (LIGER_PREFILL_NOALLOC_SCRATCH_BYTES)
// until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "liger_attn.h"

namespace liger {
void set_last_error(liger_status status, const char* message);
bool prefill_uses_workspace(int B, int Hq, int Hkv, int T, int d, int w, liger_dtype dt,
                            const float* initial_state);
}

// Scratch shared by every call on a device.  In host code this name is only a
// host-side stand-in: kernels must be given the device address obtained below.
static __device__ __align__(256) unsigned char g_prefill_scratch[LIGER_PREFILL_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
// Bytes at the start of the scratch that hold the tensor-core prefill's error word,
// first timeout site and segment count.
constexpr size_t kHeaderBytes = 16;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

DriverFns driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return fns;
}

std::mutex g_setup_mutex;
struct CachedAddress {
  unsigned long long ctx_id;   // context the address belongs to (0: none cached)
  void* addr;
};
CachedAddress g_cache[kMaxDevices] = {};

liger_status cuda_fail(cudaError_t e, const char* what) {
  char buf[256];
  snprintf(buf, sizeof buf, "%s: %s", what, cudaGetErrorString(e));
  liger::set_last_error(LIGER_ERR_CUDA, buf);
  return LIGER_ERR_CUDA;
}

// Device address of the scratch array in the current device's context.  The lookup is
// done once per context: the cached address is tagged with the context's unique id, so a
// context destroyed and created again (cudaDeviceReset) gets a fresh lookup.
liger_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    liger::set_last_error(LIGER_ERR_UNSUPPORTED, "device index beyond the no-alloc entry point's table");
    return LIGER_ERR_UNSUPPORTED;
  }
  // (Before the device's first runtime call there is no current context: the id stays 0,
  // the lookup below creates the context, and the next call caches against its id.)
  unsigned long long ctx_id = 0;
  const DriverFns fns = driver_fns();
  CUcontext ctx = nullptr;
  if (fns.get_current && fns.get_id && fns.get_current(&ctx) == CUDA_SUCCESS && ctx)
    fns.get_id(ctx, &ctx_id);
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  CachedAddress& c = g_cache[dev];
  if (c.addr == nullptr || ctx_id == 0 || c.ctx_id != ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prefill_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the prefill scratch");
    if (p == nullptr) {
      liger::set_last_error(LIGER_ERR_CUDA, "cudaGetSymbolAddress returned null");
      return LIGER_ERR_CUDA;
    }
    c.addr = p;
    c.ctx_id = ctx_id;
  }
  *out = c.addr;
  return LIGER_OK;
}

}  // namespace

extern "C" liger_status liger_attn_prefill_noalloc(const void* q, const void* k, const void* v, void* out,
                                                   float* final_state, int B, int Hq, int Hkv, int T, int d,
                                                   int w, float alpha, liger_dtype dt, const float* initial_state,
                                                   const int32_t* cu_seqlens, int n_seqs, void* swa_ring_out,
                                                   int32_t* pos_out, void* stream) {
  // Only the tensor-core path uses scratch; the size limit applies to it alone.
  const bool uses_scratch = liger::prefill_uses_workspace(B, Hq, Hkv, T, d, w, dt, initial_state);
  if (uses_scratch &&
      liger_attn_prefill_workspace_size(B, Hq, Hkv, T, d, n_seqs, dt) > (size_t)LIGER_PREFILL_NOALLOC_SCRATCH_BYTES) {
    liger::set_last_error(LIGER_ERR_UNSUPPORTED,
                          "these sizes need more scratch than the no-alloc prefill holds "
                          "(LIGER_PREFILL_NOALLOC_SCRATCH_BYTES); use liger_attn_prefill with a workspace");
    return LIGER_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const liger_status st = scratch_address(&scratch);
  if (st != LIGER_OK) return st;
  if (!uses_scratch) {
    // The general kernel writes no status: clear the header so that
    // liger_attn_prefill_noalloc_status() describes this call, not an earlier one.
    const cudaError_t e = cudaMemsetAsync(scratch, 0, kHeaderBytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the scratch header");
  }
  return liger_attn_prefill(q, k, v, out, final_state, B, Hq, Hkv, T, d, w, alpha, dt, initial_state,
                            cu_seqlens, n_seqs, swa_ring_out, pos_out, scratch,
                            (size_t)LIGER_PREFILL_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" liger_status liger_attn_prefill_noalloc_status(void) {
  void* scratch = nullptr;
  const liger_status st = scratch_address(&scratch);
  if (st != LIGER_OK) return st;
  return liger_attn_prefill_status(scratch, (size_t)LIGER_PREFILL_NOALLOC_SCRATCH_BYTES);
}
