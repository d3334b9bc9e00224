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
#include <cuda_runtime.h>

#include <mutex>

#include "liger_attn.h"

namespace liger {
void set_last_error(liger_status status, const char* message);
}

// Scratch shared by every call on a device.  In host code this name is only a
// host-side stand-in: kernels must be given the device address obtained below.
static __device__ __align__(256) unsigned char g_prefill_scratch[LIGER_PREFILL_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
liger_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    liger::set_last_error(LIGER_ERR_CUDA, cudaGetErrorString(e));
    return LIGER_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    liger::set_last_error(LIGER_ERR_UNSUPPORTED, "device index beyond the no-alloc entry point's table");
    return LIGER_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prefill_scratch);
    if (e != cudaSuccess || p == nullptr) {
      liger::set_last_error(LIGER_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                             : "cudaGetSymbolAddress returned null");
      return LIGER_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LIGER_OK;
}

}  // namespace

extern "C" liger_status liger_attn_prefill_noalloc(const void* q, const void* k, const void* v, void* out,
                                                   float* final_state, int B, int Hq, int Hkv, int T, int d,
                                                   int w, float alpha, liger_dtype dt, const float* initial_state,
                                                   const int32_t* cu_seqlens, int n_seqs, void* swa_ring_out,
                                                   int32_t* pos_out, void* stream) {
  const size_t need = liger_attn_prefill_workspace_size(B, Hq, Hkv, T, d, n_seqs, dt);
  if (need > (size_t)LIGER_PREFILL_NOALLOC_SCRATCH_BYTES) {
    liger::set_last_error(LIGER_ERR_UNSUPPORTED,
                          "these sizes need more scratch than the no-alloc prefill holds "
                          "(LIGER_PREFILL_NOALLOC_SCRATCH_BYTES); use liger_attn_prefill with a workspace");
    return LIGER_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const liger_status st = scratch_address(&scratch);
  if (st != LIGER_OK) return st;
  return liger_attn_prefill(q, k, v, out, final_state, B, Hq, Hkv, T, d, w, alpha, dt, initial_state,
                            cu_seqlens, n_seqs, swa_ring_out, pos_out, scratch,
                            (size_t)LIGER_PREFILL_NOALLOC_SCRATCH_BYTES, stream);
}
