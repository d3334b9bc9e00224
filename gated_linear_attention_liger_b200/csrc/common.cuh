// common.cuh -- small device helpers shared by the Liger Attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace liger {

// Diagnostic options, read from the environment once, when the library is
// loaded (later changes to the environment have no effect):
//   LIGER_PREFILL_PATH=general   every prefill takes the general (CUDA-core) kernel
//   LIGER_WAIT_LIMIT_NS=<n>      give-up time of each bounded wait in the
//                                tensor-core prefill (default 2 s)
//   LIGER_TEST_INJECT_STALL=<n>  the first n tensor-core prefill calls of the
//                                process withhold one MMA completion, so that a
//                                bounded wait runs out (exercises failure
//                                detection without a fault); later calls run
//                                normally
struct Options {
  bool force_general_prefill;
  unsigned long long wait_limit_ns;   // 0: the kernel's default
  long inject_stall_calls;
};
const Options& options();
// True for the first options().inject_stall_calls calls (thread-safe).
bool take_injected_stall();

// Storage type <-> fp32.
template <typename T> struct io;
template <> struct io<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float x) { *p = x; }
};
template <> struct io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// log sigmoid(m) without overflow on either side: -softplus(-m).
__device__ __forceinline__ float log_sigmoid(float m) {
  return m >= 0.f ? -log1pf(expf(-m)) : m - log1pf(expf(m));
}

// Sequence [begin, end) on the packed token axis.  With offsets, they are
// clamped into [0, T_total] and made non-decreasing so that every access stays
// in bounds even for malformed offsets.
__device__ __forceinline__ void seq_range(const int32_t* cu, int seq, long T, long T_total,
                                          long* begin, long* end) {
  if (cu) {
    long b = cu[seq], e = cu[seq + 1];
    b = b < 0 ? 0 : (b > T_total ? T_total : b);
    e = e < b ? b : (e > T_total ? T_total : e);
    *begin = b;
    *end = e;
  } else {
    *begin = (long)seq * T;
    *end = *begin + T;
  }
}

}  // namespace liger
