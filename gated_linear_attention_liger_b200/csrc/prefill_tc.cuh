// prefill_tc.cuh -- bf16 chunked prefill on the tcgen05 tensor cores (sm_100a).
#pragma once

#include "liger_attn.h"
#include "common.cuh"

namespace liger {
namespace tc {

struct PrefillProblem {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* final_state;
  const int32_t* cu;
  int B, Hq, Hkv;
  long T;
  int d, n_seqs;
  float alpha;
};

inline bool supports(int d) { (void)d; return false; }
inline size_t workspace_bytes(int, int, int, long, int, int) { return 0; }
inline const char* last_message() { return "tensor-core prefill not built"; }
inline liger_status run_prefill(const PrefillProblem&, void*, cudaStream_t) { return LIGER_ERR_UNSUPPORTED; }

}  // namespace tc
}  // namespace liger
