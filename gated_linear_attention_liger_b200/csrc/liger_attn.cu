// liger_attn.cu -- the C ABI (include/liger_attn.h): argument checks, path
// selection and kernel launches on the caller's stream.  No allocation, no
// host synchronisation.
#include "liger_attn.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <utility>

#include "common.cuh"
#include "decode.cuh"
#include "full_attn.cuh"
#include "prefill_bwd.cuh"
#include "prefill_seg.cuh"
#include "prefill_simt.cuh"
#include "prefill_tc.cuh"

namespace {

thread_local std::string g_last_error;
thread_local cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;
thread_local uint64_t g_launches = 0;

// Bracket the dominant kernel of a call with the caller's timing events.  In a
// stream capture the records become graph nodes of their own (external flag).
void record(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  else cudaEventRecord(ev, s);
}
void mark_start(cudaStream_t s) { if (g_ev_start) record(g_ev_start, s); }
void mark_stop(cudaStream_t s) { if (g_ev_stop) record(g_ev_stop, s); }
void count_launches(int n) { g_launches += (uint64_t)n; }

// Launch with programmatic stream serialisation: the kernel may start while the
// previous kernel in the stream drains; it calls griddepcontrol.wait before it
// touches memory that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

liger_status fail(liger_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

liger_status cuda_check(const char* where) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(LIGER_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
  return LIGER_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A named NVTX range over one entry point, for profilers that attach to NVTX
// (ncu --nvtx, Nsight Systems); with none attached the calls return at once.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Which prefill kernel serves a call.
enum class PrefillPath { kSimt, kTensorCore };

PrefillPath choose_prefill_path(long ntok, int Hq, int Hkv, int d, int w, liger_dtype dt,
                                const float* initial_state) {
  if (liger::options().force_general_prefill) return PrefillPath::kSimt;
  (void)initial_state;   // taken by both paths
  if (ntok > 0 && dt == LIGER_BF16 && w == 64 && (Hq / Hkv) % 2 == 0 && liger::tc::supports(d))
    return PrefillPath::kTensorCore;
  return PrefillPath::kSimt;
}

liger_status check_common(int Hq, int Hkv, int d, int w, float alpha, liger_dtype dt) {
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(LIGER_ERR_INVALID_ARG, "need Hq >= 1, Hkv >= 1 and Hq %% Hkv == 0 (Hq=%d Hkv=%d)", Hq, Hkv);
  if (w < 1) return fail(LIGER_ERR_INVALID_ARG, "window w must be >= 1 (w=%d)", w);
  if (!(alpha >= 0.f && alpha <= 1.f))
    return fail(LIGER_ERR_INVALID_ARG, "alpha must lie in [0, 1] (alpha=%g)", (double)alpha);
  if (dt != LIGER_BF16 && dt != LIGER_FP32) return fail(LIGER_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (d != 64 && d != 128) return fail(LIGER_ERR_UNSUPPORTED, "head dim d=%d (supported: 64, 128)", d);
  if (w > 64) return fail(LIGER_ERR_UNSUPPORTED, "window w=%d (supported: 1..64)", w);
  return LIGER_OK;
}

template <typename Tin, int D, bool VG = false>
liger_status launch_simt_prefill(const liger::SimtPrefillArgs& a, long units, cudaStream_t s, bool timed = true) {
  const size_t smem = liger::simt_prefill_smem_bytes<D, VG>();
  auto kern = liger::prefill_simt_kernel<Tin, D, VG>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return cuda_check("cudaFuncSetAttribute(prefill_simt)");
  const long blocks = units * a.Hq;
  if (blocks > 0x7fffffffL) return fail(LIGER_ERR_UNSUPPORTED, "too many (sequence, head) units");
  if (timed) mark_start(s);
  kern<<<(unsigned)blocks, liger::kSimtThreads, smem, s>>>(a);
  if (timed) mark_stop(s);
  ++g_launches;
  return cuda_check("prefill_simt launch");
}

// Segment-parallel general prefill: plan, per-segment states, scan, the general kernel per
// (segment, q head); groups whose initial-state copies differ are rerun unsegmented.
template <typename Tin, int D, bool VG>
liger_status run_segmented(const liger::SimtPrefillArgs& a, int n_seqs, long T_total, void* ws,
                           cudaStream_t s) {
  namespace sg = liger::seg;
  const sg::Layout L = sg::layout(T_total, n_seqs, a.Hkv, D);
  char* w = static_cast<char*>(ws);
  auto* segs = reinterpret_cast<liger::SimtSeg*>(w + L.off_segs);
  int* count = reinterpret_cast<int*>(w);
  float* lam = reinterpret_cast<float*>(w + L.off_lam);
  float* ds = reinterpret_cast<float*>(w + L.off_ds);
  uint32_t* flags = reinterpret_cast<uint32_t*>(w + L.off_flags);
  if (L.cap * a.Hkv > 0x7fffffffL || L.cap * a.Hq > 0x7fffffffL ||
      (long)n_seqs * a.Hkv * (D * D / liger::seg::kScanThreads) > 0x7fffffffL)
    return fail(LIGER_ERR_UNSUPPORTED, "too many segments");
  sg::plan_kernel<<<1, 32, 0, s>>>(a.cu, a.T, n_seqs, T_total, segs, count, L.cap, flags, a.Hkv);
  ++g_launches;
  constexpr size_t seg_smem = sg::seg_state_smem_bytes<D, VG>();
  if (cudaFuncSetAttribute(sg::seg_state_kernel<Tin, D, VG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)seg_smem) != cudaSuccess)
    return cuda_check("cudaFuncSetAttribute(segment states)");
  sg::seg_state_kernel<Tin, D, VG><<<(unsigned)(L.cap * a.Hkv), sg::kSegThreads, seg_smem, s>>>(
      static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v), a.Hkv, segs, count, ds, lam);
  ++g_launches;
  sg::scan_kernel<D><<<(unsigned)((long)n_seqs * a.Hkv * (D * D / sg::kScanThreads)), sg::kScanThreads, 0, s>>>(
      segs, count, a.Hq, a.Hkv, a.init_state, ds, lam, flags);
  ++g_launches;
  liger_status st = cuda_check("segmented prefill launch");
  if (st != LIGER_OK) return st;
  liger::SimtPrefillArgs b = a;
  b.segs = segs;
  b.n_segs = count;
  b.seg_state = ds;
  b.only_flagged = nullptr;
  st = launch_simt_prefill<Tin, D, VG>(b, L.cap, s);
  if (st != LIGER_OK || !a.init_state) return st;
  liger::SimtPrefillArgs f = a;
  f.segs = nullptr;
  f.only_flagged = flags;
  return launch_simt_prefill<Tin, D, VG>(f, n_seqs, s, false);
}

template <typename Tin>
liger_status launch_ring(const void* k, const void* v, void* ring, int32_t* pos, const int32_t* cu,
                         long T, int n_seqs, int Hkv, int d, int w, cudaStream_t s) {
  if (!ring && !pos) return LIGER_OK;
  dim3 grid((unsigned)n_seqs, (unsigned)Hkv);
  liger::prefill_ring_kernel<Tin><<<grid, 256, 0, s>>>(
      static_cast<const Tin*>(k), static_cast<const Tin*>(v), static_cast<Tin*>(ring), pos, cu, T,
      Hkv, d, w);
  ++g_launches;
  return cuda_check("prefill_ring launch");
}

// Error word of the streamed decode kernels (bit 0: a bounded wait gave up; word 1:
// the first site), one per device; read and cleared by liger_attn_decode_status().
__device__ uint32_t g_decode_err[2];

// The persistent stream (one CTA per SM) over `units` units of G heads each.
template <typename Tin, int D, int G, bool PER_HEAD>
liger_status launch_decode_stream(const liger::DecodeArgs& a, unsigned units, cudaStream_t s) {
  constexpr size_t smem = liger::kvs::Layout<Tin, D, G>::BYTES;
  auto kern = liger::kvs::decode_stream_kernel<Tin, D, G, PER_HEAD>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return cuda_check("cudaFuncSetAttribute(decode_stream)");
  void* err = nullptr;
  const cudaError_t ge = cudaGetSymbolAddress(&err, g_decode_err);
  if (ge != cudaSuccess) return fail(LIGER_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(ge));
  liger::kvs::Args c{a, (int)units, static_cast<uint32_t*>(err), liger::tc::wait_limit_ns()};
  const int sms = liger::tc::num_sms();
  const unsigned grid = units < (unsigned)sms ? units : (unsigned)sms;   // one CTA per SM
  mark_start(s);
  if (launch_pdl(kern, dim3(grid), dim3(liger::kvs::threads<G>()), smem, s, c) != cudaSuccess)
    return cuda_check("decode_stream launch");
  mark_stop(s);
  ++g_launches;
  return cuda_check("decode_stream launch");
}

template <typename Tin, int D>
liger_status launch_decode(const liger::DecodeArgs& a, unsigned blocks, cudaStream_t s) {
  if constexpr (liger::kvs::fits<Tin, D, 1>()) return launch_decode_stream<Tin, D, 1, true>(a, blocks, s);
  constexpr size_t smem = liger::decode_smem_bytes<Tin, D>();
  auto kern = liger::decode_kernel<Tin, D>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return cuda_check("cudaFuncSetAttribute(decode)");
  mark_start(s);
  if (launch_pdl(kern, dim3(blocks), dim3(liger::kDecodeThreads), smem, s, a) != cudaSuccess)
    return cuda_check("decode launch");
  mark_stop(s);
  ++g_launches;
  return cuda_check("decode launch");
}

template <typename Tin, int D, int G>
liger_status launch_decode_kvshared(const liger::DecodeArgs& a, unsigned blocks, cudaStream_t s) {
  if constexpr (liger::kvs::fits<Tin, D, G>()) return launch_decode_stream<Tin, D, G, false>(a, blocks, s);
  constexpr size_t smem = liger::decode_smem_bytes<Tin, D>();
  auto kern = liger::decode_kvshared_kernel<Tin, D, G>;
  // static + dynamic shared memory can exceed the default 48 KiB: always raise the limit
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return cuda_check("cudaFuncSetAttribute(decode_kvshared)");
  mark_start(s);
  if (launch_pdl(kern, dim3(blocks), dim3(liger::kDecodeThreads), smem, s, a) != cudaSuccess)
    return cuda_check("decode_kvshared launch");
  mark_stop(s);
  ++g_launches;
  return cuda_check("decode_kvshared launch");
}

template <typename Tin, int D>
liger_status decode_kvshared_g(const liger::DecodeArgs& a, int G, unsigned blocks, cudaStream_t s) {
  switch (G) {
    case 1: return launch_decode_kvshared<Tin, D, 1>(a, blocks, s);
    case 2: return launch_decode_kvshared<Tin, D, 2>(a, blocks, s);
    case 4: return launch_decode_kvshared<Tin, D, 4>(a, blocks, s);
    default: return fail(LIGER_ERR_UNSUPPORTED, "shared-state decode supports Hq/Hkv in {1, 2, 4} (got %d)", G);
  }
}

template <typename Tin, bool VG = false>
liger_status prefill_simt_dispatch(const liger::SimtPrefillArgs& a, int d, int n_seqs, cudaStream_t s) {
  return d == 64 ? launch_simt_prefill<Tin, 64, VG>(a, n_seqs, s) : launch_simt_prefill<Tin, 128, VG>(a, n_seqs, s);
}

template <typename Tin, bool VG>
liger_status segmented_dispatch(const liger::SimtPrefillArgs& a, int d, int n_seqs, long T_total, void* ws,
                                cudaStream_t s) {
  return d == 64 ? run_segmented<Tin, 64, VG>(a, n_seqs, T_total, ws, s)
                 : run_segmented<Tin, 128, VG>(a, n_seqs, T_total, ws, s);
}

// Error word of the causal-attention kernel (bit 0: a bounded wait gave up; word 1: the
// first site), one per device; read and cleared by liger_attn_full_causal_status().
__device__ uint32_t g_full_attn_err[2];

template <int D>
liger_status launch_full_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const liger::fa::Params& prm, int Hq, int n_seqs, cudaStream_t s) {
  auto kern = liger::fa::full_attn_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)liger::fa::Smem<D>::BYTES) !=
      cudaSuccess)
    return cuda_check("cudaFuncSetAttribute(full_attn)");
  const dim3 grid((unsigned)((prm.n_qblk + 1) / 2), (unsigned)Hq, (unsigned)n_seqs);   // pairs of query blocks
  mark_start(s);
  kern<<<grid, liger::fa::kThreads, liger::fa::Smem<D>::BYTES, s>>>(mq, mk, mv, prm);
  mark_stop(s);
  ++g_launches;
  return cuda_check("full_attn launch");
}

}  // namespace

namespace liger {

namespace {
Options read_options() {
  Options o{};
  const char* path = std::getenv("LIGER_PREFILL_PATH");
  o.force_general_prefill = path && (std::strcmp(path, "general") == 0 || std::strcmp(path, "simt") == 0);
  const char* lim = std::getenv("LIGER_WAIT_LIMIT_NS");
  o.wait_limit_ns = (lim && *lim) ? std::strtoull(lim, nullptr, 10) : 0ull;
  const char* stall = std::getenv("LIGER_TEST_INJECT_STALL");
  o.inject_stall_calls = (stall && *stall) ? std::strtol(stall, nullptr, 10) : 0;
  return o;
}
// Initialised when the library is loaded; never re-read.
const Options g_options = read_options();
std::atomic<long> g_stalls_taken{0};
}  // namespace

const Options& options() { return g_options; }

bool take_injected_stall() {
  if (g_options.inject_stall_calls <= 0) return false;
  return g_stalls_taken.fetch_add(1) < g_options.inject_stall_calls;
}

// Records a failure for liger_last_error() from other translation units of the library.
void set_last_error(liger_status status, const char* message) { fail(status, "%s", message); }

// Whether a prefill with these arguments runs on the tensor-core path, the only one that
// uses the workspace.
bool prefill_uses_workspace(int B, int Hq, int Hkv, int T, int d, int w, liger_dtype dt,
                            const float* initial_state) {
  if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv) return false;
  return choose_prefill_path((long)B * T, Hq, Hkv, d, w, dt, initial_state) == PrefillPath::kTensorCore;
}
}  // namespace liger

extern "C" {

int liger_abi_version(void) { return LIGER_ABI_VERSION; }

const char* liger_last_error(void) { return g_last_error.c_str(); }

void liger_set_timing_events(void* start_event, void* stop_event) {
  g_ev_start = static_cast<cudaEvent_t>(start_event);
  g_ev_stop = static_cast<cudaEvent_t>(stop_event);
}

uint64_t liger_kernel_launches(void) { return g_launches; }

size_t liger_attn_prefill_workspace_size(int B, int Hq, int Hkv, int T, int d, int n_seqs,
                                         liger_dtype dt) {
  if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv) return 0;
  if (dt != LIGER_BF16 || (d != 64 && d != 128) || (Hq / Hkv) % 2) return 0;
  const int n = n_seqs > 0 ? n_seqs : B;
  return liger::tc::workspace_bytes(B, Hq, Hkv, (long)T, d, n);
}

liger_status liger_attn_prefill_plan(int B, int Hq, int Hkv, int T, int d, int n_seqs, int packed,
                                     int* chunks_per_segment, int* max_segments,
                                     int* state_subsegments, int* sm_count, size_t* plan_bytes) {
  g_last_error.clear();
  if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv)
    return fail(LIGER_ERR_INVALID_ARG, "need B >= 1, T >= 0, Hq >= 1, Hkv >= 1, Hq %% Hkv == 0");
  if (packed) {
    if (B != 1 || n_seqs < 1)
      return fail(LIGER_ERR_INVALID_ARG, "packed input needs B == 1 and n_seqs >= 1 (B=%d n_seqs=%d)", B, n_seqs);
  } else if (n_seqs != B) {
    return fail(LIGER_ERR_INVALID_ARG, "without packing n_seqs must equal B (n_seqs=%d B=%d)", n_seqs, B);
  }
  if (!liger::tc::supports(d) || (Hq / Hkv) % 2)
    return fail(LIGER_ERR_UNSUPPORTED, "the general kernel takes these sizes (d=%d, Hq/Hkv=%d); it needs no plan",
                d, Hq / Hkv);
  const liger::tc::Plan pl = liger::tc::make_plan(B, Hq, Hkv, (long)T, d, n_seqs, packed != 0);
  if (chunks_per_segment) *chunks_per_segment = pl.L;
  if (max_segments) *max_segments = pl.n_seg_max;
  if (state_subsegments) *state_subsegments = pl.nsub;
  if (sm_count) *sm_count = liger::tc::num_sms();
  if (plan_bytes) *plan_bytes = pl.total;
  return LIGER_OK;
}

liger_status liger_attn_prefill(const void* q, const void* k, const void* v, void* out,
                                float* final_state, int B, int Hq, int Hkv, int T, int d, int w,
                                float alpha, liger_dtype dt, const float* initial_state,
                                const int32_t* cu_seqlens, int n_seqs, void* swa_ring_out,
                                int32_t* pos_out, void* workspace, size_t workspace_bytes,
                                void* stream) {
  const NvtxRange range("liger_attn_prefill");
  g_last_error.clear();
  liger_status st = check_common(Hq, Hkv, d, w, alpha, dt);
  if (st != LIGER_OK) return st;
  if (B < 1 || T < 0) return fail(LIGER_ERR_INVALID_ARG, "need B >= 1 and T >= 0 (B=%d T=%d)", B, T);
  if (cu_seqlens) {
    if (B != 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (B=%d)", B);
    if (n_seqs < 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires n_seqs >= 1 (n_seqs=%d)", n_seqs);
  } else if (n_seqs != B) {
    return fail(LIGER_ERR_INVALID_ARG, "without cu_seqlens n_seqs must equal B (n_seqs=%d B=%d)", n_seqs, B);
  }
  const long ntok = (long)B * T;
  if ((long)T * B * Hq > (1L << 40) / d || (long)T * B > 0x7fffffffL - 1024)   // 32-bit token indices
    return fail(LIGER_ERR_UNSUPPORTED, "tensor too large");
  if (ntok > 0 && (!q || !k || !v || !out))
    return fail(LIGER_ERR_INVALID_ARG, "q, k, v and out must be non-null");
  const void* ptrs[] = {q, k, v, out, final_state, initial_state, swa_ring_out, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(LIGER_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens must be 4-byte aligned");
  if (pos_out && (reinterpret_cast<uintptr_t>(pos_out) & 3u))
    return fail(LIGER_ERR_INVALID_ARG, "pos_out must be 4-byte aligned");

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const PrefillPath path = choose_prefill_path(ntok, Hq, Hkv, d, w, dt, initial_state);
  if (path == PrefillPath::kTensorCore) {
    const size_t need = liger::tc::workspace_bytes(B, Hq, Hkv, (long)T, d, n_seqs);
    if (need > workspace_bytes || (need && !workspace))
      return fail(LIGER_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", need, workspace_bytes);
    liger::tc::PrefillProblem pb{q, k, v, out, final_state, initial_state, cu_seqlens, B, Hq, Hkv, (long)T, d,
                                 n_seqs, alpha};
    const liger::tc::LaunchHooks hooks{mark_start, mark_stop, count_launches};
    const uint32_t* s0_flags = nullptr;
    st = liger::tc::run_prefill(pb, workspace, s, hooks, &s0_flags);
    if (st != LIGER_OK) return fail(st, "%s", liger::tc::last_message());
    if (initial_state) {
      // Groups whose q heads start from different initial states: the general kernel
      // recomputes those (sequence, kv head) units; its other CTAs return at once.
      liger::SimtPrefillArgs a{q, k, v, out, final_state, initial_state, cu_seqlens, Hq, Hkv, w, (long)T, alpha,
                               s0_flags};
      const auto hooks_off = std::make_pair(g_ev_start, g_ev_stop);
      g_ev_start = g_ev_stop = nullptr;   // the timing events bracket the chunk pass only
      st = prefill_simt_dispatch<__nv_bfloat16>(a, d, n_seqs, s);
      g_ev_start = hooks_off.first;
      g_ev_stop = hooks_off.second;
      if (st != LIGER_OK) return st;
    }
  } else {
    liger::SimtPrefillArgs a{q, k, v, out, final_state, initial_state, cu_seqlens, Hq, Hkv, w, (long)T, alpha,
                             nullptr};
    st = dt == LIGER_BF16 ? prefill_simt_dispatch<__nv_bfloat16>(a, d, n_seqs, s)
                          : prefill_simt_dispatch<float>(a, d, n_seqs, s);
    if (st != LIGER_OK) return st;
  }
  if (dt == LIGER_BF16)
    return launch_ring<__nv_bfloat16>(k, v, swa_ring_out, pos_out, cu_seqlens, T, n_seqs, Hkv, d, w, s);
  return launch_ring<float>(k, v, swa_ring_out, pos_out, cu_seqlens, T, n_seqs, Hkv, d, w, s);
}

size_t liger_attn_prefill_vector_gate_workspace_size(int B, int Hq, int Hkv, int T, int d, int n_seqs,
                                                     liger_dtype dt) {
  if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || (d != 64 && d != 128)) return 0;
  if (dt != LIGER_BF16 && dt != LIGER_FP32) return 0;
  const int n = n_seqs > 0 ? n_seqs : B;
  // packed input (B == 1, n sequences) and B separate sequences: the larger layout
  const size_t a = liger::seg::layout((long)B * T, B, Hkv, d).total;
  const size_t b = liger::seg::layout((long)B * T, n, Hkv, d).total;
  return a > b ? a : b;
}

liger_status liger_attn_prefill_vector_gate(const void* q, const void* k, const void* v, void* out,
                                            float* final_state, int B, int Hq, int Hkv, int T, int d, int w,
                                            float alpha, liger_dtype dt, const float* initial_state,
                                            const int32_t* cu_seqlens, int n_seqs, void* swa_ring_out,
                                            int32_t* pos_out, void* workspace, size_t workspace_bytes,
                                            void* stream) {
  const NvtxRange range("liger_attn_prefill_vector_gate");
  g_last_error.clear();
  liger_status st = check_common(Hq, Hkv, d, w, alpha, dt);
  if (st != LIGER_OK) return st;
  if (B < 1 || T < 0) return fail(LIGER_ERR_INVALID_ARG, "need B >= 1 and T >= 0 (B=%d T=%d)", B, T);
  if (cu_seqlens) {
    if (B != 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (B=%d)", B);
    if (n_seqs < 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires n_seqs >= 1 (n_seqs=%d)", n_seqs);
  } else if (n_seqs != B) {
    return fail(LIGER_ERR_INVALID_ARG, "without cu_seqlens n_seqs must equal B (n_seqs=%d B=%d)", n_seqs, B);
  }
  if ((long)T * B * Hq > (1L << 40) / d || (long)T * B > 0x7fffffffL - 1024)
    return fail(LIGER_ERR_UNSUPPORTED, "tensor too large");
  if ((long)B * T > 0 && (!q || !k || !v || !out))
    return fail(LIGER_ERR_INVALID_ARG, "q, k, v and out must be non-null");
  const void* ptrs[] = {q, k, v, out, final_state, initial_state, swa_ring_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(LIGER_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens must be 4-byte aligned");
  if (pos_out && (reinterpret_cast<uintptr_t>(pos_out) & 3u))
    return fail(LIGER_ERR_INVALID_ARG, "pos_out must be 4-byte aligned");
  if (workspace && !aligned16(workspace))
    return fail(LIGER_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  const long T_total = (long)B * T;
  const size_t need = T_total > 0 ? liger::seg::layout(T_total, n_seqs, Hkv, d).total : 0;
  if (need > workspace_bytes || (need && !workspace))
    return fail(LIGER_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", need, workspace_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  liger::SimtPrefillArgs a{q, k, v, out, final_state, initial_state, cu_seqlens, Hq, Hkv, w, (long)T, alpha, nullptr};
  if (T_total > 0) {
    st = dt == LIGER_BF16 ? segmented_dispatch<__nv_bfloat16, true>(a, d, n_seqs, T_total, workspace, s)
                          : segmented_dispatch<float, true>(a, d, n_seqs, T_total, workspace, s);
  } else {
    st = dt == LIGER_BF16 ? prefill_simt_dispatch<__nv_bfloat16, true>(a, d, n_seqs, s)
                          : prefill_simt_dispatch<float, true>(a, d, n_seqs, s);
  }
  if (st != LIGER_OK) return st;
  if (dt == LIGER_BF16)
    return launch_ring<__nv_bfloat16>(k, v, swa_ring_out, pos_out, cu_seqlens, T, n_seqs, Hkv, d, w, s);
  return launch_ring<float>(k, v, swa_ring_out, pos_out, cu_seqlens, T, n_seqs, Hkv, d, w, s);
}

namespace {
liger_status decode_impl(const void* q, const void* k, const void* v, float* state, void* swa_ring, void* out,
                         int32_t* pos, int B, int Hq, int Hkv, int d, int w, float alpha, liger_dtype dt,
                         void* stream, int vector_gate);
}

liger_status liger_attn_decode_vector_gate(const void* q, const void* k, const void* v, float* state,
                                           void* swa_ring, void* out, int32_t* pos, int B, int Hq, int Hkv,
                                           int d, int w, float alpha, liger_dtype dt, void* stream) {
  const NvtxRange range("liger_attn_decode_vector_gate");
  return decode_impl(q, k, v, state, swa_ring, out, pos, B, Hq, Hkv, d, w, alpha, dt, stream, 1);
}

liger_status liger_attn_decode(const void* q, const void* k, const void* v, float* state,
                               void* swa_ring, void* out, int32_t* pos, int B, int Hq, int Hkv,
                               int d, int w, float alpha, liger_dtype dt, void* stream) {
  const NvtxRange range("liger_attn_decode");
  return decode_impl(q, k, v, state, swa_ring, out, pos, B, Hq, Hkv, d, w, alpha, dt, stream, 0);
}

}  // extern "C"

namespace {
liger_status decode_impl(const void* q, const void* k, const void* v, float* state, void* swa_ring, void* out,
                         int32_t* pos, int B, int Hq, int Hkv, int d, int w, float alpha, liger_dtype dt,
                         void* stream, int vector_gate) {
  g_last_error.clear();
  liger_status st = check_common(Hq, Hkv, d, w, alpha, dt);
  if (st != LIGER_OK) return st;
  if (B < 1) return fail(LIGER_ERR_INVALID_ARG, "need B >= 1 (B=%d)", B);
  if ((long)B * Hq > 0x7fffffffL) return fail(LIGER_ERR_UNSUPPORTED, "too many (sequence, head) units");
  if (!q || !k || !v || !state || !swa_ring || !out || !pos)
    return fail(LIGER_ERR_INVALID_ARG, "all decode pointers must be non-null");
  const void* ptrs[] = {q, k, v, state, swa_ring, out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(LIGER_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(pos) & 3u) return fail(LIGER_ERR_INVALID_ARG, "pos must be 4-byte aligned");

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  liger::DecodeArgs a{q, k, v, state, swa_ring, out, pos, Hq, Hkv, w, alpha, vector_gate};
  const unsigned blocks = (unsigned)((long)B * Hq);
  if (dt == LIGER_BF16) st = d == 64 ? launch_decode<__nv_bfloat16, 64>(a, blocks, s)
                                     : launch_decode<__nv_bfloat16, 128>(a, blocks, s);
  else st = d == 64 ? launch_decode<float, 64>(a, blocks, s) : launch_decode<float, 128>(a, blocks, s);
  if (st != LIGER_OK) return st;
  if (launch_pdl(liger::advance_pos_kernel, dim3((B + 255) / 256), dim3(256), 0, s, pos, B) != cudaSuccess)
    return cuda_check("advance_pos launch");
  ++g_launches;
  return cuda_check("advance_pos launch");
}
}  // namespace

extern "C" {

liger_status liger_attn_prefill_status(const void* workspace, size_t workspace_bytes) {
  g_last_error.clear();
  if (!workspace || workspace_bytes < 12) return LIGER_OK;   // no tensor-core pass ran with it
  uint32_t hdr[3] = {0u, 0u, 0u};
  const cudaError_t e = cudaMemcpy(hdr, workspace, sizeof hdr, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(LIGER_ERR_CUDA, "reading the workspace header: %s", cudaGetErrorString(e));
  if (hdr[0] & 1u)
    return fail(LIGER_ERR_TIMEOUT, "a prefill kernel gave up waiting (site 0x%08x: role %u, barrier %u, chunk %u)",
                hdr[1], hdr[1] >> 28, (hdr[1] >> 20) & 0xFFu, hdr[1] & 0xFFFFFu);
  if (hdr[0]) return fail(LIGER_ERR_CUDA, "prefill error word 0x%x", hdr[0]);
  return LIGER_OK;
}

size_t liger_attn_prefill_backward_workspace_size(int B, int Hq, int Hkv, int T, int d, int n_seqs,
                                                  liger_dtype dt) {
  if (B < 1 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv) return 0;
  if (dt != LIGER_BF16 || (d != 64 && d != 128) || (Hq / Hkv) % 2) return 0;
  return liger::bwd::bwd_workspace_bytes(B, Hq, Hkv, (long)T, d, n_seqs > 0 ? n_seqs : B);
}

liger_status liger_attn_prefill_backward(const void* q, const void* k, const void* v, const void* d_out,
                                         const float* d_final_state, const float* initial_state, int B, int Hq,
                                         int Hkv, int T, int d, int w, float alpha, liger_dtype dt,
                                         const int32_t* cu_seqlens, int n_seqs, void* dq, void* dk, void* dv,
                                         float* d_initial_state, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  const NvtxRange range("liger_attn_prefill_backward");
  g_last_error.clear();
  liger_status st = check_common(Hq, Hkv, d, w, alpha, dt);
  if (st != LIGER_OK) return st;
  if (B < 1 || T < 0) return fail(LIGER_ERR_INVALID_ARG, "need B >= 1 and T >= 0 (B=%d T=%d)", B, T);
  if (cu_seqlens) {
    if (B != 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (B=%d)", B);
    if (n_seqs < 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires n_seqs >= 1 (n_seqs=%d)", n_seqs);
  } else if (n_seqs != B) {
    return fail(LIGER_ERR_INVALID_ARG, "without cu_seqlens n_seqs must equal B (n_seqs=%d B=%d)", n_seqs, B);
  }
  if (dt != LIGER_BF16 || w != 64 || (Hq / Hkv) % 2)
    return fail(LIGER_ERR_UNSUPPORTED, "the backward takes bf16, w = 64 and an even Hq/Hkv (dt=%d w=%d G=%d)",
                (int)dt, w, Hq / Hkv);
  if ((long)T * B * Hq > (1L << 40) / d || (long)T * B > 0x7fffffffL - 1024)
    return fail(LIGER_ERR_UNSUPPORTED, "tensor too large");
  const long ntok = (long)B * T;
  if (ntok > 0 && (!q || !k || !v || !d_out || !dq || !dk || !dv))
    return fail(LIGER_ERR_INVALID_ARG, "q, k, v, d_out, dq, dk and dv must be non-null");
  const void* ptrs[] = {q, k, v, d_out, d_final_state, initial_state, dq, dk, dv, d_initial_state, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return fail(LIGER_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens must be 4-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ntok == 0) {   // no tokens: the state passes through unchanged
    if (d_initial_state) {
      const size_t bytes = (size_t)n_seqs * Hkv * d * d * 4;
      if (!d_final_state) {
        if (cudaMemsetAsync(d_initial_state, 0, bytes, s) != cudaSuccess) return cuda_check("cudaMemsetAsync");
      } else {
        return fail(LIGER_ERR_UNSUPPORTED, "an empty backward with d_final_state: sum the group's heads instead");
      }
    }
    return LIGER_OK;
  }
  const size_t need = liger::bwd::bwd_workspace_bytes(B, Hq, Hkv, (long)T, d, n_seqs);
  if (need > workspace_bytes || !workspace)
    return fail(LIGER_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", need, workspace_bytes);
  liger::bwd::BwdProblem pb{q, k, v, d_out, d_final_state, initial_state, dq, dk, dv, d_initial_state, cu_seqlens,
                            B, Hq, Hkv, (long)T, d, n_seqs, alpha};
  const liger::tc::LaunchHooks hooks{mark_start, mark_stop, count_launches};
  st = liger::bwd::run_backward(pb, workspace, s, hooks);
  if (st != LIGER_OK) return fail(st, "%s", liger::tc::last_message());
  return LIGER_OK;
}

liger_status liger_attn_full_causal(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                                    int Hkv, int T, int d, liger_dtype dt, const int32_t* cu_seqlens, int n_seqs,
                                    int max_seqlen, void* stream) {
  const NvtxRange range("liger_attn_full_causal");
  g_last_error.clear();
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(LIGER_ERR_INVALID_ARG, "need Hq >= 1, Hkv >= 1 and Hq %% Hkv == 0 (Hq=%d Hkv=%d)", Hq, Hkv);
  if (B < 1 || T < 0) return fail(LIGER_ERR_INVALID_ARG, "need B >= 1 and T >= 0 (B=%d T=%d)", B, T);
  if (dt != LIGER_BF16 && dt != LIGER_FP32) return fail(LIGER_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
  if (dt != LIGER_BF16) return fail(LIGER_ERR_UNSUPPORTED, "causal attention takes bf16 inputs");
  if (d != 64 && d != 128) return fail(LIGER_ERR_UNSUPPORTED, "head dim d=%d (supported: 64, 128)", d);
  if (cu_seqlens) {
    if (B != 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (B=%d)", B);
    if (n_seqs < 1) return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens requires n_seqs >= 1 (n_seqs=%d)", n_seqs);
    if (max_seqlen < 0 || max_seqlen > T)
      return fail(LIGER_ERR_INVALID_ARG, "max_seqlen must lie in [0, T] (max_seqlen=%d T=%d)", max_seqlen, T);
    if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)
      return fail(LIGER_ERR_INVALID_ARG, "cu_seqlens must be 4-byte aligned");
  } else if (n_seqs != B) {
    return fail(LIGER_ERR_INVALID_ARG, "without cu_seqlens n_seqs must equal B (n_seqs=%d B=%d)", n_seqs, B);
  }
  const long NT = (long)B * T;
  if (NT == 0) return LIGER_OK;
  if (NT * Hq > (1L << 40) / d || NT > 0x7fffffffL - 1024)   // TMA token coordinates are 32-bit
    return fail(LIGER_ERR_UNSUPPORTED, "tensor too large");
  if (!q || !k || !v || !out) return fail(LIGER_ERR_INVALID_ARG, "q, k, v and out must be non-null");
  const void* ptrs[] = {q, k, v, out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return fail(LIGER_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const long longest = cu_seqlens ? (long)max_seqlen : (long)T;
  const long n_qblk = (longest + liger::fa::BM - 1) / liger::fa::BM;
  if (n_qblk == 0) return LIGER_OK;
  if (n_qblk > 0x7fffffffL || (long)n_seqs > 65535 || Hq > 65535)
    return fail(LIGER_ERR_UNSUPPORTED, "grid too large");
  CUtensorMap mq, mk, mv;
  const auto enc = reinterpret_cast<liger::fa::EncodeTiledFn>(liger::tc::encode_fn());
  if (!liger::fa::make_map(enc, &mq, q, d, Hq, NT) || !liger::fa::make_map(enc, &mk, k, d, Hkv, NT) ||
      !liger::fa::make_map(enc, &mv, v, d, Hkv, NT))
    return fail(LIGER_ERR_CUDA, "cuTensorMapEncodeTiled failed for the causal attention");
  void* err = nullptr;
  const cudaError_t ge = cudaGetSymbolAddress(&err, g_full_attn_err);
  if (ge != cudaSuccess) return fail(LIGER_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(ge));
  liger::fa::Params prm{};
  prm.out = out;
  prm.cu = cu_seqlens;
  prm.T = T;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.n_qblk = (int)n_qblk;
  prm.err = static_cast<uint32_t*>(err);
  prm.wait_ns = liger::tc::wait_limit_ns();
  prm.scale_log2 = 1.4426950408889634f / std::sqrt((float)d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_full_attn<64>(mq, mk, mv, prm, Hq, n_seqs, s)
                 : launch_full_attn<128>(mq, mk, mv, prm, Hq, n_seqs, s);
}

liger_status liger_attn_decode_status(void) {
  g_last_error.clear();
  uint32_t hdr[2] = {0u, 0u};
  cudaError_t e = cudaMemcpyFromSymbol(hdr, g_decode_err, sizeof hdr);
  if (e != cudaSuccess) return fail(LIGER_ERR_CUDA, "reading the decode's error word: %s", cudaGetErrorString(e));
  const uint32_t zero[2] = {0u, 0u};
  e = cudaMemcpyToSymbol(g_decode_err, zero, sizeof zero);
  if (e != cudaSuccess) return fail(LIGER_ERR_CUDA, "clearing the decode's error word: %s", cudaGetErrorString(e));
  if (hdr[0] & 1u)
    return fail(LIGER_ERR_TIMEOUT, "a decode kernel gave up waiting (site 0x%08x: role %u, barrier %u, unit %u)",
                hdr[1], hdr[1] >> 28, (hdr[1] >> 20) & 0xFFu, hdr[1] & 0xFFFFFu);
  return LIGER_OK;
}

liger_status liger_attn_full_causal_status(void) {
  g_last_error.clear();
  uint32_t hdr[2] = {0u, 0u};
  cudaError_t e = cudaMemcpyFromSymbol(hdr, g_full_attn_err, sizeof hdr);
  if (e != cudaSuccess) return fail(LIGER_ERR_CUDA, "reading the causal attention's error word: %s", cudaGetErrorString(e));
  const uint32_t zero[2] = {0u, 0u};
  e = cudaMemcpyToSymbol(g_full_attn_err, zero, sizeof zero);
  if (e != cudaSuccess) return fail(LIGER_ERR_CUDA, "clearing the causal attention's error word: %s", cudaGetErrorString(e));
  if (hdr[0] & 1u)
    return fail(LIGER_ERR_TIMEOUT, "a causal attention kernel gave up waiting (site 0x%08x: role %u, barrier %u, block %u)",
                hdr[1], hdr[1] >> 28, (hdr[1] >> 20) & 0xFFu, hdr[1] & 0xFFFFFu);
  return LIGER_OK;
}

liger_status liger_attn_decode_kvshared(const void* q, const void* k, const void* v, float* state,
                                        void* swa_ring, void* out, int32_t* pos, int B, int Hq, int Hkv,
                                        int d, int w, float alpha, liger_dtype dt, void* stream) {
  const NvtxRange range("liger_attn_decode_kvshared");
  g_last_error.clear();
  liger_status st = check_common(Hq, Hkv, d, w, alpha, dt);
  if (st != LIGER_OK) return st;
  if (B < 1) return fail(LIGER_ERR_INVALID_ARG, "need B >= 1 (B=%d)", B);
  if ((long)B * Hkv > 0x7fffffffL) return fail(LIGER_ERR_UNSUPPORTED, "too many (sequence, kv head) units");
  if (!q || !k || !v || !state || !swa_ring || !out || !pos)
    return fail(LIGER_ERR_INVALID_ARG, "all decode pointers must be non-null");
  const void* ptrs[] = {q, k, v, state, swa_ring, out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(LIGER_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(pos) & 3u) return fail(LIGER_ERR_INVALID_ARG, "pos must be 4-byte aligned");
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4)
    return fail(LIGER_ERR_UNSUPPORTED, "shared-state decode supports Hq/Hkv in {1, 2, 4} (got %d)", G);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  liger::DecodeArgs a{q, k, v, state, swa_ring, out, pos, Hq, Hkv, w, alpha};
  const unsigned blocks = (unsigned)((long)B * Hkv);
  if (dt == LIGER_BF16)
    st = d == 64 ? decode_kvshared_g<__nv_bfloat16, 64>(a, G, blocks, s)
                 : decode_kvshared_g<__nv_bfloat16, 128>(a, G, blocks, s);
  else st = d == 64 ? decode_kvshared_g<float, 64>(a, G, blocks, s) : decode_kvshared_g<float, 128>(a, G, blocks, s);
  if (st != LIGER_OK) return st;
  if (launch_pdl(liger::advance_pos_kernel, dim3((B + 255) / 256), dim3(256), 0, s, pos, B) != cudaSuccess)
    return cuda_check("advance_pos launch");
  ++g_launches;
  return cuda_check("advance_pos launch");
}

}  // extern "C"
