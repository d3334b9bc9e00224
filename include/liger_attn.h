/*
 * liger_attn.h -- C ABI of the Liger Attention forward pass for NVIDIA B200
 * (sm_100a).  Built into libliger_attn.so.
 *
 * The operation.  Liger Attention ("Liger: Linearizing Large Language Models
 * to Gated Recurrent Structures", Paper-Notes page, sections
 * "核心思想：Key 投影复用构建门控", "统一的门控线性循环框架" and
 * "Liger Attention：层内混合注意力"; news article on Liger, section
 * "手法の説明") mixes, per query head h with key/value head kv = h / (Hq/Hkv):
 *
 *   gated recurrent branch (GRM):
 *     g_t   = sigmoid(mean_d k_t)                 (pooled key gate, kept as log g)
 *     phi() = softmax over the head dimension d   (applied to q_t and to k_t)
 *     S_t   = g_t * S_{t-1} + phi(k_t)^T v_t      (d x d, row = key dim, col = value dim)
 *     grm_t = phi(q_t) S_t                        (state updated before it is read)
 *   sliding-window branch (SWA), window w (64 on the pages):
 *     swa_t = sum_{j=t-w+1..t} softmax_j(q_t . k_j / sqrt(d)) v_j   (self included)
 *   output:
 *     o_t   = alpha * grm_t + (1 - alpha) * swa_t
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     contiguous, 16-byte aligned.  The library never allocates device memory
 *     and never synchronizes the host; it enqueues kernels on `stream` (a
 *     cudaStream_t, NULL = legacy default stream) and returns.
 *   - Errors: a bad argument returns LIGER_ERR_INVALID_ARG, a legal but
 *     unimplemented combination LIGER_ERR_UNSUPPORTED, a failed CUDA call
 *     LIGER_ERR_CUDA; nothing is launched in those cases (for LIGER_ERR_CUDA,
 *     launches made before the failing call stay enqueued).  The message of the
 *     last failure on the calling thread is returned by liger_last_error().
 *   - No C++ exception crosses the ABI; calls from several host threads are
 *     safe as long as they do not share output buffers.
 *   - dt is the storage type of q, k, v, out and the window ring.  The
 *     recurrent state is always fp32.  Arithmetic is fp32 (bf16 tensor-core
 *     operands with fp32 accumulation on the bf16 prefill path).
 *   - Supported: d in {64, 128}; 1 <= w <= 64 (the bf16 tensor-core prefill
 *     needs w == 64 and an even Hq/Hkv and falls back to the general kernel
 *     otherwise); Hq % Hkv == 0; 0 <= alpha <= 1.
 */
#ifndef LIGER_ATTN_H
#define LIGER_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LIGER_OK = 0,
  LIGER_ERR_INVALID_ARG = 1,
  LIGER_ERR_UNSUPPORTED = 2,
  LIGER_ERR_CUDA = 3,
  LIGER_ERR_TIMEOUT = 4
} liger_status;

typedef enum { LIGER_BF16 = 0, LIGER_FP32 = 1 } liger_dtype;

/* ABI version of this header (bumped on any signature change). */
#define LIGER_ABI_VERSION 1
int liger_abi_version(void);

/*
 * Bytes of device workspace liger_attn_prefill needs for these sizes
 * (0 is a valid answer).  T is the tokens per sequence, or the packed total
 * when cu_seqlens is used (then B == 1 and n_seqs is the number of sequences;
 * otherwise pass n_seqs = B).  Returns 0 for sizes the prefill would reject.
 */
size_t liger_attn_prefill_workspace_size(int B, int Hq, int Hkv, int T, int d, int n_seqs,
                                         liger_dtype dt);

/*
 * The launch plan the tensor-core prefill (bf16, d in {64, 128}, even
 * Hq/Hkv, w = 64) uses for these sizes.  Host only: no
 * device work; the planner reads the current device's SM count, or assumes
 * 148 when no device is present.  (The pages have no counterpart: the
 * sequence split is this implementation's way of filling the GPU.)
 *   B, Hq, Hkv, T, d, n_seqs  as for liger_attn_prefill; packed != 0 describes
 *                a call with cu_seqlens (then B == 1 and n_seqs >= 1),
 *                otherwise n_seqs must equal B.
 *   chunks_per_segment  (out, nullable) segment length in 64-token chunks: one
 *                chunk-kernel CTA per (segment, q-head pair); the length
 *                minimises waves x (length + 1.5) at one CTA per SM.
 *   max_segments        (out, nullable) the bound on segments the workspace holds.
 *   state_subsegments   (out, nullable) sub-segments per segment in the state
 *                pass (two CTAs per SM; minimises waves x (sub-length + 0.5)).
 *   sm_count            (out, nullable) the SM count the plan assumed.
 *   plan_bytes          (out, nullable) device workspace this plan uses (at most
 *                liger_attn_prefill_workspace_size for the same sizes).
 * Returns LIGER_ERR_INVALID_ARG for sizes the prefill rejects, and
 * LIGER_ERR_UNSUPPORTED for sizes the tensor-core path does not take (the
 * general kernel needs no plan); outputs are then left untouched.
 */
liger_status liger_attn_prefill_plan(int B, int Hq, int Hkv, int T, int d, int n_seqs, int packed,
                                     int* chunks_per_segment, int* max_segments,
                                     int* state_subsegments, int* sm_count, size_t* plan_bytes);

/*
 * Prefill: runs the recurrence and the window over whole sequences.
 * Sources: the recurrence and the hybrid above (Paper-Notes page, sections
 * 统一的门控线性循环框架 and Liger Attention); the parallel-in-chunk,
 * recurrent-across-chunk evaluation is the reordering the news article's
 * section "軽量ファインチューニング" credits for the linear cost.
 *
 *   q            [B, T, Hq, d]  dt          (in)
 *   k, v         [B, T, Hkv, d] dt          (in)
 *   out          [B, T, Hq, d]  dt          (out)
 *   final_state  [n, Hq, d, d]  fp32        (out, nullable) state after the last
 *                token of each sequence; every q head of a group gets its copy.
 *   initial_state[n, Hq, d, d]  fp32        (in, nullable = zero) seeds the
 *                recurrence; the window still starts at the first token.  The
 *                tensor-core path runs the q heads of a group from one state; a
 *                (sequence, group) whose heads' initial states differ is
 *                recomputed by the general kernel within the same call (correct,
 *                slower).  A final_state passed back as the next call's
 *                initial_state always has equal copies.
 *   cu_seqlens   [n + 1]        int32       (in, nullable) packed variable-length
 *                sequences: offsets into the T axis, first 0, last T, non-
 *                decreasing; requires B == 1.  The state and the window restart
 *                at each sequence start.  Without it, n = B sequences of T.
 *   swa_ring_out [n, Hkv, 2, w, d] dt       (out, nullable) window ring for decode:
 *                [., ., 0] keys, [., ., 1] values; position p of a sequence at
 *                slot p mod w for its last min(len, w) positions, zeros elsewhere.
 *   pos_out      [n]            int32       (out, nullable) sequence lengths.
 *   workspace    device scratch of at least liger_attn_prefill_workspace_size()
 *                bytes (nullable when that size is 0); contents on entry are
 *                ignored; the caller must not touch it until the call's work
 *                on `stream` is done.
 */
liger_status liger_attn_prefill(const void* q, const void* k, const void* v, void* out,
                                float* final_state, int B, int Hq, int Hkv, int T, int d, int w,
                                float alpha, liger_dtype dt, const float* initial_state,
                                const int32_t* cu_seqlens, int n_seqs, void* swa_ring_out,
                                int32_t* pos_out, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * Status of the last prefill that used this workspace (tensor-core path):
 * LIGER_ERR_TIMEOUT if one of its kernels gave up waiting on an internal
 * barrier (every wait is bounded, by default 2 s; the kernel then drains and
 * exits, the outputs are unspecified and the CUDA context stays usable),
 * LIGER_OK otherwise.  Reads the workspace header with a synchronous copy:
 * call it after the prefill's stream has completed.  (The pages have no
 * counterpart; this is failure detection.)
 */
liger_status liger_attn_prefill_status(const void* workspace, size_t workspace_bytes);

/*
 * Decode: one new token for each of B independent sequences.
 * Source: the same recurrence and hybrid, stepped once; the constant-size
 * state replacing the growing key/value cache is the linear-time,
 * constant-memory decoding both Liger pages describe (news article,
 * introduction and section "実験分析"; Paper-Notes page, section "亮点与洞察").
 *
 *   q            [B, Hq, d]        dt    (in)
 *   k, v         [B, Hkv, d]       dt    (in)
 *   state        [B, Hq, d, d]     fp32  (in/out) each q head's state is
 *                updated independently: S <- g S + phi(k)^T v.
 *   swa_ring     [B, Hkv, 2, w, d] dt    (in/out) the new key and value are
 *                written at slot pos mod w.
 *   out          [B, Hq, d]        dt    (out)
 *   pos          [B]               int32 (in/out) tokens seen so far; +1 per call.
 *                The window of the new token covers positions
 *                max(0, pos - w + 1) .. pos; slots outside it are never read.
 */
liger_status liger_attn_decode(const void* q, const void* k, const void* v, float* state,
                               void* swa_ring, void* out, int32_t* pos, int B, int Hq, int Hkv,
                               int d, int w, float alpha, liger_dtype dt, void* stream);

/*
 * Decode over one state per (sequence, kv head).  Same operation as
 * liger_attn_decode when the G = Hq/Hkv per-head states of a group are equal,
 * which holds by construction after liger_attn_prefill (it writes identical
 * copies) and under liger_attn_decode (identical updates).  The state is then
 * stored once per group, and each step moves G times less of it.
 *
 *   q      [B, Hq, d] dt; k, v [B, Hkv, d] dt; out [B, Hq, d] dt
 *   state  [B, Hkv, d, d] fp32 (in/out): S <- g S + phi(k)^T v once per group
 *   swa_ring, pos: as for liger_attn_decode.
 * Supported: G in {1, 2, 4} (other group sizes return LIGER_ERR_UNSUPPORTED).
 */
liger_status liger_attn_decode_kvshared(const void* q, const void* k, const void* v, float* state,
                                        void* swa_ring, void* out, int32_t* pos, int B, int Hq, int Hkv,
                                        int d, int w, float alpha, liger_dtype dt, void* stream);

/*
 * Timeout report of the decodes.  Except for fp32 at d = 128, every decode step
 * (liger_attn_decode, liger_attn_decode_kvshared, liger_attn_decode_vector_gate)
 * runs as one persistent CTA per SM whose internal waits are bounded (as for the
 * prefill); a wait that gives up leaves that step's outputs incomplete.  Returns
 * LIGER_ERR_TIMEOUT if any decode on the current device gave up since the last
 * query, else LIGER_OK (synchronous read; call it after the stream has completed;
 * it clears the report).
 */
liger_status liger_attn_decode_status(void);

/*
 * Prefill without caller-provided scratch (the pages have no counterpart; this
 * is a deployment convenience).  For callers that cannot allocate device
 * memory where they run the prefill -- a plugin whose host framework owns all
 * device allocations and offers it no allocator, a serving loop that reserved
 * all device memory up front, a latency-critical path that must not take the
 * implicit synchronisation of cudaMalloc/cudaFree.  Same arguments and results
 * as liger_attn_prefill without the workspace pair; the scratch is a fixed
 * array of LIGER_PREFILL_NOALLOC_SCRATCH_BYTES in this library's device image,
 * which every GPU that loads the library holds until the process exits.
 *   - Calls that take the tensor-core path (the only one that uses scratch)
 *     and whose liger_attn_prefill_workspace_size() exceeds that maximum are
 *     rejected with LIGER_ERR_UNSUPPORTED before anything is launched; calls
 *     served by the general kernel have no size limit here.
 *   - The first call in a device's context looks up the array's device address
 *     (with that device current) and caches it, tagged with the context, so a
 *     context created again after cudaDeviceReset gets a fresh lookup; make
 *     that first call before any stream capture.
 *   - The function itself allocates nothing: no cudaMalloc, no cudaFree, no
 *     allocating library routine.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls whose work may
 *     overlap on the GPU (different streams, or several host threads) race on
 *     it: serialise them, or use liger_attn_prefill with separate workspaces.
 */
#define LIGER_PREFILL_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
liger_status liger_attn_prefill_noalloc(const void* q, const void* k, const void* v, void* out,
                                        float* final_state, int B, int Hq, int Hkv, int T, int d, int w,
                                        float alpha, liger_dtype dt, const float* initial_state,
                                        const int32_t* cu_seqlens, int n_seqs, void* swa_ring_out,
                                        int32_t* pos_out, void* stream);

/*
 * Status of the last liger_attn_prefill_noalloc call on the current device, as
 * liger_attn_prefill_status reports it for a workspace: LIGER_ERR_TIMEOUT
 * (with the site in liger_last_error()) if one of its kernels gave up on a
 * bounded wait, LIGER_OK otherwise.  Reads the scratch header with a
 * synchronous copy: call it after that call's stream has completed.  (No
 * counterpart on the pages; failure detection.)
 */
liger_status liger_attn_prefill_noalloc_status(void);

/*
 * Diagnostic options (no counterpart on the pages), read from the environment
 * once, when the library is loaded; later changes have no effect:
 *   LIGER_PREFILL_PATH=general   every prefill takes the general (CUDA-core) kernel
 *   LIGER_WAIT_LIMIT_NS=<n>      give-up time of each bounded wait (default 2 s)
 *   LIGER_TEST_INJECT_STALL=<n>  the first n tensor-core prefill calls of the
 *                                process withhold one internal completion, so
 *                                that a bounded wait runs out and the call
 *                                reports LIGER_ERR_TIMEOUT (for testing failure
 *                                detection without a GPU fault); later calls
 *                                run normally
 */

/*
 * The gated recurrent branch with one gate per key dimension (a vector gate;
 * Paper-Notes page, section 统一的门控线性循环框架: Liger adapts to
 * GLA, Mamba2, mLSTM, HGRN2 and RWKV6 through the form of the gate G_t in
 * S_t = G_t (.) S_{t-1} + phi(k_t)^T v_t).  The pooling of the key is taken per
 * element: G_t[r] = sigmoid(k_t[r]) scales row r (key dimension) of the state,
 * as GLA's diagonal gate does; the window branch and the mix are unchanged.
 * Arguments, layouts and errors as liger_attn_prefill / liger_attn_decode.  The
 * prefill runs on the CUDA cores in fp32, split into segments of 256 tokens that
 * are processed in parallel after a scan over the segments' states; workspace
 * is device scratch of at least liger_attn_prefill_vector_gate_workspace_size()
 * bytes (16-byte aligned; a smaller one is LIGER_ERR_INVALID_ARG), owned by the
 * caller and not read after the call's kernels end.  Supported: d in {64, 128},
 * bf16 or fp32, w <= 64, any group size.
 */
size_t liger_attn_prefill_vector_gate_workspace_size(int B, int Hq, int Hkv, int T, int d, int n_seqs,
                                                     liger_dtype dt);
liger_status liger_attn_prefill_vector_gate(const void* q, const void* k, const void* v, void* out,
                                            float* final_state, int B, int Hq, int Hkv, int T, int d, int w,
                                            float alpha, liger_dtype dt, const float* initial_state,
                                            const int32_t* cu_seqlens, int n_seqs, void* swa_ring_out,
                                            int32_t* pos_out, void* workspace, size_t workspace_bytes,
                                            void* stream);
liger_status liger_attn_decode_vector_gate(const void* q, const void* k, const void* v, float* state,
                                           void* swa_ring, void* out, int32_t* pos, int B, int Hq, int Hkv,
                                           int d, int w, float alpha, liger_dtype dt, void* stream);

/*
 * Gradient of liger_attn_prefill (bf16 tensor-core path).  The pages give no
 * backward pass; the linearisation fine-tune of the news article on Liger
 * (section "軽量ファインチューニング": LoRA on the Q/K/V projections, trained
 * with next-token cross-entropy through this layer) needs one.  For the loss
 * L = sum(d_out * out) + sum(d_final_state * final_state) of the prefill with
 * the same q, k, v, w, alpha, cu_seqlens and initial state:
 *   dq           [B, T, Hq, d]  bf16  (out)  dL/dq
 *   dk, dv       [B, T, Hkv, d] bf16  (out)  dL/dk, dL/dv (summed over each group's q heads)
 *   d_out        [B, T, Hq, d]  bf16  (in)
 *   d_final_state[n, Hq, d, d]  fp32  (in, nullable = zero)
 *   initial_state[n, Hkv, d, d] fp32  (in, nullable = zero) the initial state as the
 *                recurrence carries it, one per (sequence, kv head); a per-q-head
 *                state whose G copies are equal (as every final_state is) passes as
 *                its first copy of each group.
 *   d_initial_state [n, Hkv, d, d] fp32 (out, nullable) dL/d initial_state (the sum
 *                over the group's heads of the per-head gradients).
 *   workspace    liger_attn_prefill_backward_workspace_size() bytes of device scratch.
 * Supported: bf16, d in {64, 128}, w = 64, even Hq/Hkv (else LIGER_ERR_UNSUPPORTED).
 * Every internal wait is bounded; liger_attn_prefill_status(workspace, bytes)
 * reports a timeout as for the forward.
 */
size_t liger_attn_prefill_backward_workspace_size(int B, int Hq, int Hkv, int T, int d, int n_seqs,
                                                  liger_dtype dt);
liger_status liger_attn_prefill_backward(const void* q, const void* k, const void* v, const void* d_out,
                                         const float* d_final_state, const float* initial_state, int B, int Hq,
                                         int Hkv, int T, int d, int w, float alpha, liger_dtype dt,
                                         const int32_t* cu_seqlens, int n_seqs, void* dq, void* dk, void* dv,
                                         float* d_initial_state, void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * Causal softmax attention: the standard attention layer of the inter-layer
 * hybrid (news article on Liger, section "ハイブリッドメカニズム": one full
 * softmax attention layer after every seven Liger layers; Paper-Notes page,
 * section "Liger 整体架构").  Per query head h with kv head h / (Hq/Hkv):
 *   o_t = sum_{j <= t} softmax_j(q_t . k_j / sqrt(d)) v_j   within each sequence.
 *
 *   q, out  [B, T, Hq, d]  bf16;  k, v  [B, T, Hkv, d]  bf16
 *   cu_seqlens [n + 1] int32 (device, nullable) packed sequences as for the
 *           prefill (then B == 1 and n = n_seqs; otherwise n_seqs == B);
 *   max_seqlen  the longest sequence (read only with cu_seqlens; it sizes the
 *           grid, so it must be at least every sequence's length).
 * Supported: bf16, d in {64, 128}.  fp32 returns LIGER_ERR_UNSUPPORTED.  Every
 * internal wait is bounded (as for the prefill); liger_attn_full_causal_status()
 * reports whether any call on the current device gave up since the last query
 * (synchronous read; call it after the stream has completed; it clears the report).
 */
liger_status liger_attn_full_causal(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                                    int Hkv, int T, int d, liger_dtype dt, const int32_t* cu_seqlens, int n_seqs,
                                    int max_seqlen, void* stream);
liger_status liger_attn_full_causal_status(void);

/* Message of the last failure on the calling thread ("" if none). */
const char* liger_last_error(void);

/*
 * Measurement hooks (no counterpart on the pages; they serve the roofline
 * measurement).  liger_set_timing_events(start, stop) takes two cudaEvent_t
 * (or NULL, NULL to switch off); while set, every later prefill or decode call
 * on the calling thread records `start` just before and `stop` just after its
 * dominant kernel (the prefill's chunk pass, the decode's state stream) on the
 * call's stream.  liger_kernel_launches() returns how many kernels the calling
 * thread has launched through this library so far (launches captured into a
 * CUDA graph are counted once, at capture).
 */
void liger_set_timing_events(void* start_event, void* stop_event);
uint64_t liger_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* LIGER_ATTN_H */
