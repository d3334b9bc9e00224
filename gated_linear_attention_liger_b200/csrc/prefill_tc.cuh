// prefill_tc.cuh -- bf16 chunked prefill on the sm_100a tensor cores.
//
// The recurrence S_t = g_t S_{t-1} + phi(k_t)^T v_t, o_t = phi(q_t) S_t and the
// 64-token window ("Liger: Linearizing Large Language Models to Gated Recurrent
// Structures", Paper-Notes page, sections 统一的门控线性循环框架 and Liger
// Attention) are evaluated in 64-token chunks: inside a chunk the recurrence is
// unrolled into decay-masked dense products, across chunks only the d x d fp32
// state is carried.  With b_i the running sum of log g inside a chunk (b_C at
// its last token) and S the state entering the chunk:
//   grm_i  = e^{b_i} phi(q_i) S + sum_{j<=i} e^{b_i-b_j} (phi(q_i).phi(k_j)) v_j
//   S_next = e^{b_C} S + sum_j (e^{b_C-b_j} phi(k_j))^T v_j
// Every exponent is a difference of running sums taken later-minus-earlier,
// so it is <= 0 and cannot overflow however small the gates are.
//
// Work split (one GPU), launches chained with programmatic dependent launch:
//   plan      : segment table from the sequence offsets (device side, so the
//               launch needs no host synchronisation).
//   seg_state : per (sub-segment, kv head) the state it adds from a zero start,
//               dS = sum over its chunks, and its total log decay.
//   scan      : per (sequence, kv head) the state entering each segment, folded
//               from the sub-segment contributions in order.
//   chunk     : per (segment, pair of q heads of one kv head) the fused pass.
//               Its prologue loads the entering state into TMEM; after the last
//               chunk of a sequence it writes the final state.  TMA stages q/k/v
//               chunks and the state pass's key-tile images; an 8-warp feature
//               group computes e_q, the bf16 state copy for the readout and, one
//               chunk behind, scales and stores the output; four window warps run
//               the window softmax and the recurrent probability tile on TMEM rows;
//               one thread issues the tcgen05 MMAs:
//                 Ss = Q [K_slot0 | K_slot1]^T   raw scores of the window band
//                 Sg = e_Q (e^{b_C-b_j} phi(K))^T recurrent scores (e_Q phi(K)^T when
//                                                the decay does not factor)
//                 O  = e_Q (e^{b_C} S)           inter-chunk readout (e^{b_i} e_Q and S
//                                                when the decay does not factor)
//                 S += (e^{b_C-b_j} phi(K))^T V  state carry (fp32, in TMEM)
//                 O += P_prev V_prev + P_cur V_cur + A_grm V_cur
//               (P and A_grm are written to TMEM and read from there as the A
//               operand); e_Q (which also carries alpha) holds unnormalised
//               exponentials, their sums and the row factor e^{b_i - b_C} of the
//               decay are folded into per-row scalars, and the output is stored as
//               bf16 rows.
// Rows of the MMA tile interleave the two heads: row = 2 * token + head, which
// is exactly the order a TMA box over (d, head, token) produces.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "liger_attn.h"
#include "sm100.cuh"

namespace liger {
namespace tc {

using namespace liger::sm100;

constexpr int C = 64;             // tokens per chunk
constexpr int ROWS = 128;         // MMA M: two heads x 64 tokens
constexpr int kSegThreads = 320;  // state pass: warps 0-7 rows, warp 8 TMA, warp 9 MMA
constexpr uint64_t kDefaultWaitNs = 2000000000ull;   // 2 s per wait

struct SegInfo {
  int32_t seq, t_begin, t_end, q0;   // tokens [t_begin, t_end) of the sequence starting at q0
};
struct SeqInfo {
  int32_t first_seg, n_seg;
};

struct PrefillProblem {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* final_state;
  const float* s0;       // initial state [n, Hq, D, D] or null
  const int32_t* cu;
  int B, Hq, Hkv;
  long T;
  int d, n_seqs;
  float alpha;
};

// Workspace layout (bytes from its start).
struct Plan {
  int L;            // chunks per segment
  int n_seg_max;    // upper bound on segments
  int nsub, Ls;     // sub-segments per segment for the state pass, and their length in chunks
  size_t off_seqs, off_segs, off_lam, off_ds, off_kimg, off_bimg, off_flags, total;
};

// Largest total log gate of a chunk for which its decay is factored at the chunk end
// (both factors then lie within e^{+-60}); the state pass and the chunk pass take the
// same decision from the same stored sum.
constexpr float kFactorFloor = -60.f;

constexpr int kMaxSub = 8;

struct DevParams {
  const SegInfo* segs;
  const SeqInfo* seqs;
  const int32_t* n_segs;
  float* lam;            // [n_seg_max][nsub][Hkv] total log gate of each sub-segment
  float* ds;             // [n_seg_max][nsub][Hkv][D][D]: state each sub-segment adds from a zero
                         // start; the scan replaces [s][0] by the state entering segment s
  char* kimg;            // [n_seg_max * L][Hkv]: per chunk, the chunk pass's key tile as a
                         // shared-memory image (C x D bf16, 128-byte swizzle, K-major blocks):
                         // e^{b_C - b_j} phi(k_j) when the decay factors (b_C >= -60), else phi(k_j)
  float* bimg;           // [n_seg_max * L][Hkv][C]: per chunk, the running log-gate sums b_j
                         // (constant past the chunk's last valid token)
  uint32_t* err;
  void* out;
  float* final_state;
  const float* s0;       // [n][Hq][D][D] initial states or null: the scan starts each group from
                         // its first head's copy
  uint32_t* s0_flags;    // [n][Hkv]: set when the G copies of a group's initial state differ
  const int32_t* cu;
  long T, NT;
  int Hq, Hkv, n_seqs, n_seg_max, L, nsub, Ls;
  float alpha;
  uint64_t wait_ns;
  int out_v8;            // out is 32-byte aligned: 256-bit stores
  int inject_stall;      // test switch: withhold one MMA completion so a wait runs out
};

// ============================================================== plan kernel

__global__ void plan_kernel(DevParams p, SeqInfo* seqs, SegInfo* segs, int32_t* n_segs) {
  griddep_wait_and_release();   // the previous call's kernels are done with the workspace
  if (p.s0)
    for (int i = threadIdx.x; i < p.n_seqs * p.Hkv; i += blockDim.x) p.s0_flags[i] = 0u;
  if (threadIdx.x != 0) return;
  p.err[0] = 0u;
  p.err[1] = 0u;
  int seg = 0;
  const long span = (long)C * p.L;
  for (int s = 0; s < p.n_seqs; ++s) {
    long q0, q1;
    seq_range(p.cu, s, p.T, p.NT, &q0, &q1);
    const long len = q1 - q0;
    const int nseg = (int)((len + span - 1) / span);
    if (seg + nseg > p.n_seg_max) {   // cannot happen with the host's bound; fail safe
      atomicOr(p.err, 2u);
      seqs[s] = SeqInfo{seg, 0};
      continue;
    }
    seqs[s] = SeqInfo{seg, nseg};
    for (int i = 0; i < nseg; ++i) {
      const long b = q0 + i * span;
      const long e = b + span < q1 ? b + span : q1;
      segs[seg++] = SegInfo{s, (int32_t)b, (int32_t)e, (int32_t)q0};
    }
  }
  *n_segs = seg;
}

// Final state of the sequences that have no token (packed input only): the initial
// state of that head, or zero.  Grid (n_seqs, Hq), 256 threads.
template <int D>
__global__ void zero_empty_kernel(DevParams p) {
  griddep_wait_and_release();
  if (p.seqs[blockIdx.x].n_seg != 0) return;
  const size_t off = ((size_t)blockIdx.x * p.Hq + blockIdx.y) * D * D;
  float4* dst = reinterpret_cast<float4*>(p.final_state + off);
  const float4* src = p.s0 ? reinterpret_cast<const float4*>(p.s0 + off) : nullptr;
  for (int e = threadIdx.x; e < D * D / 4; e += blockDim.x) dst[e] = src ? src[e] : make_float4(0.f, 0.f, 0.f, 0.f);
}

// 32 bytes to global memory in one store (the address must be 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* ptr, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(ptr), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// Per (sequence, kv head): folds the sub-segment contributions in order and
// stores the state entering each segment in its first sub-segment slot.  Grid
// (n_seqs * Hkv, D*D / 1024), 256 threads x 4 floats.
template <int D>
__global__ void scan_kernel(DevParams p) {
  griddep_wait_and_release();
  const int seq = blockIdx.x / p.Hkv, kv = blockIdx.x % p.Hkv;
  const size_t e = ((size_t)blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (e >= (size_t)D * D) return;
  const SeqInfo si = p.seqs[seq];
  const int nsub = p.nsub;
  // The sequence's sub-segment contributions in order, 20 loads in flight at a
  // time; the state entering a segment is stored over its first sub-segment's slot
  // (after that slot has been read).
  constexpr int kBatch = 20;
  const int n_units = si.n_seg * nsub;
  const size_t u0 = (size_t)si.first_seg * nsub;
  float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
  if (p.s0) {
    // The recurrence is linear in its start: every head of the group runs from the group's
    // first copy of the initial state.  When another head's copy differs, the group is
    // flagged and recomputed by the general kernel after the chunk pass.
    const int G = p.Hq / p.Hkv;
    const float* s0g = p.s0 + ((size_t)seq * p.Hq + (size_t)kv * G) * D * D + e;
    run = *reinterpret_cast<const float4*>(s0g);
    bool differ = false;
    for (int g = 1; g < G; ++g) {
      const float4 o = *reinterpret_cast<const float4*>(s0g + (size_t)g * D * D);
      differ |= __float_as_uint(o.x) != __float_as_uint(run.x) || __float_as_uint(o.y) != __float_as_uint(run.y) ||
                __float_as_uint(o.z) != __float_as_uint(run.z) || __float_as_uint(o.w) != __float_as_uint(run.w);
    }
    if (differ) atomicOr(p.s0_flags + (size_t)seq * p.Hkv + kv, 1u);
  }
  for (int base = 0; base < n_units; base += kBatch) {
    float4 d[kBatch];
    float g[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (base + k < n_units) {
        const size_t u = u0 + base + k;
        d[k] = __ldcs(reinterpret_cast<const float4*>(p.ds + (u * p.Hkv + kv) * D * D + e));
        g[k] = __expf(p.lam[u * p.Hkv + kv]);
      }
    }
    int rr = base % nsub;   // sub-segment index of unit base + k
#pragma unroll
    for (int k = 0; k < kBatch; ++k, rr = rr + 1 == nsub ? 0 : rr + 1) {
      if (base + k < n_units) {
        if (rr == 0) *reinterpret_cast<float4*>(p.ds + ((u0 + base + k) * p.Hkv + kv) * D * D + e) = run;
        run = make_float4(fmaf(g[k], run.x, d[k].x), fmaf(g[k], run.y, d[k].y), fmaf(g[k], run.z, d[k].z),
                          fmaf(g[k], run.w, d[k].w));
      }
    }
  }
}

// ============================================================== row helpers

// Element e (0..D-1) of 128-byte-swizzled row `row` in a K-major tile whose
// 64-element blocks are `block_stride` bytes apart.
__device__ __forceinline__ uint32_t kmajor_off(int row, int e, uint32_t block_stride) {
  return (uint32_t)(e >> 6) * block_stride + sw128(row, (e & 63) >> 3) + (uint32_t)((e & 7) << 1);
}

// Load 8 bf16 (one 16-byte chunk) as floats.
__device__ __forceinline__ void ld_chunk8(const char* base, uint32_t off, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(base + off);
  x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
  x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
  x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z);
  x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}
__device__ __forceinline__ void st_chunk8(char* base, uint32_t off, const float* x) {
  uint4 u;
  u.x = pack_bf16(x[0], x[1]);
  u.y = pack_bf16(x[2], x[3]);
  u.z = pack_bf16(x[4], x[5]);
  u.w = pack_bf16(x[6], x[7]);
  *reinterpret_cast<uint4*>(base + off) = u;
}

// Running sums of the log gates of one chunk: lane l of every warp of the group
// holds the sums up to tokens 2l and 2l+1; b_at() fetches token x's sum.
struct GateSums {
  float b0, b1;
  __device__ __forceinline__ float at(int x) const {
    const float v0 = __shfl_sync(0xffffffffu, b0, x >> 1);
    const float v1 = __shfl_sync(0xffffffffu, b1, x >> 1);
    return (x & 1) ? v1 : v0;
  }
};

// log sigmoid(m) = -softplus(-m) with the fast exp/log units (no overflow either side).
__device__ __forceinline__ float log_sigmoid_fast(float m) {
  const float t = __logf(1.0f + __expf(-fabsf(m)));
  return fminf(m, 0.f) - t;
}

// Largest log2 spread max - shift of a row whose exponentials are taken against a
// shift other than its maximum: values stay below 2^24, leaving fp32 and bf16 headroom
// for the per-row and per-key factors applied later.
constexpr float kShiftSpan = 24.f;

// Feature map and gate of one chunk of keys, shared by the seg_state and chunk
// kernels.  TPT threads (2 or 4, adjacent lanes) share a key token: thread r owns
// elements [h D/TPT, (h+1) D/TPT) of token j = r / TPT, h = r % TPT, and the group
// is 64 TPT threads.  Computes e = exp(k - shift) (bf16, not yet divided by its sum;
// the shift cancels once the sum is divided out), keeps this thread's values packed
// in ek and writes them to `ebuf` (if not null) in the key tile's swizzled layout;
// writes the log gates to lg[0..63] (0 past the valid tokens); returns 1 / sum_d e,
// which the callers fold into per-token scalars, and the running sums in gs (every
// warp scans the 64 gates itself); lanes of the group's first warp also store the
// sums to bsh.  The loops run over 16-byte groups and stay short: the role loops of
// the chunk kernel share one SM sub-partition, and long straight-line code for all
// of them would not stay in the instruction caches.
template <int D, int TPT = 2, uint32_t KSTRIDE = C * 128>   // KSTRIDE: byte stride of the raw tile's 64-element blocks
__device__ __forceinline__ float key_features(const char* kraw, char* ebuf, float* lg, float* bsh, int r, int nv,
                                              GateSums& gs, uint32_t (&ek)[D / TPT / 2]) {
  constexpr int PART = D / TPT;
  constexpr float kLog2e = 1.4426950408889634f;
  const int j = r / TPT, h = r % TPT;
  // One pass: raw sum (for the gate), maximum, and e = exp(k - k_0) with k_0 the
  // token's first element.  Any shift leaves the normalised features unchanged; the
  // maximum is needed only when the token's spread would leave too little fp32
  // headroom, and then the exponentials are redone against it.
  const float sl = bf16_lo(*reinterpret_cast<const uint32_t*>(kraw + kmajor_off(j, 0, KSTRIDE))) * kLog2e;
  float m = -INFINITY, sa = 0.f, sb = 0.f, za = 0.f, zb = 0.f;
#pragma unroll
  for (int c = 0; c < PART / 8; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(kraw + kmajor_off(j, h * PART + c * 8, KSTRIDE));
    m = fmaxf(m, bf16x8_max(u));
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
    float x[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) { x[2 * q] = bf16_lo(w4[q]); x[2 * q + 1] = bf16_hi(w4[q]); }
    sa += (x[0] + x[1]) + (x[2] + x[3]);
    sb += (x[4] + x[5]) + (x[6] + x[7]);
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = ex2(fmaf(x[q], kLog2e, -sl));
    za += (x[0] + x[1]) + (x[2] + x[3]);
    zb += (x[4] + x[5]) + (x[6] + x[7]);
#pragma unroll
    for (int q = 0; q < 4; ++q) ek[4 * c + q] = pack_bf16(x[2 * q], x[2 * q + 1]);
    if (ebuf)
      *reinterpret_cast<uint4*>(ebuf + kmajor_off(j, h * PART + c * 8, C * 128)) =
          make_uint4(ek[4 * c], ek[4 * c + 1], ek[4 * c + 2], ek[4 * c + 3]);
  }
  float sum = sa + sb, z = za + zb;
#pragma unroll
  for (int o = 1; o < TPT; o <<= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    z += __shfl_xor_sync(0xffffffffu, z, o);
  }
  // The redo is decided per token (the same on all its lanes) but entered by the whole
  // warp, so that the shuffles below always see every lane.
  const bool redo = m * kLog2e - sl > kShiftSpan;
  if (__any_sync(0xffffffffu, redo)) {
    float zr = 0.f;
    if (redo) {
      const float ml = m * kLog2e;
      za = 0.f;
      zb = 0.f;
#pragma unroll
      for (int c = 0; c < PART / 8; ++c) {
        float x[8];
        ld_chunk8(kraw, kmajor_off(j, h * PART + c * 8, KSTRIDE), x);
#pragma unroll
        for (int q = 0; q < 8; ++q) x[q] = ex2(fmaf(x[q], kLog2e, -ml));
        za += (x[0] + x[1]) + (x[2] + x[3]);
        zb += (x[4] + x[5]) + (x[6] + x[7]);
#pragma unroll
        for (int q = 0; q < 4; ++q) ek[4 * c + q] = pack_bf16(x[2 * q], x[2 * q + 1]);
        if (ebuf)
          *reinterpret_cast<uint4*>(ebuf + kmajor_off(j, h * PART + c * 8, C * 128)) =
              make_uint4(ek[4 * c], ek[4 * c + 1], ek[4 * c + 2], ek[4 * c + 3]);
      }
      zr = za + zb;
    }
#pragma unroll
    for (int o = 1; o < TPT; o <<= 1) zr += __shfl_xor_sync(0xffffffffu, zr, o);
    if (redo) z = zr;
  }
  if (h == 0) lg[j] = j < nv ? log_sigmoid_fast(sum / (float)D) : 0.f;
  named_bar(1, 64 * TPT);
  {   // inclusive running sum over the 64 tokens, two per lane, in every warp
    const int lane = r & 31;
    const float a0 = lg[2 * lane], a1 = lg[2 * lane + 1];
    float s = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float t = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += t;
    }
    const float before = s - a0 - a1;
    gs.b0 = before + a0;
    gs.b1 = before + a0 + a1;
    if (r < 32 && bsh) {
      bsh[2 * r] = gs.b0;
      bsh[2 * r + 1] = gs.b1;
    }
  }
  return 1.0f / z;
}

// Decay-scaled keys sc * e (sc = e^{b_C - b_j} / z_j, zero past the valid tokens), from
// this thread's packed features ek (as key_features stored them) to `kt` in the key
// tile's swizzled layout (thread layout as in key_features); read by the MMA as the
// MN-major A operand K^T.
template <int D, int TPT = 2>
__device__ __forceinline__ void write_ktilde(const uint32_t (&ek)[D / TPT / 2], char* kt, int r, float sc) {
  constexpr int PART = D / TPT;
  const int j = r / TPT, h = r % TPT;
#pragma unroll
  for (int c = 0; c < PART / 8; ++c) {
    float x[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      x[2 * q] = bf16_lo(ek[4 * c + q]) * sc;
      x[2 * q + 1] = bf16_hi(ek[4 * c + q]) * sc;
    }
    st_chunk8(kt, kmajor_off(j, h * PART + c * 8, C * 128), x);
  }
}

// ============================================================== seg_state kernel

template <int D>
struct SegSmem {
  static constexpr uint32_t KV = C * D * 2;        // one chunk of k (or v)
  // key ring (2 slots, released by the row warps once the features are out), value
  // ring (2 slots, released by the MMA), decay-scaled keys (2 slots)
  static constexpr uint32_t K0 = 0, V0 = 2 * KV, KT = 4 * KV, SMALL = 6 * KV;
  static constexpr uint32_t BYTES = SMALL + 1024 + 1024;   // + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kSegThreads, 2)
    seg_state_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     DevParams p) {
  griddep_wait_and_release();
  using L = SegSmem<D>;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::SMALL);
  uint64_t* k_full = bars;         // [2]
  uint64_t* img_ready = bars + 2;  // [2] the chunk's key image written over its raw keys (256 arrivals)
  uint64_t* v_full = bars + 4;     // [2]
  uint64_t* v_empty = bars + 7;    // [2]
  uint64_t* feat = bars + 10;
  uint64_t* mma_done = bars + 11;  // [2], per keys~ slot
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never = tmem_slot + 2;          // stays 0: drain waits ignore aborts
  float* lg = reinterpret_cast<float*>(bars + 16);   // 64 floats

  const int unit = blockIdx.x / p.Hkv, kv = blockIdx.x % p.Hkv;
  const int seg = unit / p.nsub, sub = unit % p.nsub;
  if (seg >= *p.n_segs) return;
  const SegInfo sg0 = p.segs[seg];
  const int nch_seg = (sg0.t_end - sg0.t_begin + C - 1) / C;
  const int c_lo = sub * p.Ls, c_hi = min(c_lo + p.Ls, nch_seg);
  float* const ds_out = p.ds + ((size_t)unit * p.Hkv + kv) * D * D;
  if (c_lo >= c_hi) {   // an empty sub-segment adds nothing
    for (int e = threadIdx.x; e < D * D / 4; e += blockDim.x)
      reinterpret_cast<float4*>(ds_out)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x == 0) p.lam[(size_t)unit * p.Hkv + kv] = 0.f;
    return;
  }
  SegInfo sg = sg0;   // this CTA's tokens
  sg.t_begin = sg0.t_begin + c_lo * C;
  sg.t_end = min(sg0.t_end, sg0.t_begin + c_hi * C);
  const int nch = c_hi - c_lo;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t TCOLS = D < 32 ? 32 : D;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(&k_full[i], 1); mbar_init(&img_ready[i], 256); }
    for (int i = 0; i < 2; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    mbar_init(feat, 256); mbar_init(&mma_done[0], 1); mbar_init(&mma_done[1], 1); mbar_init(drain, 1);
    *abort_flag = 0u;
    *never = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err, p.wait_ns};

  if (warp == 8) {   // ---------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      // The key image of step c is written by the row warps over step c's raw keys; this
      // thread stores it to the workspace in one bulk copy and then refills the slot.
      auto store_img = [&](int c) {
        const size_t ci = (size_t)(seg * p.L + sub * p.Ls + (nch - 1 - c)) * p.Hkv + kv;
        bulk_store(p.kimg + ci * L::KV, smem + L::K0 + (c & 1) * L::KV, L::KV);
        bulk_commit();
      };
      int k_issued = 0, v_issued = 0, stored = 0;
      for (int c = 0; c < nch; ++c) {   // step c handles chunk nch - 1 - c (last to first)
        const int t = sg.t_begin + (nch - 1 - c) * C;
        const int ks = c & 1, vs = c & 1;
        if (c >= 2) {
          if (!mbar_wait(&img_ready[ks], ((c >> 1) - 1) & 1, wc)) break;
          store_img(c - 2);
          stored = c - 1;
          bulk_wait_read_all();   // the slot's image is read out: it may take the next keys
        }
        mbar_arrive_expect_tx(&k_full[ks], L::KV);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(smem + L::K0 + ks * L::KV + kb * C * 128, &tmk, &k_full[ks], kb * 64, kv, t);
        k_issued = c + 1;
        if (c >= 2 && !mbar_wait(&v_empty[vs], ((c >> 1) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&v_full[vs], L::KV);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(smem + L::V0 + vs * L::KV + kb * C * 128, &tmv, &v_full[vs], kb * 64, kv, t);
        v_issued = c + 1;
      }
      // the images of the last steps
      for (int c = stored; c < k_issued; ++c) {
        if (!mbar_wait(&img_ready[c & 1], (c >> 1) & 1, wc)) break;
        store_img(c);
      }
      bulk_wait_all();   // the images are in the workspace before the CTA ends
      // never leave the CTA with copies in flight
      const WaitCtx dw{never, nullptr, p.wait_ns};
      for (int c = (k_issued > 2 ? k_issued - 2 : 0); c < k_issued; ++c) mbar_wait(&k_full[c & 1], (c >> 1) & 1, dw);
      for (int c = (v_issued > 2 ? v_issued - 2 : 0); c < v_issued; ++c) mbar_wait(&v_full[c & 1], (c >> 1) & 1, dw);
    }
  } else if (warp == 9) {   // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, D, 1, 1);
      const uint32_t lbo_a = D == 128 ? C * 128 : 0;   // d = 64: both M halves read the same block
      for (int c = 0; c < nch; ++c) {
        const int vs = c & 1;
        if (!mbar_wait(&v_full[vs], (c >> 1) & 1, wc)) break;
        if (!mbar_wait(feat, c & 1, wc)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t a = sdesc_sw128(smem_u32(smem + L::KT + (c & 1) * L::KV) + kk * 2048, lbo_a, 1024);
          const uint64_t b = sdesc_sw128(smem_u32(smem + L::V0 + vs * L::KV) + kk * 2048, C * 128, 1024);
          mma_bf16_ss(tmem, a, b, idesc, (c > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&mma_done[c & 1]);
        mma_commit(&v_empty[vs]);
      }
      mma_commit(drain);
    }
  } else {   // ---------------- rows (threads 0..255: four per key token; warps w and w + 4
             // share TMEM lanes 32 (w & 3) .. and split the state's columns)
    const int r = threadIdx.x;
    const int row = r & 127, half = warp >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    // The chunks are taken last to first, so the decay from a chunk to the end of the
    // sub-segment (lam, the sum of the later chunks' totals) is known when it is
    // processed: its keys~ carry it, e^{lam + b_C - b_j} phi(k_j) (exponent <= 0), and
    // the products accumulate onto dS with no rescale in between.
    float lam = 0.f;
    // Row threads never leave the loop early: after a timeout every wait returns
    // at once (the CTA's abort flag is set), so all rows still meet at each
    // named barrier and warp-collective TMEM access stays uniform.
    for (int c = 0; c < nch; ++c) {
      const int slot = c & 1;
      const int cc = nch - 1 - c;
      const int nv = min(C, sg.t_end - (sg.t_begin + cc * C));
      mbar_wait(&k_full[slot], (c >> 1) & 1, wc);
      GateSums gs;
      uint32_t ek[D / 8];
      // (key_features ends with a barrier of the group after its last read of the raw keys)
      const float iz = key_features<D, 4>(smem + L::K0 + slot * L::KV, nullptr, lg, nullptr, r, nv, gs, ek);
      const float bC = gs.at(nv - 1);
      const float bj = gs.at(r >> 2);
      const bool live = (r >> 2) < nv;
      // The chunk pass's key tile for this chunk (written once, read by its q-head
      // pairs): factored at the chunk end when the chunk's decay allows, else phi(k).  It
      // goes over the raw keys in shared memory, and the TMA warp stores it in one bulk copy.
      {
        const size_t ci = (size_t)(seg * p.L + sub * p.Ls + cc) * p.Hkv + kv;
        const float sc = live ? (bC >= kFactorFloor ? __expf(bC - bj) * iz : iz) : 0.f;
        write_ktilde<D, 4>(ek, smem + L::K0 + slot * L::KV, r, sc);
        fence_proxy_async_smem();
        mbar_arrive(&img_ready[slot]);
        if (r < 32) {
          p.bimg[ci * C + 2 * r] = gs.b0;
          p.bimg[ci * C + 2 * r + 1] = gs.b1;
        }
      }
      if (c >= 2) {   // the product two steps back is done with this keys~ slot
        mbar_wait(&mma_done[slot], ((c >> 1) - 1) & 1, wc);
        tc_fence_after();
      }
      write_ktilde<D, 4>(ek, smem + L::KT + slot * L::KV, r, live ? __expf(lam + bC - bj) * iz : 0.f);
      lam += bC;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(feat);
      named_bar(1, 256);   // lg is rewritten by the next chunk
    }
    if (nch > 0 && warp_all(mbar_wait(&mma_done[(nch - 1) & 1], ((nch - 1) >> 1) & 1, wc) && !*abort_flag)) {
      tc_fence_after();
      float* dst = ds_out + (size_t)row * D;
#pragma unroll 1
      for (int col = half * (D / 2); col < (half + 1) * (D / 2); col += 32) {
        float v[32];
        tmem_ld32(lane_base + col, v);
        tmem_wait_ld();
        if (row < D) {
#pragma unroll
          for (int u = 0; u < 32; u += 4)
            *reinterpret_cast<float4*>(dst + col + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
        }
      }
      if (r == 0) p.lam[(size_t)unit * p.Hkv + kv] = lam;
    }
  }
  __syncthreads();
  if (warp == 0) {
    mbar_wait(drain, 0, WaitCtx{never, nullptr, p.wait_ns});
    tc_fence_after();
    tmem_dealloc(tmem, TCOLS);
  }
}

// ============================================================== chunk kernel

// Rows of the state entering segment `seg` (columns [c0, c0 + NC)) from the scan's
// output, stored to TMEM.
template <int D, int NC>
__device__ __forceinline__ void entering_state(const DevParams& p, int seg, int kv, int row, uint32_t taddr,
                                               int c0) {
  static_assert(NC % 16 == 0, "columns come in groups of 16");
  const float* src = p.ds + (((size_t)seg * p.nsub * p.Hkv + kv) * D + row) * D;
#pragma unroll 1
  for (int col = c0; col < c0 + NC; col += 16) {
    float v[16];
#pragma unroll
    for (int u = 0; u < 16; u += 4) {
      const float4 x = *reinterpret_cast<const float4*>(src + col + u);
      v[u] = x.x; v[u + 1] = x.y; v[u + 2] = x.z; v[u + 3] = x.w;
    }
    tmem_st16(taddr + col, v);
  }
  tmem_wait_st();
}

template <int D>
struct ChunkSmem {
  static constexpr uint32_t QB = ROWS * D * 2;    // q tile (two heads): raw q, then scaled phi(q)
  static constexpr uint32_t KV = C * D * 2;       // one chunk of k or v
  static constexpr uint32_t Q0 = 0;
  static constexpr uint32_t EQ = Q0 + QB;         // e_q' = alpha exp(q - q_0), bf16
  static constexpr uint32_t K0 = EQ + QB;         // 2 key slots, laid out [64-d block][slot][64 rows]
  static constexpr uint32_t V0 = K0 + 2 * KV;     // 3 value slots
  static constexpr uint32_t KI = V0 + 3 * KV;     // 2 slots of the state pass's key-tile images
  static constexpr uint32_t SB = KI + 2 * KV;     // bf16 copy of the readout's state
  static constexpr uint32_t SMALL = SB + D * D * 2;
  static constexpr uint32_t SMALL_BYTES = 4096;
  static constexpr uint32_t BI = SMALL + 3072;    // 2 slots of the chunks' running log-gate sums
  static constexpr uint32_t BYTES = SMALL + SMALL_BYTES + 1024;   // + alignment slack
};

// TMEM columns of the chunk kernel (fp32 cells, lane = tile row).
constexpr uint32_t kColSs = 0;     // window scores, previous keys then current keys (128)
constexpr uint32_t kColSg = 128;   // recurrent scores (64)
constexpr uint32_t kColP = 192;    // probability tile, bf16 pairs: previous keys, current keys (64)
constexpr uint32_t kColO = 256;    // output accumulator (D); the state follows it (D)

// warps 0-3 window, 4-11 features (and the output), 12 TMA, 13 MMA
constexpr int kFeatWarp0 = 4;
constexpr int kTmaWarp = kFeatWarp0 + 8, kMmaWarp = kTmaWarp + 1;
constexpr int kChunkThreads = 32 * (kMmaWarp + 1);

template <int D>
__global__ void __launch_bounds__(kChunkThreads, 1)
    chunk_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, DevParams p) {
  griddep_wait_and_release();
  using L = ChunkSmem<D>;
  constexpr uint32_t kColS = kColO + D;
  constexpr uint32_t TCOLS = 512;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::SMALL);
  uint64_t* k_full = bars;           // [2]
  uint64_t* k_empty = bars + 2;      // [2]
  uint64_t* v_full = bars + 4;       // [3]
  uint64_t* v_empty = bars + 7;      // [3]
  uint64_t* q_full = bars + 10;
  uint64_t* q_empty = bars + 11;
  uint64_t* ss_done = bars + 12;     // window scores written; raw q read
  uint64_t* feat = bars + 13;        // key and query tiles of the chunk ready (256 arrivals)
  uint64_t* sg_done = bars + 14;     // recurrent scores and state carry done
  uint64_t* mma2_done = bars + 15;   // + readout done: feature buffers free again
  uint64_t* s_read = bars + 16;      // score tiles read out of TMEM (128 arrivals)
  uint64_t* p_ready = bars + 17;     // probability tile in TMEM (128 arrivals)
  uint64_t* o_done = bars + 18;      // output accumulator complete
  uint64_t* o_free = bars + 19;      // output read out (128 arrivals)
  uint64_t* drain = bars + 20;
  uint64_t* state_ready = bars + 22; // state copied, S rescaled (256 arrivals)
  uint64_t* state_done = bars + 23;  // the chunk's state carry done
  uint64_t* kimg_full = bars + 24;   // [2] key-tile image and gate sums landed
  uint64_t* kimg_empty = bars + 26;  // [2] the chunk's products are done with the image slot
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 30);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never = tmem_slot + 2;                     // stays 0: drain waits ignore aborts
  float* bsh2 = reinterpret_cast<float*>(smem + L::SMALL + 256 + 64);  // [2][64] running log-gate sums
  float* zq2 = bsh2 + 128;                                     // [2][128] Z = sum_d e_q per row
  float* fast2 = zq2 + 256;                                     // [2] factored decay usable
  float* osc2 = reinterpret_cast<float*>(smem + L::SMALL + 1920);  // [2][128] output row scales

  const int npairs = p.Hq / 2;
  const int seg = blockIdx.x / npairs, pair = blockIdx.x % npairs;
  if (seg >= *p.n_segs) return;
  const SegInfo sg = p.segs[seg];
  const int G = p.Hq / p.Hkv;
  const int h0 = pair * 2, kv = h0 / G;
  const int nch = (sg.t_end - sg.t_begin + C - 1) / C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < 3; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    mbar_init(q_full, 1); mbar_init(q_empty, 2);
    mbar_init(ss_done, 1); mbar_init(feat, 256); mbar_init(sg_done, 1); mbar_init(mma2_done, 1);
    mbar_init(state_ready, 256); mbar_init(state_done, 1);
    mbar_init(s_read, 128); mbar_init(p_ready, 128); mbar_init(o_done, 1); mbar_init(o_free, 256);
    mbar_init(drain, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(&kimg_full[i], 1); mbar_init(&kimg_empty[i], 1); }
    *abort_flag = 0u;
    *never = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err, p.wait_ns};

  if (warp == kTmaWarp) {   // ---------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      // key / value load u holds tokens t_begin + 64 (u - 1): u = 0 is the chunk before the segment
      auto load_k = [&](int u) {
        const int slot = u & 1;
        mbar_arrive_expect_tx(&k_full[slot], L::KV);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(smem + L::K0 + slot * (C * 128) + kb * (2 * C * 128), &tmk, &k_full[slot], kb * 64, kv,
                      sg.t_begin + (u - 1) * C);
      };
      auto load_v = [&](int u) {
        const int slot = u % 3;
        mbar_arrive_expect_tx(&v_full[slot], L::KV);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(smem + L::V0 + slot * L::KV + kb * C * 128, &tmv, &v_full[slot], kb * 64, kv,
                      sg.t_begin + (u - 1) * C);
      };
      auto load_q = [&](int c) {
        mbar_arrive_expect_tx(q_full, L::QB);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(smem + L::Q0 + kb * ROWS * 128, &tmq, q_full, kb * 64, h0, sg.t_begin + c * C);
      };
      auto load_img = [&](int c) {   // the state pass's key tile and gate sums of chunk c
        const int slot = c & 1;
        const size_t ci = (size_t)(seg * p.L + c) * p.Hkv + kv;
        mbar_arrive_expect_tx(&kimg_full[slot], L::KV + C * 4);
        bulk_load(smem + L::KI + slot * L::KV, p.kimg + ci * L::KV, L::KV, &kimg_full[slot]);
        bulk_load(smem + L::BI + slot * (C * 4), p.bimg + ci * C, C * 4, &kimg_full[slot]);
      };
      int k_issued = 2, v_issued = 2, q_issued = 1, i_issued = 1;
      load_img(0);
      load_k(0); load_v(0);
      load_k(1); load_v(1);
      load_q(0);
      for (int c = 0; c + 1 < nch; ++c) {
        const int u = c + 2;
        if (c >= 1 && !mbar_wait(&kimg_empty[(c + 1) & 1], (((c + 1) >> 1) - 1) & 1, wc, wsite(1, 4, c))) break;
        load_img(c + 1);
        i_issued = c + 2;
        if (!mbar_wait(&k_empty[u & 1], ((u >> 1) - 1) & 1, wc, wsite(1, 1, c))) break;
        load_k(u);
        k_issued = u + 1;
        if (u >= 3 && !mbar_wait(&v_empty[u % 3], (u / 3 - 1) & 1, wc, wsite(1, 2, c))) break;
        load_v(u);
        v_issued = u + 1;
        if (!mbar_wait(q_empty, c & 1, wc, wsite(1, 3, c))) break;
        load_q(c + 1);
        q_issued = c + 2;
      }
      const WaitCtx dw{never, nullptr, p.wait_ns};   // never leave with copies in flight
      for (int u = (k_issued > 2 ? k_issued - 2 : 0); u < k_issued; ++u) mbar_wait(&k_full[u & 1], (u >> 1) & 1, dw);
      for (int u = (v_issued > 3 ? v_issued - 3 : 0); u < v_issued; ++u) mbar_wait(&v_full[u % 3], (u / 3) & 1, dw);
      mbar_wait(q_full, (q_issued - 1) & 1, dw);
      for (int c = (i_issued > 2 ? i_issued - 2 : 0); c < i_issued; ++c) mbar_wait(&kimg_full[c & 1], (c >> 1) & 1, dw);
    }
  } else if (warp == kMmaWarp) {   // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_n64 = idesc_bf16(128, 64, 0, 0);
      const uint32_t id_n128 = idesc_bf16(128, 128, 0, 0);
      const uint32_t id_inter = idesc_bf16(128, D, 0, 1);
      const uint32_t id_state = idesc_bf16(128, D, 1, 1);
      const uint32_t lbo_kt = D == 128 ? C * 128 : 0;   // d = 64: both M halves read the same block
      const uint32_t q_base = smem_u32(smem + L::Q0);
      const uint32_t eq_base = smem_u32(smem + L::EQ);
      const uint32_t ki_base = smem_u32(smem + L::KI);
      const uint32_t sb_base = smem_u32(smem + L::SB);
      bool ok = true;
      auto issue_ss = [&](int c) {   // window scores against the previous and the current keys
        if (c == 0) ok = ok && mbar_wait(&k_full[0], 0, wc, wsite(2, 1, c));
        ok = ok && mbar_wait(&k_full[(c + 1) & 1], ((c + 1) >> 1) & 1, wc, wsite(2, 2, c));
        ok = ok && mbar_wait(q_full, c & 1, wc, wsite(2, 3, c));
        if (c > 0) ok = ok && mbar_wait(s_read, (c - 1) & 1, wc, wsite(2, 4, c));
        if (!ok) return;
        tc_fence_after();
        // both key slots as one 128-row operand: score columns [slot 0 | slot 1], that is
        // [previous | current] for even chunks and [current | previous] for odd ones
        const uint32_t kb = smem_u32(smem + L::K0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_sw128(q_base + (kk >> 2) * (ROWS * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(kb + (kk >> 2) * (2 * C * 128) + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss(tmem + kColSs, a, b, id_n128, kk > 0);
        }
        mma_commit(ss_done);
        mma_commit(q_empty);           // one of the q buffer's two releases (the raw q was read)
        mma_commit(&k_empty[c & 1]);   // the previous chunk's keys are no longer needed
      };
      auto issue_pv = [&](int c) {   // O += P_prev V_prev + P_cur V_cur, P read from TMEM (P_cur holds the recurrent tile too)
        if (c == 0) ok = ok && mbar_wait(&v_full[0], 0, wc, wsite(2, 5, c));
        ok = ok && mbar_wait(p_ready, c & 1, wc, wsite(2, 6, c));
        if (!ok) return;
        tc_fence_after();
        const uint32_t vp = smem_u32(smem + L::V0 + (c % 3) * L::KV);
        const uint32_t vc = smem_u32(smem + L::V0 + ((c + 1) % 3) * L::KV);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t bp = sdesc_sw128(vp + kk * 2048, C * 128, 1024);
          const uint64_t bc = sdesc_sw128(vc + kk * 2048, C * 128, 1024);
          mma_bf16_ts(tmem + kColO, tmem + kColP + kk * 8, bp, id_inter, 1u);        // previous keys
          mma_bf16_ts(tmem + kColO, tmem + kColP + 32 + kk * 8, bc, id_inter, 1u);   // current keys (window + recurrent)
        }
        mma_commit(o_done);
        mma_commit(&v_empty[c % 3]);   // the previous chunk's values are no longer needed
      };
      auto issue_sg_state = [&](int c) {
        // recurrent scores as soon as the feature warps are done
        ok = ok && mbar_wait(&kimg_full[c & 1], (c >> 1) & 1, wc, wsite(2, 11, c));
        ok = ok && mbar_wait(feat, c & 1, wc, wsite(2, 7, c));
        if (!ok) return;
        tc_fence_after();
        // the image holds the decay-scaled keys (factored mode) or phi(k) (exact mode)
        const uint32_t kf_base = ki_base + (c & 1) * L::KV;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * (ROWS * 128) + (kk & 3) * 32;
          const uint32_t ko = (kk >> 2) * (C * 128) + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColSg, sdesc_sw128(eq_base + qo, 16, 1024), sdesc_sw128(kf_base + ko, 16, 1024),
                      id_n64, kk > 0);
        }
        // (failure-detection test: withhold the first completion; the waits downstream
        // then run out, record a timeout and drain)
        if (!(p.inject_stall && c == 0)) mma_commit(sg_done);
        // the state carry once the window warps have copied and rescaled S
        ok = ok && mbar_wait(state_ready, c & 1, wc, wsite(2, 10, c));
        ok = ok && mbar_wait(&v_full[(c + 1) % 3], ((c + 1) / 3) & 1, wc, wsite(2, 8, c));
        if (!ok) return;
        tc_fence_after();
        const uint32_t vc = smem_u32(smem + L::V0 + ((c + 1) % 3) * L::KV);
        // (exact mode: the feature warps have scaled the image to the decay-scaled keys by now)
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
          mma_bf16_ss(tmem + kColS, sdesc_sw128(kf_base + kk * 2048, lbo_kt, 1024),
                      sdesc_sw128(vc + kk * 2048, C * 128, 1024), id_state, 1u);
        mma_commit(state_done);
        mma_commit(&kimg_empty[c & 1]);   // the image slot may take chunk c + 2
      };
      auto issue_inter = [&](int c) {   // O = e_q' (e^{b_C} S) or (e^{b_i} e_q') S, the state as MN-major B
        if (c > 0) ok = ok && mbar_wait(o_free, (c - 1) & 1, wc, wsite(2, 9, c));
        if (!ok) return;
        tc_fence_after();
        // factored mode: the scaled e_q tile already is the A operand; otherwise it sits in the q buffer
        const bool fast = fast2[c & 1] != 0.f;
        const uint32_t a_base = fast ? eq_base : q_base;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * (ROWS * 128) + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColO, sdesc_sw128(a_base + qo, 16, 1024),
                      sdesc_sw128(sb_base + kk * 2048, D * 128, 1024), id_inter, kk > 0);
        }
        mma_commit(mma2_done);
        if (!fast) mma_commit(q_empty);   // exact decay: the readout read e^{b_i} e_q from the q buffer
      };
      // The next chunk's window scores go out as soon as the window warps have read the
      // previous scores, ahead of the previous chunk's P.V, so the window warps' next
      // softmax does not wait for that product.  The probability tile is rewritten only
      // after the recurrent scores' completion, which the tensor pipe signals after every
      // earlier product, P.V included.  The readout of a chunk waits for the feature
      // warps to have stored the previous chunk's output.
      issue_ss(0);
      issue_sg_state(0);
      issue_inter(0);
      for (int c = 1; c < nch && ok; ++c) {
        issue_ss(c);
        issue_pv(c - 1);
        issue_sg_state(c);
        issue_inter(c);
      }
      issue_pv(nch - 1);
      mma_commit(drain);
    }
  } else if (warp >= kFeatWarp0) {   // ---------------- features (256 threads)
    // Per chunk: the query features (two threads per row), then the state copy (two warps
    // per TMEM lane quarter, half the columns each).  The key features come ready from the
    // state pass (the image slots).  Never leaves the loop early: after a timeout every wait
    // returns at once (the CTA's abort flag is set), so the group still meets at each named
    // barrier and warp-collective TMEM access stays uniform.
    const int t = threadIdx.x - 32 * kFeatWarp0;
    const int half = t >> 7, lrow = t & 127;   // state-column half, TMEM lane (state row)
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    constexpr float kLog2e = 1.4426950408889634f;
    char* const qb = smem + L::Q0;
    char* const eqb = smem + L::EQ;
    char* const sbb = smem + L::SB;
    // The e_q tile carries the branch weight: e_q' = a e_q with a = alpha, taken into the
    // exponent (2^{log2 a}), so that the readout's state copy needs no multiply.  Z is summed
    // from the same scaled values and divided by a, so any rounding of log2 a cancels.  A
    // weight below 2^-20 (0 included) stays on the copy instead (a = 1), which keeps the
    // scaled scores far above fp32's smallest normal.
    const float qa = p.alpha >= 0x1p-20f ? p.alpha : 1.f;
    const float lqa = log2f(qa), iqa = 1.f / qa;
    const float copy_scale = p.alpha / qa;   // 1, or alpha when it stays on the copy

    // Output of chunk cc: this warp's lane quarter (rows 2 * token + head), its column half;
    // O / Z times the row factor from the window warps, bf16.  Frees the accumulator.
    __nv_bfloat16* const out = static_cast<__nv_bfloat16*>(p.out);
    auto epilogue = [&](int cc) {
      const bool live = mbar_wait(o_done, cc & 1, wc, wsite(3, 8, cc)) && !*abort_flag;
      tc_fence_after();
      const int t0c = sg.t_begin + cc * C, nvc = min(C, sg.t_end - t0c);
      const int i = lrow >> 1;
      const float os = osc2[(cc & 1) * 128 + lrow];
      __nv_bfloat16* orow = out + ((size_t)((long)t0c + i) * p.Hq + h0 + (lrow & 1)) * D;
      const bool store = i < nvc && live;
      const float2 os2 = make_float2(os, os);
#pragma unroll 1
      for (int col = half * (D / 2); col < (half + 1) * (D / 2); col += 32) {
        float v[32];
        tmem_ld32(lane_base + kColO + col, v);
        tmem_wait_ld();
        if (store) {
          uint32_t pw[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float2 y = fmul2(make_float2(v[2 * u], v[2 * u + 1]), os2);
            pw[u] = pack_bf16(y.x, y.y);
          }
          if (p.out_v8) {   // two full 32-byte sectors per instruction
            st_global_v8(orow + col, pw);
            st_global_v8(orow + col + 16, pw + 8);
          } else {
#pragma unroll
            for (int u = 0; u < 16; u += 4)
              *reinterpret_cast<uint4*>(orow + col + 2 * u) = make_uint4(pw[u], pw[u + 1], pw[u + 2], pw[u + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(o_free);
    };

    // state entering the segment: this warp's quarter of the first half of the columns
    // (the window warps load the second half)
    entering_state<D, D / 4>(p, seg, kv, lrow % D, lane_base + kColS, half * (D / 4));
    tc_fence_before();
    named_bar(2, 256 + 128);
    tc_fence_after();

    for (int c = 0; c < nch; ++c) {
      const int slot = c & 1;
      float* bsh = bsh2 + (c & 1) * 64;
      const float* bimg = reinterpret_cast<const float*>(smem + L::BI + slot * (C * 4));
      mbar_wait(&kimg_full[slot], (c >> 1) & 1, wc, wsite(3, 1, c));
      const int row = t >> 1, qh = t & 1;
      mbar_wait(q_full, c & 1, wc, wsite(3, 2, c));
      if (c > 0) mbar_wait(mma2_done, (c - 1) & 1, wc, wsite(3, 6, c));   // e_q tile, state copy, row buffers free
      tc_fence_after();
      // Factored mode (the chunk's total log gate b_C >= -60): e^{b_i - b_j} =
      // e^{b_i - b_C} e^{b_C - b_j}, both factors within e^{+-60}.  The key factor is the one
      // the image's decay-scaled keys carry, so the recurrent scores need no per-key scalar;
      // the row factor goes to the epilogue, and the readout uses e^{b_C} S, which is the
      // rescaled state.  Otherwise the image holds phi(k) and the window warps apply the
      // decay per element.
      const float bC = bimg[C - 1];
      const bool fast = bC >= kFactorFloor;   // the same decision for the whole CTA
      if (t < C) bsh[t] = bimg[t];
      if (t == 0) fast2[c & 1] = fast ? 1.f : 0.f;

      // queries: e_q' = a exp(q - q_0) per row (bf16, with the branch weight a above; not
      // divided by Z = sum_d e_q: the window warps fold Z into P and 1/Z into the output);
      // two threads per row.  One pass against the row's first element q_0 (the tiles carry
      // e_q unnormalised, so the shift cancels against Z); a row whose Z exceeds 2^24 (every
      // row with an element more than kShiftSpan above q_0, in log2) is redone against its
      // maximum.
      const float sl = bf16_lo(*reinterpret_cast<const uint32_t*>(qb + kmajor_off(row, 0, ROWS * 128))) * kLog2e;
      const float2 nsla = make_float2(lqa - sl, lqa - sl), l2e = make_float2(kLog2e, kLog2e);
      float2 zacc = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int c8 = 0; c8 < D / 16; ++c8) {
        const uint32_t off = kmajor_off(row, qh * (D / 2) + c8 * 8, ROWS * 128);
        const uint4 u = *reinterpret_cast<const uint4*>(qb + off);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
        float2 x[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          x[q] = ffma2(make_float2(bf16_lo(w4[q]), bf16_hi(w4[q])), l2e, nsla);
          x[q].x = ex2(x[q].x);
          x[q].y = ex2(x[q].y);
        }
        zacc = fadd2(zacc, fadd2(fadd2(x[0], x[1]), fadd2(x[2], x[3])));
        *reinterpret_cast<uint4*>(eqb + off) = make_uint4(pack_bf16(x[0].x, x[0].y), pack_bf16(x[1].x, x[1].y),
                                                          pack_bf16(x[2].x, x[2].y), pack_bf16(x[3].x, x[3].y));
      }
      float zq = zacc.x + zacc.y;
      zq += __shfl_xor_sync(0xffffffffu, zq, 1);
      // decided per row (the same on both of its threads), entered by the whole warp so
      // that the shuffles see every lane
      const bool redo = !(zq * iqa <= 0x1p24f);
      if (__any_sync(0xffffffffu, redo)) {
        float mq = -INFINITY;
        if (redo) {
#pragma unroll 1
          for (int c8 = 0; c8 < D / 16; ++c8)
            mq = fmaxf(mq, bf16x8_max(*reinterpret_cast<const uint4*>(
                               qb + kmajor_off(row, qh * (D / 2) + c8 * 8, ROWS * 128))));
        }
        mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, 1));
        float zr = 0.f;
        if (redo) {
          const float mql = mq * kLog2e - lqa;
#pragma unroll 1
          for (int c8 = 0; c8 < D / 16; ++c8) {
            const uint32_t off = kmajor_off(row, qh * (D / 2) + c8 * 8, ROWS * 128);
            float x[8];
            ld_chunk8(qb, off, x);
#pragma unroll
            for (int q = 0; q < 8; ++q) x[q] = ex2(fmaf(x[q], kLog2e, -mql));
            zr += ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
            st_chunk8(eqb, off, x);
          }
        }
        zr += __shfl_xor_sync(0xffffffffu, zr, 1);
        if (redo) zq = zr;
      }
      if (qh == 0) zq2[(c & 1) * 128 + row] = zq * iqa;
      // The q buffer is released twice per chunk: by the score MMA's commit, and by this
      // group once done with the raw q (factored mode) or by the readout's commit (exact
      // mode: the buffer then holds e^{b_i} e_q, the readout's A operand).
      if (fast) {
        named_bar(1, 256);
        if (t == 0) mbar_arrive(q_empty);
      } else {
        mbar_wait(ss_done, c & 1, wc, wsite(3, 4, c));
        const float ebi = __expf(bimg[row >> 1]);
#pragma unroll 4
        for (int c8 = 0; c8 < D / 16; ++c8) {
          const uint32_t off = kmajor_off(row, qh * (D / 2) + c8 * 8, ROWS * 128);
          float x[8];
          ld_chunk8(eqb, off, x);
#pragma unroll
          for (int q = 0; q < 8; ++q) x[q] *= ebi;
          st_chunk8(qb, off, x);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(feat);

      if (!fast) {
        // exact mode: once the recurrent scores have read phi(k) from the image, scale it in
        // place to the decay-scaled keys e^{b_C - b_j} phi(k_j) the state carry needs
        mbar_wait(sg_done, c & 1, wc, wsite(3, 3, c));
        const int j = t >> 2, h = t & 3;
        const float sc = __expf(bC - bimg[j]);
        char* const ki = smem + L::KI + slot * L::KV;
#pragma unroll
        for (int c8 = 0; c8 < D / 32; ++c8) {
          const uint32_t off = kmajor_off(j, h * (D / 4) + c8 * 8, C * 128);
          float x[8];
          ld_chunk8(ki, off, x);
#pragma unroll
          for (int q = 0; q < 8; ++q) x[q] *= sc;
          st_chunk8(ki, off, x);
        }
      }

      // State for this chunk: the bf16 copy of the readout's state (MN-major B operand),
      // then S <- e^{b_C} S in TMEM before the chunk's carry accumulates onto it (the
      // previous carry and readout are done).  Factored mode reads out e^{b_C} S, the
      // rescaled state itself; exact mode reads out S (its q buffer holds e^{b_i} e_q).
      // Either copy carries the part of alpha that the e_q tile does not.
      if (c > 0) mbar_wait(state_done, (c - 1) & 1, wc, wsite(3, 7, c));
      tc_fence_after();
      {
        const float dec = __expf(bC);
        const float2 dec2 = make_float2(dec, dec);
        if (fast && copy_scale == 1.f) {   // the same for the whole CTA
#pragma unroll 1
          for (int col = half * (D / 2); col < (half + 1) * (D / 2); col += 32) {
            float v[32];
            tmem_ld32(lane_base + kColS + col, v);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              const float2 y = fmul2(make_float2(v[u], v[u + 1]), dec2);
              v[u] = y.x;
              v[u + 1] = y.y;
            }
            if (lrow < D) {
#pragma unroll
              for (int u = 0; u < 32; u += 8)
                st_chunk8(sbb, (uint32_t)((col + u) >> 6) * (D * 128) + sw128(lrow, ((col + u) & 63) >> 3), v + u);
            }
            tmem_st32(lane_base + kColS + col, v);
          }
        } else {
          const float sc = fast ? copy_scale * dec : copy_scale;
#pragma unroll 1
          for (int col = half * (D / 2); col < (half + 1) * (D / 2); col += 16) {
            float v[16];
            tmem_ld16(lane_base + kColS + col, v);
            tmem_wait_ld();
            if (lrow < D) {
#pragma unroll
              for (int u = 0; u < 16; u += 8) {
                float x[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) x[q] = sc * v[u + q];
                st_chunk8(sbb, (uint32_t)((col + u) >> 6) * (D * 128) + sw128(lrow, ((col + u) & 63) >> 3), x);
              }
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] *= dec;
            tmem_st16(lane_base + kColS + col, v);
          }
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(state_ready);
      // the previous chunk's output (its P.V finished long ago); the readout of this chunk
      // waits for the accumulator to be free
      if (c > 0) epilogue(c - 1);
    }
    if (nch > 0) epilogue(nch - 1);
    // final state of the sequence: the carry after the last chunk of its last segment
    const SeqInfo si = p.seqs[sg.seq];
    const bool last = seg == si.first_seg + si.n_seg - 1;
    if (p.final_state && last && warp_all(mbar_wait(mma2_done, (nch - 1) & 1, wc, wsite(3, 5, nch)) && !*abort_flag)) {
      tc_fence_after();
#pragma unroll 1
      for (int col = half * (D / 2); col < (half + 1) * (D / 2); col += 32) {
        float v[32];
        tmem_ld32(lane_base + kColS + col, v);
        tmem_wait_ld();
        if (lrow < D) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float* dst = p.final_state + (((size_t)sg.seq * p.Hq + h0 + hh) * D + lrow) * D + col;
#pragma unroll
            for (int u = 0; u < 32; u += 4)
              *reinterpret_cast<float4*>(dst + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
          }
        }
      }
    }
  } else {   // ---------------- window softmax and the probability tile (128 threads, warps 0-3)
    const int r = threadIdx.x;
    const int i = r >> 1;
    const int wq = warp, il = i - 16 * wq;
    const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
    const float alpha = p.alpha, beta = 1.0f - p.alpha;
    // the part of alpha that the e_q tile (and so the recurrent scores) does not carry
    const float gscale = alpha / (alpha >= 0x1p-20f ? alpha : 1.f);
    const float sscale = 1.4426950408889634f / sqrtf((float)D);
    // state entering the segment, second half of the columns (the feature warps load the
    // first half; TMEM: the state follows O)
    entering_state<D, D / 2>(p, seg, kv, r % D, lane_base + kColO + D, D / 2);
    tc_fence_before();
    named_bar(2, 256 + 128);
    tc_fence_after();

    for (int c = 0; c < nch; ++c) {
      const int t0 = sg.t_begin + c * C;
      const int nv = min(C, sg.t_end - t0);
      const float* bsh = bsh2 + (c & 1) * 64;
      // Window band.  Key index x over [previous chunk | current chunk] (0..127): row i
      // sees x in [i+1, i+64].  This quarter's tokens are 16 wq .. 16 wq + 15, so it reads
      // the 80 columns starting at 16 wq; column j then holds x = 16 wq + j and is live for
      // j in [il+1, il+64], il = i - 16 wq (only x >= 64 in the sequence's first chunk).
      const int jlo = max(il + 1, t0 == sg.q0 ? 64 - 16 * wq : 0), jhi = il + 64;
      // score column of key x: (x + 64 (c & 1)) mod 128 (the two key slots form one operand)
      const int ss_rot = 16 * wq + ((c & 1) << 6);
      auto ss_col = [&](int q5) { return lane_base + kColSs + ((ss_rot + 16 * q5) & 127); };
      mbar_wait(ss_done, c & 1, wc, wsite(4, 6, c));
      tc_fence_after();
      // The row's 80 scores, loaded once: mask (-inf, whose exponential is 0), maximum,
      // exponentials and their sum in registers, then the exponentials written back over
      // the scores for the rolled probability pass below (short code for the instruction
      // caches the roles share).  Columns 16..63 are inside every row's band except in the
      // sequence's first chunk: only the outer groups (and that chunk) take the mask.
      const bool first = t0 == sg.q0;
      float lsum;
      {
        float s[80];
#pragma unroll
        for (int q5 = 0; q5 < 5; ++q5) tmem_ld16(ss_col(q5), s + 16 * q5);
        tmem_wait_ld();
#pragma unroll
        for (int q5 = 0; q5 < 5; ++q5) {
          if (first || q5 == 0 || q5 == 4) {
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const int j = 16 * q5 + u;
              s[16 * q5 + u] = (j >= jlo && j <= jhi) ? s[16 * q5 + u] : -INFINITY;
            }
          }
        }
        float m = -INFINITY;
#pragma unroll
        for (int u = 0; u < 80; u += 2) m = fmax3(m, s[u], s[u + 1]);
        const float2 sc2 = make_float2(sscale, sscale), nmsc = make_float2(-m * sscale, -m * sscale);
        float2 ls = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 80; u += 2) {
          float2 y = ffma2(make_float2(s[u], s[u + 1]), sc2, nmsc);
          y.x = ex2(y.x);
          y.y = ex2(y.y);
          s[u] = y.x;
          s[u + 1] = y.y;
          ls = fadd2(ls, y);
        }
        lsum = ls.x + ls.y;
#pragma unroll
        for (int q5 = 0; q5 < 5; ++q5) tmem_st16(ss_col(q5), s + 16 * q5);
        tmem_wait_st();
      }
      // Z of the rows and the recurrent scores come with the feature tiles
      mbar_wait(sg_done, c & 1, wc, wsite(4, 1, c));
      tc_fence_after();
      const bool fast = fast2[c & 1] != 0.f;
      // The tiles carry e_q unnormalised: P is scaled by Z and the output by 1/Z.  In
      // factored mode P also carries e^{b_C - b_i} and the output e^{b_i - b_C}.
      const float zrow = zq2[(c & 1) * 128 + r];
      const float bi = bsh[i];
      const float mrow = fast ? bsh[nv - 1] - bi : 0.f;
      const float coef = beta * zrow * __expf(mrow) / lsum;
      osc2[(c & 1) * 128 + r] = __expf(-mrow) / zrow;   // the feature warps scale and store the output
      const float2 coef2 = make_float2(coef, coef), gs2 = make_float2(gscale, gscale);
      // Probability tile over [previous | current] keys.  The recurrent tile covers the
      // same current keys (kk <= i) and multiplies the same values, so it is added to the
      // window tile's current half here: one P V product per half.  Group q5 holds the
      // current keys kk = 16 bb + u with bb = q5 + wq - 4 when bb >= 0.
#pragma unroll 1
      for (int q5 = 0; q5 < 5; ++q5) {
        const int bb = q5 + wq - 4;
        float sv[16], g[16];
        tmem_ld16(ss_col(q5), sv);
        if (bb >= 0) tmem_ld16(lane_base + kColSg + 16 * bb, g);
        tmem_wait_ld();
        if (bb >= 0) {
          if (!fast) {   // exact mode: scores against phi(k); the decay per element
#pragma unroll
            for (int u = 0; u < 16; ++u) g[u] *= __expf(bi - bsh[16 * bb + u]);
          }
          if (bb == wq) {   // the diagonal block is causal
#pragma unroll
            for (int u = 0; u < 16; ++u) g[u] = 16 * bb + u <= i ? g[u] : 0.f;
          }
          // factored: the scores already carry e^{b_C - b_kk} / z_kk
#pragma unroll
          for (int u = 0; u < 16; u += 2) {
            const float2 y = ffma2(make_float2(g[u], g[u + 1]), gs2, fmul2(make_float2(sv[u], sv[u + 1]), coef2));
            sv[u] = y.x;
            sv[u + 1] = y.y;
          }
        } else {
#pragma unroll
          for (int u = 0; u < 16; u += 2) {
            const float2 y = fmul2(make_float2(sv[u], sv[u + 1]), coef2);
            sv[u] = y.x;
            sv[u + 1] = y.y;
          }
        }
        uint32_t pw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pw[k] = pack_bf16(sv[2 * k], sv[2 * k + 1]);
        tmem_st8u(lane_base + kColP + 8 * wq + 8 * q5, pw);
      }
      {   // zeros for the keys outside this quarter's band
        const uint32_t zero8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
        for (int k = 0; k < 3; ++k) tmem_st8u(lane_base + kColP + ((8 * wq + 40 + 8 * k) & 63), zero8);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(s_read);    // the scores are consumed: their TMEM may be reused
      mbar_arrive(p_ready);   // the probability tile is in TMEM

    }
  }
  __syncthreads();
  if (warp == 0) {
    mbar_wait(drain, 0, WaitCtx{never, nullptr, p.wait_ns});
    tc_fence_after();
    tmem_dealloc(tmem, TCOLS);
  }
}

// ============================================================== host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

inline thread_local const char* g_msg = "";
inline const char* last_message() { return g_msg; }

inline bool supports(int d) { return d == 64 || d == 128; }

inline int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Segment length (chunks) and the bound on segments: a segment is one chunk
// CTA per q-head pair; pick the length that minimises waves x (length + fixed
// per-segment cost) for one CTA per SM.
inline Plan make_plan(int B, int Hq, int Hkv, long T, int d, int n_seqs, bool varlen) {
  Plan pl{};
  const long NT = varlen ? T : (long)B * T;
  const long chunks_total = (NT + C - 1) / C + (varlen ? n_seqs : 0);
  const long chunks_per_seq = varlen ? 0 : (T + C - 1) / C;
  const int sms = num_sms();
  const int pairs = Hq / 2;
  double best = 1e300;
  int bestL = 1;
  const long maxL = chunks_total > 0 ? chunks_total : 1;
  for (long Lc = 1; Lc <= maxL; Lc = Lc < 64 ? Lc + 1 : Lc + Lc / 8) {
    long nseg = varlen ? (NT + C * Lc - 1) / (C * Lc) + n_seqs : (long)B * ((chunks_per_seq + Lc - 1) / Lc);
    if (nseg < 1) nseg = 1;
    const double waves = std::ceil((double)nseg * pairs / sms);
    const double cost = waves * ((double)Lc + 1.5);
    if (cost < best) { best = cost; bestL = (int)Lc; }
  }
  pl.L = bestL;
  long nseg = varlen ? (NT + (long)C * bestL - 1) / ((long)C * bestL) + n_seqs
                     : (long)B * ((chunks_per_seq + bestL - 1) / bestL);
  if (nseg < 1) nseg = 1;
  pl.n_seg_max = (int)nseg;
  // The state pass splits segments into sub-segments; two of its CTAs run per SM.
  // Minimise waves x sub-segment length (plus a fixed cost per CTA).
  long nsub = 1;
  {
    const long units = nseg * Hkv;
    double best_s = 1e300;
    const long max_sub = bestL < kMaxSub ? bestL : kMaxSub;
    for (long ns = 1; ns <= max_sub; ++ns) {
      const double waves = std::ceil((double)units * ns / (2.0 * sms));
      const double cost = waves * (std::ceil((double)bestL / ns) + 0.5);
      if (cost < best_s - 1e-9) { best_s = cost; nsub = ns; }
    }
  }
  pl.nsub = (int)nsub;
  pl.Ls = (int)((bestL + nsub - 1) / nsub);
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 256;   // header: error word, first timeout, segment count
  pl.off_seqs = off;  off = al(off + sizeof(SeqInfo) * (size_t)n_seqs);
  pl.off_segs = off;  off = al(off + sizeof(SegInfo) * (size_t)nseg);
  pl.off_lam = off;   off = al(off + sizeof(float) * (size_t)nseg * nsub * Hkv);
  pl.off_ds = off;    off = al(off + sizeof(float) * (size_t)nseg * nsub * Hkv * d * d);
  pl.off_kimg = off;  off = al(off + (size_t)2 * C * d * (size_t)nseg * bestL * Hkv);
  pl.off_bimg = off;  off = al(off + sizeof(float) * C * (size_t)nseg * bestL * Hkv);
  pl.off_flags = off; off = al(off + sizeof(uint32_t) * (size_t)n_seqs * Hkv);
  pl.total = off;
  return pl;
}

inline size_t workspace_bytes(int B, int Hq, int Hkv, long T, int d, int n_seqs) {
  (void)n_seqs;
  // The varlen bound is the larger one; use it so one size serves both forms.
  const Plan a = make_plan(B, Hq, Hkv, T, d, B, false);
  const Plan b = make_plan(1, Hq, Hkv, (long)B * T, d, n_seqs > 0 ? n_seqs : B, true);
  return a.total > b.total ? a.total : b.total;
}

inline bool make_map(CUtensorMap* m, const void* ptr, int d, int H, long NT, int box_h) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)NT};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_h, (cuuint32_t)C};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch hooks supplied by the ABI layer (timing events and launch counting).
struct LaunchHooks {
  void (*before_main)(cudaStream_t);
  void (*after_main)(cudaStream_t);
  void (*count)(int);
};

inline uint64_t wait_limit_ns() {
  const unsigned long long v = options().wait_limit_ns;
  return v > 0 ? (uint64_t)v : kDefaultWaitNs;
}

// Launch with programmatic stream serialisation: the grid may be scheduled while
// the previous grid in the stream drains; every prefill kernel starts with
// griddep_wait_and_release, so nothing is read before its producer has finished.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
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

// On return, *s0_flags (when not null) points at the per-(sequence, kv head) flags the scan
// sets for groups whose initial-state copies differ (only meaningful with pb.s0).
// Kernel parameters of a call whose workspace `w` follows plan `pl`.
inline DevParams fill_params(const PrefillProblem& pb, char* w, const Plan& pl, long NT) {
  DevParams p{};
  p.seqs = reinterpret_cast<const SeqInfo*>(w + pl.off_seqs);
  p.segs = reinterpret_cast<const SegInfo*>(w + pl.off_segs);
  p.n_segs = reinterpret_cast<const int32_t*>(w + 8);
  p.err = reinterpret_cast<uint32_t*>(w);
  p.lam = reinterpret_cast<float*>(w + pl.off_lam);
  p.ds = reinterpret_cast<float*>(w + pl.off_ds);
  p.kimg = w + pl.off_kimg;
  p.bimg = reinterpret_cast<float*>(w + pl.off_bimg);
  p.out = pb.out;
  p.final_state = pb.final_state;
  p.s0 = pb.s0;
  p.s0_flags = reinterpret_cast<uint32_t*>(w + pl.off_flags);
  p.cu = pb.cu;
  p.T = pb.T;
  p.NT = NT;
  p.Hq = pb.Hq;
  p.Hkv = pb.Hkv;
  p.n_seqs = pb.n_seqs;
  p.n_seg_max = pl.n_seg_max;
  p.L = pl.L;
  p.nsub = pl.nsub;
  p.Ls = pl.Ls;
  p.alpha = pb.alpha;
  p.wait_ns = wait_limit_ns();
  p.out_v8 = (reinterpret_cast<uintptr_t>(pb.out) & 31u) == 0 ? 1 : 0;
  return p;
}

template <int D>
liger_status run_prefill_d(const PrefillProblem& pb, void* ws, cudaStream_t s, const LaunchHooks& hk,
                           const uint32_t** s0_flags) {
  const bool varlen = pb.cu != nullptr;
  const long NT = varlen ? pb.T : (long)pb.B * pb.T;
  const Plan pl = make_plan(pb.B, pb.Hq, pb.Hkv, pb.T, D, pb.n_seqs, varlen);
  char* w = static_cast<char*>(ws);
  DevParams p = fill_params(pb, w, pl, NT);
  p.inject_stall = take_injected_stall() ? 1 : 0;

  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, pb.q, D, pb.Hq, NT, 2) || !make_map(&mk, pb.k, D, pb.Hkv, NT, 1) ||
      !make_map(&mv, pb.v, D, pb.Hkv, NT, 1)) {
    g_msg = "cuTensorMapEncodeTiled failed (driver entry point missing or unsupported layout)";
    return LIGER_ERR_CUDA;
  }
  cudaError_t e;
  e = launch_chained(plan_kernel, dim3(1), dim3(32), 0, s, p, reinterpret_cast<SeqInfo*>(w + pl.off_seqs),
                     reinterpret_cast<SegInfo*>(w + pl.off_segs), reinterpret_cast<int32_t*>(w + 8));
  hk.count(1);
  if (e != cudaSuccess) { g_msg = cudaGetErrorString(e); return LIGER_ERR_CUDA; }

  auto seg_k = seg_state_kernel<D>;
  if (cudaFuncSetAttribute(seg_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SegSmem<D>::BYTES) !=
      cudaSuccess) {
    g_msg = "cudaFuncSetAttribute(seg_state) failed";
    cudaGetLastError();
    return LIGER_ERR_CUDA;
  }
  e = launch_chained(seg_k, dim3((unsigned)pl.n_seg_max * pl.nsub * pb.Hkv), dim3(kSegThreads), SegSmem<D>::BYTES,
                     s, mk, mv, p);
  hk.count(1);
  if (e != cudaSuccess) { g_msg = cudaGetErrorString(e); return LIGER_ERR_CUDA; }

  e = launch_chained(scan_kernel<D>, dim3((unsigned)(pb.n_seqs * pb.Hkv), (unsigned)(D * D / 1024)), dim3(256), 0,
                     s, p);
  hk.count(1);
  if (e != cudaSuccess) { g_msg = cudaGetErrorString(e); return LIGER_ERR_CUDA; }

  if (varlen && pb.final_state) {
    e = launch_chained(zero_empty_kernel<D>, dim3((unsigned)pb.n_seqs, (unsigned)pb.Hq), dim3(256), 0, s, p);
    hk.count(1);
    if (e != cudaSuccess) { g_msg = cudaGetErrorString(e); return LIGER_ERR_CUDA; }
  }

  auto chunk_k = chunk_kernel<D>;
  if (cudaFuncSetAttribute(chunk_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ChunkSmem<D>::BYTES) !=
      cudaSuccess) {
    g_msg = "cudaFuncSetAttribute(chunk) failed";
    cudaGetLastError();
    return LIGER_ERR_CUDA;
  }
  hk.before_main(s);
  e = launch_chained(chunk_k, dim3((unsigned)pl.n_seg_max * (pb.Hq / 2)), dim3(kChunkThreads), ChunkSmem<D>::BYTES,
                     s, mq, mk, mv, p);
  hk.after_main(s);
  hk.count(1);
  if (e != cudaSuccess) { g_msg = cudaGetErrorString(e); return LIGER_ERR_CUDA; }
  if (s0_flags) *s0_flags = p.s0_flags;
  return LIGER_OK;
}

inline liger_status run_prefill(const PrefillProblem& pb, void* ws, cudaStream_t s, const LaunchHooks& hk,
                                const uint32_t** s0_flags = nullptr) {
  g_msg = "";
  return pb.d == 64 ? run_prefill_d<64>(pb, ws, s, hk, s0_flags) : run_prefill_d<128>(pb, ws, s, hk, s0_flags);
}

}  // namespace tc
}  // namespace liger
