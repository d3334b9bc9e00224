// prefill_seg.cuh -- segment-parallel general prefill (CUDA cores, fp32 arithmetic).
//
// The general kernel steps the recurrence token by token, one CTA per (sequence,
// q head).  This file splits each sequence into segments of kSegTokens tokens so
// that the token-serial work runs on many CTAs at once:
//   1. plan          the segment table from the sequence lengths (device side);
//   2. seg_state     per (segment, kv head): the segment's own contribution to the
//                    state, dS = sum_j diag(e^{B - B_j}) phi(k_j)^T v_j, and its total
//                    log gate B (a vector over the key dimensions, or one value
//                    repeated, for the pooled gate), B_j the running sum up to j;
//   3. scan          per (sequence, kv head): the state entering each segment,
//                    S_in(s+1) = diag(e^{B_s}) S_in(s) + dS_s, written over dS_s;
//   4. the general kernel in segmented mode, per (segment, q head), from S_in.
// The state is carried per kv head (the recurrence never reads q); an initial
// state whose G copies in a group differ is handled by the caller, which reruns
// those groups with the unsegmented kernel.
//
// Recurrence: "Liger: Linearizing Large Language Models to Gated Recurrent
// Structures" (Paper-Notes page), section 统一的门控线性循环框架; the state of a
// run of tokens is the sum of its tokens' outer products, each decayed by the
// gates after it, which is what makes the scan associative.
#pragma once

#include "prefill_simt.cuh"

namespace liger {
namespace seg {

constexpr int kSegTokens = 256;   // tokens per segment
constexpr int kSegThreads = 256;
constexpr int kStage = 64;        // tokens staged in shared memory at a time

// Upper bound of the segment count: every sequence adds at most one partial (or empty)
// segment.
inline long max_segments(long T_total, int n_seqs) { return T_total / kSegTokens + n_seqs; }

// One thread: walks the sequences and writes the segment table and its length.
// Also clears the per-(sequence, kv head) flags the scan sets.
__global__ void plan_kernel(const int32_t* cu, long T, int n_seqs, long T_total, SimtSeg* segs, int* n_segs,
                            long cap, uint32_t* flags, int Hkv) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  for (long i = 0; i < (long)n_seqs * Hkv; ++i) flags[i] = 0u;
  long n = 0;
  for (int s = 0; s < n_seqs; ++s) {
    long b, e;
    seq_range(cu, s, T, T_total, &b, &e);
    // an empty sequence still gets one (empty) segment: it writes the final state
    for (long t = b; (t < e || t == b) && n < cap; t += kSegTokens, ++n) {
      SimtSeg g;
      g.t_begin = t;
      g.t_end = min(e, t + kSegTokens);
      g.seq_begin = b;
      g.seq = s;
      g.flags = (t == b ? 1 : 0) | (g.t_end == e ? 2 : 0);
      segs[n] = g;
    }
  }
  *n_segs = (int)n;
}

// Per (segment slot, kv head), 256 threads: thread (row group rg, column quad cq) owns
// the tile of rows rg*RPG .. rg*RPG+RPG-1 and columns 4cq .. 4cq+3 of dS (the general
// kernel's recurrence tile; the keys and weights are stored in its padded row-group
// layout, so a thread's RPG rows are float4 loads without bank conflicts).  Tokens are
// staged 64 at a time, last to first: lam[r] = B - B_j (the gates after token j) is then
// known when j is reached, and w_j[r] = e^{lam[r]} phi(k_j)[r] <= phi(k_j)[r].
template <typename Tin, int D, bool VG>
__global__ void __launch_bounds__(kSegThreads) seg_state_kernel(const Tin* __restrict__ k,
                                                                const Tin* __restrict__ v, int Hkv,
                                                                const SimtSeg* segs, const int* n_segs,
                                                                float* __restrict__ ds, float* __restrict__ lam_out) {
  constexpr int NT = kSegThreads, S = kStage;
  using RT = SimtRows<D>;
  static_assert(kSegThreads == kSimtThreads, "the general kernel's tile");
  constexpr int RPG = RT::RPG, RGS = RT::RGS, FS = RT::FS, NRG = RT::NRG, EPL = D / 32;
  extern __shared__ __align__(16) float seg_smem[];
  float (*kw)[FS] = reinterpret_cast<float (*)[FS]>(seg_smem);           // [S][FS] raw keys, then the weights w_j
  float (*vs)[D] = reinterpret_cast<float (*)[D]>(seg_smem + S * FS);    // [S][D]
  float (*lg)[VG ? D : 1] = reinterpret_cast<float (*)[VG ? D : 1]>(seg_smem + S * (FS + D));   // [S] log gates
  __shared__ float lam[D];                   // gates after the staged block
  const int slot = blockIdx.x / Hkv, kv = blockIdx.x % Hkv;
  if (slot >= *n_segs) return;
  const SimtSeg sg = segs[slot];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rg = tid % NRG, cq = tid / NRG;
  float4 acc[RPG];
#pragma unroll
  for (int r = 0; r < RPG; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (tid < D) lam[tid] = 0.f;
  for (long t1 = sg.t_end; t1 > sg.t_begin; t1 -= S) {
    const long t0 = max(sg.t_begin, t1 - S);
    const int n = (int)(t1 - t0);
    __syncthreads();   // the previous block's weights are consumed
    {   // every load of a thread in flight before its first store
      RowPieces<Tin, D, S, NT> pk, pv;
      pk.load(k + ((size_t)t0 * Hkv + kv) * D, (size_t)Hkv * D, n, tid);
      pv.load(v + ((size_t)t0 * Hkv + kv) * D, (size_t)Hkv * D, n, tid);
      pk.store(n, tid, [=](int i, int e) { return &kw[i][RT::at(e)]; });
      pv.store(n, tid, [=](int i, int e) { return &vs[i][e]; });
    }
    __syncthreads();
    // phi(k) and the log gates, one warp per token
    for (int i = warp; i < n; i += NT / 32) {
      float x[EPL], m = -INFINITY, sum = 0.f, z = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = kw[i][RT::at(lane + 32 * j)]; m = fmaxf(m, x[j]); sum += x[j]; }
      m = warp_max(m);
      sum = warp_sum(sum);
      if (VG) {
#pragma unroll
        for (int j = 0; j < EPL; ++j) lg[i][VG ? lane + 32 * j : 0] = log_sigmoid(x[j]);
      } else if (lane == 0) {
        lg[i][0] = log_sigmoid(sum / (float)D);
      }
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
      z = warp_sum(z);
#pragma unroll
      for (int j = 0; j < EPL; ++j) kw[i][RT::at(lane + 32 * j)] = x[j] / z;
    }
    __syncthreads();
    // weights, last token first: one thread per key dimension
    if (tid < D) {
      float l = lam[tid];
      const int at = RT::at(tid);
      for (int i = n - 1; i >= 0; --i) {
        kw[i][at] *= expf(l);
        l += lg[i][VG ? tid : 0];
      }
      lam[tid] = l;
    }
    __syncthreads();
    for (int i = 0; i < n; ++i) {
      const float4 v4 = *reinterpret_cast<const float4*>(&vs[i][4 * cq]);
      const float2 v01 = make_float2(v4.x, v4.y), v23 = make_float2(v4.z, v4.w);
#pragma unroll
      for (int r4 = 0; r4 < RPG; r4 += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(&kw[i][rg * RGS + r4]);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const float wr = rr == 0 ? w4.x : rr == 1 ? w4.y : rr == 2 ? w4.z : w4.w;
          const float2 w2 = make_float2(wr, wr);
          float4& a = acc[r4 + rr];
          const float2 a01 = sm100::ffma2(w2, v01, make_float2(a.x, a.y));
          const float2 a23 = sm100::ffma2(w2, v23, make_float2(a.z, a.w));
          a = make_float4(a01.x, a01.y, a23.x, a23.y);
        }
      }
    }
  }
  float* dst = ds + ((size_t)slot * Hkv + kv) * D * D;
#pragma unroll
  for (int r = 0; r < RPG; ++r) *reinterpret_cast<float4*>(dst + (size_t)(rg * RPG + r) * D + 4 * cq) = acc[r];
  __syncthreads();
  if (tid < D) lam_out[((size_t)slot * Hkv + kv) * D + tid] = lam[tid];
}

template <int D, bool VG>
constexpr size_t seg_state_smem_bytes() {
  return sizeof(float) * (size_t)kStage * (SimtRows<D>::FS + D + (VG ? D : 1));
}

// Per (sequence, kv head, block of 256 state elements): folds the segments'
// contributions in order, overwriting each segment's dS with the state entering it
// (every element of the state evolves on its own: S_in(s+1)[r][c] = e^{B_s[r]} S_in(s)[r][c]
// + dS_s[r][c]).  The scan starts from the group's first copy of the initial state; when
// another copy of the group differs, the (sequence, kv head) flag is set and the caller
// recomputes that group unsegmented.
constexpr int kScanThreads = 256;
template <int D>
__global__ void __launch_bounds__(kScanThreads) scan_kernel(const SimtSeg* segs, const int* n_segs, int Hq,
                                                            int Hkv, const float* __restrict__ init_state,
                                                            float* __restrict__ ds, const float* __restrict__ lam,
                                                            uint32_t* flags) {
  constexpr int BPU = D * D / kScanThreads;   // blocks per (sequence, kv head)
  const int unit = blockIdx.x / BPU, blk = blockIdx.x % BPU;
  const int seq = unit / Hkv, kv = unit % Hkv;
  const int e = blk * kScanThreads + threadIdx.x, r = e / D;
  const int G = Hq / Hkv;
  float s = 0.f;
  if (init_state) {
    const float* s0 = init_state + ((size_t)seq * Hq + (size_t)kv * G) * D * D + e;
    s = s0[0];
    bool differ = false;
    for (int hh = 1; hh < G; ++hh) differ |= s0[(size_t)hh * D * D] != s;
    if (__syncthreads_or(differ) && threadIdx.x == 0) atomicOr(&flags[(size_t)seq * Hkv + kv], 1u);
  }
  // the segments of one sequence are consecutive in the table, which is sorted by
  // sequence: both ends are found by bisection, so the loop below knows its length
  const int n = *n_segs;
  auto lower = [&](int key) {
    int lo = 0, hi = n;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (segs[mid].seq < key) lo = mid + 1;
      else hi = mid;
    }
    return lo;
  };
  const int first = lower(seq), last = lower(seq + 1);
  // PF segments' dS and log gates are loaded before their serial multiply-adds, so that
  // the loads of a batch are in flight together
  constexpr int PF = 8;
  for (int base = first; base < last; base += PF) {
    float dv[PF], lv[PF];
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      if (base + u < last) {
        const size_t su = (size_t)(base + u) * Hkv + kv;
        dv[u] = ds[su * D * D + e];
        lv[u] = lam[su * D + r];
      }
    }
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      if (base + u < last) {
        ds[((size_t)(base + u) * Hkv + kv) * D * D + e] = s;
        s = fmaf(expf(lv[u]), s, dv[u]);
      }
    }
  }
}

// Workspace of the segmented prefill: segment count, segment table, per (slot, kv
// head) the total log gate [D] and dS / the entering state [D][D], the flags.
struct Layout {
  long cap;
  size_t off_segs, off_lam, off_ds, off_flags, total;
};
inline Layout layout(long T_total, int n_seqs, int Hkv, int d) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  Layout L{};
  L.cap = max_segments(T_total, n_seqs);
  size_t off = 256;   // header: the segment count
  L.off_segs = off;   off = al(off + sizeof(SimtSeg) * (size_t)L.cap);
  L.off_lam = off;    off = al(off + sizeof(float) * (size_t)L.cap * Hkv * d);
  L.off_ds = off;     off = al(off + sizeof(float) * (size_t)L.cap * Hkv * d * d);
  L.off_flags = off;  off = al(off + sizeof(uint32_t) * (size_t)n_seqs * Hkv);
  L.total = off;
  return L;
}

}  // namespace seg
}  // namespace liger
