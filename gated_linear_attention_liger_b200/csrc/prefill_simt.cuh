// prefill_simt.cuh -- general prefill kernel on the CUDA cores, fp32 arithmetic.
//
// It serves fp32 inputs (whose tolerance rules out bf16/TF32 tensor-core
// operands), per-head initial states, and shapes the tensor-core kernel does
// not take.  One CTA per (sequence, q head); the recurrent state lives in
// registers, spread over the CTA (thread = one value column x a block of key
// rows), so the token-serial update S <- g S + phi(k)^T v and the readout
// phi(q) S need no synchronisation inside a chunk.  Everything that is
// parallel across the tokens of a chunk (feature maps, gates, window scores,
// window softmax and its value sum) is done first, chunk by chunk.  In segmented
// mode (prefill_seg.cuh) one CTA takes one segment of a sequence per q head, from the
// state a segment scan computed, with the window reaching back before the segment.
//
// Recurrence and hybrid: "Liger: Linearizing Large Language Models to Gated
// Recurrent Structures" (Paper-Notes page), sections 统一的门控线性循环框架 and
// Liger Attention; gate: section 核心思想 (mean pooling of the key).
#pragma once

#include "common.cuh"

namespace liger {

// A run of tokens of one sequence that one CTA per q head processes (segmented mode):
// the state entering it comes from a segment scan, the window reaches back into the
// tokens before it.
struct SimtSeg {
  long t_begin, t_end;   // the segment's tokens
  long seq_begin;        // first token of its sequence (the window starts no earlier)
  int seq;               // sequence index
  int flags;             // bit 0: first segment of its sequence; bit 1: last
};

struct SimtPrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* final_state;        // [n, Hq, d, d] or null
  const float* init_state;   // [n, Hq, d, d] or null
  const int32_t* cu;         // [n + 1] or null
  int Hq, Hkv, w;
  long T;                    // tokens per sequence (no offsets) / packed total
  float alpha;
  const uint32_t* only_flagged;   // [n][Hkv] or null: when set, a CTA works only if its
                                  // (sequence, kv head) flag is set, and returns at once otherwise
  // Segmented mode (segs non-null): the grid is (segment slot, q head); a segment that is
  // not its sequence's first starts from seg_state[slot][kv] (the state entering it, one
  // per kv head) instead of init_state; only a last segment writes the final state.
  const SimtSeg* segs;
  const int* n_segs;
  const float* seg_state;   // [slots][Hkv][D][D]
};

constexpr int kSimtThreads = 256;
constexpr int kSimtChunk = 32;         // tokens per chunk
constexpr int kSimtRing = 96;          // >= 64 + kSimtChunk - 1 window slots
constexpr int kMaxWindow = 64;

// VG: one gate per key dimension, sigmoid(k_t[r]) on row r of the state (the
// per-dimension form of the pooled key gate); otherwise the pooled scalar gate.
template <int D, bool VG = false>
constexpr size_t simt_prefill_smem_bytes() {
  constexpr int RG = kSimtThreads / D;
  return sizeof(float) * (size_t)(2 * kSimtRing * D + 3 * kSimtChunk * D + kSimtChunk * RG * D +
                                  kSimtChunk * kMaxWindow + kSimtChunk + (VG ? kSimtChunk * D : 0));
}

template <typename Tin, int D, bool VG = false>
__global__ void __launch_bounds__(kSimtThreads) prefill_simt_kernel(SimtPrefillArgs a) {
  constexpr int NT = kSimtThreads, C = kSimtChunk, RING = kSimtRing, W64 = kMaxWindow;
  constexpr int RG = NT / D;      // row groups
  constexpr int RPT = D / RG;     // key rows per thread
  constexpr int EPL = D / 32;     // elements per lane for row-wise work
  extern __shared__ float smem[];
  float* ring_k = smem;                     // [RING][D]
  float* ring_v = ring_k + RING * D;        // [RING][D]
  float* qbuf = ring_v + RING * D;          // [C][D]  raw q, later the window output
  float* fq = qbuf + C * D;                 // [C][D]  phi(q)
  float* fk = fq + C * D;                   // [C][D]  phi(k)
  float* part = fk + C * D;                 // [C][RG][D] partial readouts
  float* sc = part + C * RG * D;            // [C][W64] window scores / probabilities
  float* gate = sc + C * W64;               // [C]
  float* gvec = gate + C;                   // [C][D] per-dimension gates (VG only)

  const Tin* __restrict__ q = static_cast<const Tin*>(a.q);
  const Tin* __restrict__ k = static_cast<const Tin*>(a.k);
  const Tin* __restrict__ v = static_cast<const Tin*>(a.v);
  Tin* __restrict__ out = static_cast<Tin*>(a.out);
  const int Hq = a.Hq, Hkv = a.Hkv, w = a.w;
  const int unit = blockIdx.x / Hq, h = blockIdx.x % Hq, kv = h / (Hq / Hkv);
  int seq = unit;
  long tb, te, sb;          // sequence start, end of this CTA's tokens, first token of them
  bool first = true, last = true;
  if (a.segs) {
    if (unit >= *a.n_segs) return;
    const SimtSeg sg = a.segs[unit];
    seq = sg.seq;
    tb = sg.seq_begin;
    sb = sg.t_begin;
    te = sg.t_end;
    first = (sg.flags & 1) != 0;
    last = (sg.flags & 2) != 0;
  } else {
    const long T_total = a.cu ? a.T : (long)gridDim.x / Hq * a.T;
    seq_range(a.cu, seq, a.T, T_total, &tb, &te);
    sb = tb;
  }
  if (a.only_flagged && a.only_flagged[(size_t)seq * Hkv + kv] == 0u) return;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid % D, rg = tid / D;
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  const float alpha = a.alpha, beta = 1.0f - a.alpha;

  float s[RPT];
  const size_t st_off = ((size_t)seq * Hq + h) * D * D;
  const float* s_in = first ? (a.init_state ? a.init_state + st_off : nullptr)
                            : a.seg_state + ((size_t)unit * Hkv + kv) * D * D;
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = s_in ? s_in[(size_t)(rg * RPT + r) * D + c] : 0.f;

  // the window's keys and values before the first token (segmented mode)
  for (long idx = tid; idx < (sb - max(tb, sb - (w - 1))) * D; idx += NT) {
    const long t = max(tb, sb - (w - 1)) + idx / D;
    const int e = (int)(idx % D);
    const int slot = (int)((t - tb) % RING);
    ring_k[slot * D + e] = io<Tin>::ld(k + ((size_t)t * Hkv + kv) * D + e);
    ring_v[slot * D + e] = io<Tin>::ld(v + ((size_t)t * Hkv + kv) * D + e);
  }

  for (long t0 = sb; t0 < te; t0 += C) {
    const int n = (int)min((long)C, te - t0);
    // 1. stage the chunk: q rows, and k/v rows into the window ring
    for (int idx = tid; idx < n * D; idx += NT) {
      const int i = idx / D, e = idx % D;
      const long t = t0 + i;
      const int slot = (int)((t - tb) % RING);
      qbuf[idx] = io<Tin>::ld(q + ((size_t)t * Hq + h) * D + e);
      ring_k[slot * D + e] = io<Tin>::ld(k + ((size_t)t * Hkv + kv) * D + e);
      ring_v[slot * D + e] = io<Tin>::ld(v + ((size_t)t * Hkv + kv) * D + e);
    }
    __syncthreads();
    // 2. feature maps and gate, one warp per token
    for (int i = warp; i < n; i += NT / 32) {
      const int slot = (int)((t0 + i - tb) % RING);
      float x[EPL];
      float m = -INFINITY, sum = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = ring_k[slot * D + lane + 32 * j]; m = fmaxf(m, x[j]); sum += x[j]; }
      m = warp_max(m);
      sum = warp_sum(sum);
      float z = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
      z = warp_sum(z);
#pragma unroll
      for (int j = 0; j < EPL; ++j) fk[i * D + lane + 32 * j] = x[j] / z;
      if (VG) {
#pragma unroll
        for (int j = 0; j < EPL; ++j) gvec[i * D + lane + 32 * j] = expf(log_sigmoid(ring_k[slot * D + lane + 32 * j]));
      } else if (lane == 0) {
        gate[i] = expf(log_sigmoid(sum / (float)D));
      }
      m = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = qbuf[i * D + lane + 32 * j]; m = fmaxf(m, x[j]); }
      m = warp_max(m);
      z = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
      z = warp_sum(z);
#pragma unroll
      for (int j = 0; j < EPL; ++j) fq[i * D + lane + 32 * j] = x[j] / z;
    }
    // 3a. window scores q_t . k_j / sqrt(d) for j = t-w+1 .. t, one warp per pair
    for (int pr = warp; pr < n * w; pr += NT / 32) {
      const int i = pr / w, jj = pr % w;
      const long j = t0 + i - (w - 1) + jj;
      float dot = -INFINITY;
      if (j >= tb) {
        const int slot = (int)((j - tb) % RING);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e)
          acc = fmaf(qbuf[i * D + lane + 32 * e], ring_k[slot * D + lane + 32 * e], acc);
        dot = warp_sum(acc) * inv_sqrt_d;
      }
      if (lane == 0) sc[i * W64 + jj] = dot;
    }
    __syncthreads();
    // 3b. window softmax, one warp per token row
    for (int i = warp; i < n; i += NT / 32) {
      const float x0 = lane < w ? sc[i * W64 + lane] : -INFINITY;
      const float x1 = lane + 32 < w ? sc[i * W64 + lane + 32] : -INFINITY;
      const float m = warp_max(fmaxf(x0, x1));   // the token itself is always valid
      const float e0 = lane < w ? expf(x0 - m) : 0.f;
      const float e1 = lane + 32 < w ? expf(x1 - m) : 0.f;
      const float z = warp_sum(e0 + e1);
      if (lane < w) sc[i * W64 + lane] = e0 / z;
      if (lane + 32 < w) sc[i * W64 + lane + 32] = e1 / z;
    }
    __syncthreads();
    // 3c. window output into qbuf (raw q no longer needed)
    for (int idx = tid; idx < n * D; idx += NT) {
      const int i = idx / D, e = idx % D;
      const long t = t0 + i;
      float acc = 0.f;
      for (int jj = 0; jj < w; ++jj) {
        const long j = t - (w - 1) + jj;
        if (j < tb) continue;
        acc = fmaf(sc[i * W64 + jj], ring_v[((int)((j - tb) % RING)) * D + e], acc);
      }
      qbuf[idx] = acc;
    }
    // 4. token-serial recurrence on the register-resident state (no syncs)
    for (int i = 0; i < n; ++i) {
      const float g = VG ? 1.f : gate[i];
      const float vc = ring_v[((int)((t0 + i - tb) % RING)) * D + c];
      const float* fki = fk + i * D + rg * RPT;
      const float* fqi = fq + i * D + rg * RPT;
      float acc = 0.f;
      const float* gvi = gvec + i * D + rg * RPT;
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        s[r] = fmaf(VG ? gvi[r] : g, s[r], fki[r] * vc);
        acc = fmaf(fqi[r], s[r], acc);
      }
      part[(i * RG + rg) * D + c] = acc;
    }
    __syncthreads();
    // 5. mix and store
    for (int idx = tid; idx < n * D; idx += NT) {
      const int i = idx / D, e = idx % D;
      float grm = 0.f;
#pragma unroll
      for (int r = 0; r < RG; ++r) grm += part[(i * RG + r) * D + e];
      io<Tin>::st(out + ((size_t)(t0 + i) * Hq + h) * D + e, alpha * grm + beta * qbuf[idx]);
    }
    __syncthreads();
  }
  if (a.final_state && last) {
#pragma unroll
    for (int r = 0; r < RPT; ++r) a.final_state[st_off + (size_t)(rg * RPT + r) * D + c] = s[r];
  }
}

// Window ring and positions after a prefill: slot p mod w holds position p of
// the sequence for its last min(len, w) positions; other slots are zero.
// Grid (n_seqs, Hkv), one thread per element of a ring row.
template <typename Tin>
__global__ void prefill_ring_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v,
                                    Tin* __restrict__ ring, int32_t* __restrict__ pos,
                                    const int32_t* __restrict__ cu, long T, int Hkv, int d, int w) {
  const int seq = blockIdx.x, kv = blockIdx.y;
  const long T_total = cu ? T : (long)gridDim.x * T;
  long tb, te;
  seq_range(cu, seq, T, T_total, &tb, &te);
  const long len = te - tb;
  if (ring) {
    Tin* rk = ring + (((size_t)seq * Hkv + kv) * 2 + 0) * w * d;
    Tin* rv = ring + (((size_t)seq * Hkv + kv) * 2 + 1) * w * d;
    for (int idx = threadIdx.x; idx < w * d; idx += blockDim.x) {
      const int s = idx / d, e = idx % d;
      float kx = 0.f, vx = 0.f;
      if (s < len) {
        const long p = s + (long)w * ((len - 1 - s) / w);   // newest position at this slot
        const long t = tb + p;
        kx = io<Tin>::ld(k + ((size_t)t * Hkv + kv) * d + e);
        vx = io<Tin>::ld(v + ((size_t)t * Hkv + kv) * d + e);
      }
      io<Tin>::st(rk + idx, kx);
      io<Tin>::st(rv + idx, vx);
    }
  }
  if (pos && kv == 0 && threadIdx.x == 0) pos[seq] = (int32_t)len;
}

}  // namespace liger
