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
#include "sm100.cuh"

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
// Shared-memory ring rows are padded by 4 floats: consecutive slots then sit in different
// 16-byte bank groups, so eight lanes reading eight slots at the same column do not conflict.
template <int D>
constexpr int simt_ring_stride() { return D + 4; }

// The recurrence's thread tile: thread = a row group of RPG key rows x one quad of value
// columns; the NRG row groups of a column quad are adjacent lanes.  phi(k), phi(q) and the
// per-row gates of a token are stored by row group, each group's RPG values padded to a
// stride of an odd number of 16-byte units, so that the row groups a warp reads in one
// vector load sit in different bank groups.
template <int D>
struct SimtRows {
  static constexpr int CQN = D / 4;                 // column quads
  static constexpr int NRG = kSimtThreads / CQN;    // row groups
  static constexpr int RPG = D / NRG;               // rows per group
  static constexpr int RGS = ((RPG / 4 + 1) % 2) ? RPG + 4 : RPG + 8;   // padded group stride (floats)
  static constexpr int FS = NRG * RGS;              // floats per token
  static_assert(NRG >= 8 && NRG <= 32 && RPG % 4 == 0, "row groups of a quad within one warp");
  __device__ __forceinline__ static int at(int e) { return (e / RPG) * RGS + e % RPG; }
};

// Up to MAXR rows of one head of a [token][head][D] tensor, staged into shared memory in
// 16-byte pieces: load() issues every load of the calling thread (read-only path), store()
// converts to fp32 and writes each piece as float4s at dst(row, element).  Calling the
// load() of several tensors before their store() puts all of a thread's loads in flight
// together, so a chunk's rows arrive in about one memory latency.
template <typename Tin, int D, int MAXR, int NT>
struct RowPieces {
  static constexpr int EPP = 16 / (int)sizeof(Tin);          // elements per piece
  static constexpr int PPR = D / EPP;                        // pieces per row
  static constexpr int MAXP = (MAXR * PPR + NT - 1) / NT;    // pieces per thread
  uint4 raw[MAXP];
  __device__ __forceinline__ void load(const Tin* __restrict__ src, size_t row_stride, int n, int tid) {
#pragma unroll
    for (int u = 0; u < MAXP; ++u) {
      const int idx = tid + u * NT;
      if (idx < n * PPR)
        raw[u] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)(idx / PPR) * row_stride + (idx % PPR) * EPP));
    }
  }
  template <typename Dst>
  __device__ __forceinline__ void store(int n, int tid, Dst dst) const {
#pragma unroll
    for (int u = 0; u < MAXP; ++u) {
      const int idx = tid + u * NT;
      if (idx < n * PPR) {
        float x[EPP];
        if constexpr (sizeof(Tin) == 2) {
          const uint32_t w4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            x[2 * q] = __uint_as_float(w4[q] << 16);
            x[2 * q + 1] = __uint_as_float(w4[q] & 0xFFFF0000u);
          }
        } else {
          x[0] = __uint_as_float(raw[u].x); x[1] = __uint_as_float(raw[u].y);
          x[2] = __uint_as_float(raw[u].z); x[3] = __uint_as_float(raw[u].w);
        }
        const int i = idx / PPR, e0 = (idx % PPR) * EPP;
#pragma unroll
        for (int e = 0; e < EPP; e += 4)
          *reinterpret_cast<float4*>(dst(i, e0 + e)) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
      }
    }
  }
};

// VG: one gate per key dimension, sigmoid(k_t[r]) on row r of the state (the
// per-dimension form of the pooled key gate); otherwise the pooled scalar gate.
template <int D, bool VG = false>
constexpr size_t simt_prefill_smem_bytes() {
  constexpr int FS = SimtRows<D>::FS;
  return sizeof(float) * (size_t)(2 * kSimtRing * simt_ring_stride<D>() + kSimtChunk * D + 2 * kSimtChunk * FS +
                                  kSimtChunk * D + kSimtChunk * kSimtRing + kSimtChunk + (VG ? kSimtChunk * FS : 0));
}

template <typename Tin, int D, bool VG = false>
__global__ void __launch_bounds__(kSimtThreads) prefill_simt_kernel(SimtPrefillArgs a) {
  constexpr int NT = kSimtThreads, C = kSimtChunk, RING = kSimtRing;
  constexpr int RS = simt_ring_stride<D>();
  using RT = SimtRows<D>;
  constexpr int NRG = RT::NRG, RPG = RT::RPG, RGS = RT::RGS, FS = RT::FS;
  constexpr int EPL = D / 32;     // elements per lane for row-wise work
  constexpr int TPW = C / (NT / 32);   // window: tokens per warp
  constexpr int XPL = RING / 32;       // window: ring positions per lane
  static_assert(RING == C + kMaxWindow && RING % 32 == 0 && C % (NT / 32) == 0 && (EPL == 2 || EPL == 4),
                "window and row tiling");
  extern __shared__ float smem[];
  float* ring_k = smem;                     // [RING][RS]
  float* ring_v = ring_k + RING * RS;       // [RING][RS]
  float* qbuf = ring_v + RING * RS;         // [C][D]  raw q, later the window output
  float* fq = qbuf + C * D;                 // [C][FS] phi(q), by row group
  float* fk = fq + C * FS;                  // [C][FS] phi(k), by row group
  float* grm = fk + C * FS;                 // [C][D] recurrent readouts
  float* sc = grm + C * D;                  // [C][RING] window probabilities over the ring positions
  float* gate = sc + C * RING;              // [C]
  float* gvec = gate + C;                   // [C][FS] per-dimension gates by row group (VG only)

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
  const int rg = tid % NRG, cq = tid / NRG;   // recurrence tile: rows rg*RPG.., columns 4cq..4cq+3
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  const float alpha = a.alpha, beta = 1.0f - a.alpha;

  float4 s[RPG];   // s[r] = row rg*RPG + r, columns 4cq .. 4cq+3
  const size_t st_off = ((size_t)seq * Hq + h) * D * D;
  const float* s_in = first ? (a.init_state ? a.init_state + st_off : nullptr)
                            : a.seg_state + ((size_t)unit * Hkv + kv) * D * D;
#pragma unroll
  for (int r = 0; r < RPG; ++r)
    s[r] = s_in ? *reinterpret_cast<const float4*>(s_in + (size_t)(rg * RPG + r) * D + 4 * cq)
                : make_float4(0.f, 0.f, 0.f, 0.f);

  // the window's keys and values before the first token (segmented mode)
  {
    const long tp = max(tb, sb - (w - 1));
    const int np = (int)(sb - tp);
    const int slot_p = (int)((tp - tb) % RING);
    auto ring_row = [&](float* ring) {
      return [=](int i, int e) {
        int sl = slot_p + i;
        sl = sl >= RING ? sl - RING : sl;
        return ring + sl * RS + e;
      };
    };
    RowPieces<Tin, D, kMaxWindow - 1, NT> pk, pv;
    pk.load(k + ((size_t)tp * Hkv + kv) * D, (size_t)Hkv * D, np, tid);
    pv.load(v + ((size_t)tp * Hkv + kv) * D, (size_t)Hkv * D, np, tid);
    pk.store(np, tid, ring_row(ring_k));
    pv.store(np, tid, ring_row(ring_v));
  }

  for (long t0 = sb; t0 < te; t0 += C) {
    const int n = (int)min((long)C, te - t0);
    // 1. stage the chunk: q rows, and k/v rows into the window ring (every load of a
    //    thread in flight before its first store)
    {
      const int slot_c = (int)((t0 - tb) % RING);
      auto ring_row = [&](float* ring) {
        return [=](int i, int e) {
          int sl = slot_c + i;
          sl = sl >= RING ? sl - RING : sl;
          return ring + sl * RS + e;
        };
      };
      RowPieces<Tin, D, C, NT> pq, pk, pv;
      pq.load(q + ((size_t)t0 * Hq + h) * D, (size_t)Hq * D, n, tid);
      pk.load(k + ((size_t)t0 * Hkv + kv) * D, (size_t)Hkv * D, n, tid);
      pv.load(v + ((size_t)t0 * Hkv + kv) * D, (size_t)Hkv * D, n, tid);
      pq.store(n, tid, [=](int i, int e) { return qbuf + i * D + e; });
      pk.store(n, tid, ring_row(ring_k));
      pv.store(n, tid, ring_row(ring_v));
    }
    __syncthreads();
    // 2. feature maps and gate, one warp per token
    for (int i = warp; i < n; i += NT / 32) {
      const int slot = (int)((t0 + i - tb) % RING);
      float x[EPL];
      float m = -INFINITY, sum = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = ring_k[slot * RS + lane + 32 * j]; m = fmaxf(m, x[j]); sum += x[j]; }
      m = warp_max(m);
      sum = warp_sum(sum);
      float z = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
      z = warp_sum(z);
#pragma unroll
      for (int j = 0; j < EPL; ++j) fk[i * FS + RT::at(lane + 32 * j)] = x[j] / z;
      if (VG) {
#pragma unroll
        for (int j = 0; j < EPL; ++j)
          gvec[i * FS + RT::at(lane + 32 * j)] = expf(log_sigmoid(ring_k[slot * RS + lane + 32 * j]));
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
      for (int j = 0; j < EPL; ++j) fq[i * FS + RT::at(lane + 32 * j)] = x[j] / z;
    }
    __syncthreads();   // features and gates of every token (phase 2 rows are spread over the warps)
    // 3. window branch over the ring, which holds positions t0 - 64 .. t0 + C - 1 (ring
    //    position x holds t0 - 64 + x; slot = (position - tb) mod RING).  Warp w takes the
    //    tokens w TPW .. w TPW + TPW - 1, lane l the ring positions l, l + 32, l + 64: each
    //    thread forms its TPW x XPL scores in registers (row i sees x in [i + 64 - w + 1,
    //    i + 64] at positions >= tb), the warp reduces each row's softmax statistics.
    const int i0 = warp * TPW;
    const long pbase = t0 - kMaxWindow;   // position of ring position 0
    const int slot0 = (int)((((pbase - tb) % RING) + RING) % RING);
    {
      int xslot[XPL];
#pragma unroll
      for (int u = 0; u < XPL; ++u) {
        const int sl = slot0 + lane + 32 * u;
        xslot[u] = sl >= RING ? sl - RING : sl;
      }
      float acc[TPW][XPL];
#pragma unroll
      for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
        for (int u = 0; u < XPL; ++u) acc[tt][u] = 0.f;
#pragma unroll 4
      for (int e = 0; e < D; e += 4) {
        float4 kq[XPL];
#pragma unroll
        for (int u = 0; u < XPL; ++u) kq[u] = *reinterpret_cast<const float4*>(ring_k + xslot[u] * RS + e);
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
          const float4 qq = *reinterpret_cast<const float4*>(qbuf + (i0 + tt) * D + e);
#pragma unroll
          for (int u = 0; u < XPL; ++u)
            acc[tt][u] = fmaf(qq.x, kq[u].x, fmaf(qq.y, kq[u].y, fmaf(qq.z, kq[u].z, fmaf(qq.w, kq[u].w, acc[tt][u]))));
        }
      }
#pragma unroll
      for (int tt = 0; tt < TPW; ++tt) {
        const int i = i0 + tt;
        float sv[XPL], m = -INFINITY;
#pragma unroll
        for (int u = 0; u < XPL; ++u) {
          const int x = lane + 32 * u;
          const bool ok = i < n && x >= i + kMaxWindow - w + 1 && x <= i + kMaxWindow && pbase + x >= tb;
          sv[u] = ok ? acc[tt][u] * inv_sqrt_d : -INFINITY;
          m = fmaxf(m, sv[u]);
        }
        m = warp_max(m);   // finite for i < n: the token itself is always in its window
        float z = 0.f;
#pragma unroll
        for (int u = 0; u < XPL; ++u) {
          sv[u] = sv[u] == -INFINITY ? 0.f : expf(sv[u] - m);
          z += sv[u];
        }
        z = warp_sum(z);
        const float iz = z > 0.f ? 1.f / z : 0.f;
#pragma unroll
        for (int u = 0; u < XPL; ++u) sc[i * RING + lane + 32 * u] = sv[u] * iz;
      }
    }
    __syncwarp();
    // window output into qbuf (this warp's tokens; lane l holds elements EPL l .. EPL l + EPL - 1)
    {
      float o[TPW][EPL];
#pragma unroll
      for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
        for (int q = 0; q < EPL; ++q) o[tt][q] = 0.f;
      // positions of this warp's windows that hold this chunk's or earlier tokens of the
      // sequence (the others hold no value of it and have zero weight)
      const int xlo = max(max(0, i0 + kMaxWindow - w + 1), (int)max(0L, tb - pbase));
      const int xhi = min(min(RING - 1, i0 + TPW - 1 + kMaxWindow), n - 1 + kMaxWindow);
      int sl = slot0 + xlo;
      sl = sl >= RING ? sl - RING : sl;
#pragma unroll 2
      for (int x = xlo; x <= xhi; ++x) {
        float vv[EPL];
        if (EPL == 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(ring_v + sl * RS + EPL * lane);
          vv[0] = t4.x; vv[1] = t4.y; vv[EPL > 2 ? 2 : 0] = t4.z; vv[EPL > 3 ? 3 : 0] = t4.w;
        } else {
          const float2 t2 = *reinterpret_cast<const float2*>(ring_v + sl * RS + EPL * lane);
          vv[0] = t2.x; vv[1] = t2.y;
        }
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
          const float pr = sc[(i0 + tt) * RING + x];
#pragma unroll
          for (int q = 0; q < EPL; ++q) o[tt][q] = fmaf(pr, vv[q], o[tt][q]);
        }
        sl = sl + 1 == RING ? 0 : sl + 1;
      }
#pragma unroll
      for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
        for (int q = 0; q < EPL; ++q) qbuf[(i0 + tt) * D + EPL * lane + q] = o[tt][q];
    }
    // 4. token-serial recurrence on the register-resident state (no syncs): each thread
    //    updates its RPG x 4 tile in packed pairs, then the readout's partial sums over the
    //    row groups are added by a reduce-scatter among the NRG adjacent lanes (after it,
    //    each lane holds the total of one of the quad's four columns)
    {
      const int slot_c = (int)((t0 - tb) % RING);
      for (int i = 0; i < n; ++i) {
        const float g = VG ? 1.f : gate[i];
        int slot = slot_c + i;
        slot = slot >= RING ? slot - RING : slot;
        const float4 v4 = *reinterpret_cast<const float4*>(ring_v + slot * RS + 4 * cq);
        const float2 v01 = make_float2(v4.x, v4.y), v23 = make_float2(v4.z, v4.w);
        const float* fki = fk + i * FS + rg * RGS;
        const float* fqi = fq + i * FS + rg * RGS;
        const float* gvi = gvec + i * FS + rg * RGS;
        float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
        for (int r4 = 0; r4 < RPG; r4 += 4) {
          const float4 kf = *reinterpret_cast<const float4*>(fki + r4);
          const float4 qf = *reinterpret_cast<const float4*>(fqi + r4);
          const float4 gf = VG ? *reinterpret_cast<const float4*>(gvi + r4) : make_float4(g, g, g, g);
#pragma unroll
          for (int rr = 0; rr < 4; ++rr) {
            const float kr = rr == 0 ? kf.x : rr == 1 ? kf.y : rr == 2 ? kf.z : kf.w;
            const float qr = rr == 0 ? qf.x : rr == 1 ? qf.y : rr == 2 ? qf.z : qf.w;
            const float gr = rr == 0 ? gf.x : rr == 1 ? gf.y : rr == 2 ? gf.z : gf.w;
            const float2 k2 = make_float2(kr, kr), g2 = make_float2(gr, gr), q2 = make_float2(qr, qr);
            float4& sr = s[r4 + rr];
            const float2 s01 = sm100::ffma2(g2, make_float2(sr.x, sr.y), sm100::fmul2(k2, v01));
            const float2 s23 = sm100::ffma2(g2, make_float2(sr.z, sr.w), sm100::fmul2(k2, v23));
            sr = make_float4(s01.x, s01.y, s23.x, s23.y);
            a01 = sm100::ffma2(q2, s01, a01);
            a23 = sm100::ffma2(q2, s23, a23);
          }
        }
        // reduce-scatter over the row groups (lane bits below NRG)
        const bool up1 = (rg & (NRG / 2)) != 0;
        float2 keep = up1 ? a23 : a01;
        const float2 send = up1 ? a01 : a23;
        keep.x += __shfl_xor_sync(0xffffffffu, send.x, NRG / 2);
        keep.y += __shfl_xor_sync(0xffffffffu, send.y, NRG / 2);
        const bool up2 = (rg & (NRG / 4)) != 0;
        float t = (up2 ? keep.y : keep.x) + __shfl_xor_sync(0xffffffffu, up2 ? keep.x : keep.y, NRG / 4);
#pragma unroll
        for (int o = NRG / 8; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if ((rg & (NRG / 4 - 1)) == 0) grm[i * D + 4 * cq + (up1 ? 2 : 0) + (up2 ? 1 : 0)] = t;
      }
    }
    __syncthreads();
    // 5. mix and store
    for (int idx = tid; idx < n * D; idx += NT) {
      const int i = idx / D, e = idx % D;
      io<Tin>::st(out + ((size_t)(t0 + i) * Hq + h) * D + e, alpha * grm[idx] + beta * qbuf[idx]);
    }
    __syncthreads();
  }
  if (a.final_state && last) {
#pragma unroll
    for (int r = 0; r < RPG; ++r)
      *reinterpret_cast<float4*>(a.final_state + st_off + (size_t)(rg * RPG + r) * D + 4 * cq) = s[r];
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
