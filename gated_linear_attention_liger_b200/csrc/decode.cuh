// decode.cuh -- one decode step: a pure HBM stream over the fp32 states.
//
// One CTA per (sequence, q head).  Per step the dominant traffic is reading
// and writing that head's d x d fp32 state.  Each thread owns a 4-column slab
// of RPT key rows and issues all of its 128-bit streaming loads first; in the
// same breath the CTA starts copying the window ring's keys and values (the
// valid slots only) into shared memory with cp.async.  S <- g S + phi(k)^T v is
// applied to the registers and phi(q) S accumulated as soon as the rows land,
// and the rows stream back before the window branch runs on the shared-memory
// ring: the CTA's state traffic is done early, and its window work overlaps the
// other CTAs' streams.  The new key/value is
// taken from the step's inputs; the group's first q head writes it to slot
// pos mod w, a slot no other CTA of the step reads.  The position counter is
// advanced by a second one-thread-per-sequence kernel so that no CTA can see
// it half-updated.
//
// Recurrence and hybrid: "Liger: Linearizing Large Language Models to Gated
// Recurrent Structures" (Paper-Notes page), sections 统一的门控线性循环框架 and
// Liger Attention; constant-memory decoding: same page, section 亮点与洞察.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace liger {

using sm100::ffma2;
using sm100::fmul2;

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  float* state;
  void* ring;
  void* out;
  const int32_t* pos;
  int Hq, Hkv, w;
  float alpha;
  int vector_gate;   // one gate per key dimension, sigmoid(k[r]) on row r of the state
};

constexpr int kDecodeThreads = 256;

// Shared-memory ring rows are padded by 16 bytes so that rows sit 4 banks apart.
template <typename Tin, int D>
constexpr int ring_row_elems() {
  return D + 16 / (int)sizeof(Tin);
}
template <typename Tin, int D>
constexpr size_t decode_smem_bytes() {
  return sizeof(Tin) * 2 * 64 * ring_row_elems<Tin, D>();   // window ring keys and values
}

// Programmatic dependent launch: let the next kernel in the stream start
// launching now, and wait for the previous kernel's memory before touching it.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float4 ld_stream(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(float* p, float4 x) {
  __stcs(reinterpret_cast<float4*>(p), x);
}
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc)
               : "memory");
}


// Copies the window's ring rows (positions p-w+1 .. p-1, slot jj of the window =
// position p-(w-1)+jj) of one (sequence, kv head) into shared memory (padded rows):
// a flat loop over (row, 16-byte piece), no integer division in the loop.
template <typename Tin, int D, int NT>
__device__ __forceinline__ void ring_to_smem(const Tin* rk, const Tin* rv, Tin* rk_s, Tin* rv_s, int p, int w,
                                             int tid) {
  constexpr int CPR = D * (int)sizeof(Tin) / 16;   // a power of two
  constexpr int RS = ring_row_elems<Tin, D>();
  const int base = (p + 1) % w;   // slot of window position jj = 0
  for (int idx = tid; idx < 2 * w * CPR; idx += NT) {
    const int rowi = idx / CPR, piece = idx % CPR;
    const int which = rowi >= w ? 1 : 0;
    const int jj = rowi - which * w;
    const int j = p - (w - 1) + jj;
    if (j < 0 || j == p) continue;
    int slot = base + jj;
    slot = slot >= w ? slot - w : slot;
    const char* src = reinterpret_cast<const char*>((which ? rv : rk) + (size_t)slot * D);
    char* dst = reinterpret_cast<char*>((which ? rv_s : rk_s) + jj * RS);
    cp_async16(dst + piece * 16, src + piece * 16);
  }
}

// Unpack 16 bytes of ring row into floats.
template <typename Tin> __device__ __forceinline__ void ld16_vals(const Tin* p, float* x);
template <> __device__ __forceinline__ void ld16_vals<__nv_bfloat16>(const __nv_bfloat16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w4[i] << 16);
    x[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
  }
}
template <> __device__ __forceinline__ void ld16_vals<float>(const float* p, float* x) {
  const float4 u = *reinterpret_cast<const float4*>(p);
  x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
}

// Window scores q_h . k_j / sqrt(d) of NH heads for the w slots, four threads per
// slot; thread quarter qq takes the 16-byte pieces qq, qq+4, ... of the row, loads
// each key piece once for all heads and reduces with two shuffles.  qv[h] is head
// h's query row (fp32, 16-byte aligned).  Window position jj sits in shared-memory
// row (row0 + jj) mod wrap of stride RS elements (on unpadded rows the two rows of
// a quarter-warp share banks, a two-way conflict on the key loads only; the query
// loads, eight times as many, stay one wavefront each).  Needs blockDim >= 4 * w.
template <typename Tin, int D, int NH, int RS = ring_row_elems<Tin, D>()>
__device__ __forceinline__ void window_scores(const float (*qv)[D], const float* ks, const Tin* rk_s,
                                              float (*sc)[64], int p, int w, int tid, int row0 = 0,
                                              int wrap = 64) {
  constexpr int EPP = 16 / (int)sizeof(Tin);      // elements per 16-byte piece
  constexpr int NP = D / EPP;                     // pieces per row
  const int jj = tid >> 2, qq = tid & 3;
  if (jj < 64) {   // all four lanes of a slot take part in the shuffles
    const int j = p - (w - 1) + jj;
    const bool live = jj < w && j >= 0;
    int row = row0 + jj;
    row = row >= wrap ? row - wrap : row;
    float2 acc[NH];   // two partial sums (packed multiply-adds)
#pragma unroll
    for (int h = 0; h < NH; ++h) acc[h] = make_float2(0.f, 0.f);
    if (live) {
#pragma unroll
      for (int pc = qq; pc < NP; pc += 4) {
        float x[EPP];
        if (j == p) {
#pragma unroll
          for (int e = 0; e < EPP; e += 4) {
            const float4 t = *reinterpret_cast<const float4*>(ks + pc * EPP + e);
            x[e] = t.x; x[e + 1] = t.y; x[e + 2] = t.z; x[e + 3] = t.w;
          }
        } else {
          ld16_vals<Tin>(rk_s + row * RS + pc * EPP, x);
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) {
#pragma unroll
          for (int e = 0; e < EPP; e += 4) {
            const float4 qf = *reinterpret_cast<const float4*>(&qv[h][pc * EPP + e]);
            acc[h] = ffma2(make_float2(qf.x, qf.y), make_float2(x[e], x[e + 1]), acc[h]);
            acc[h] = ffma2(make_float2(qf.z, qf.w), make_float2(x[e + 2], x[e + 3]), acc[h]);
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float t = acc[h].x + acc[h].y;
      t += __shfl_xor_sync(0xffffffffu, t, 1);
      t += __shfl_xor_sync(0xffffffffu, t, 2);
      if (qq == 0 && jj < w) sc[h][jj] = live ? t * (1.0f / sqrtf((float)D)) : -INFINITY;
    }
  }
}

// Window softmax of head h = warp (warps 0 .. NH-1): the scores sc[h][0..w) (-inf for
// positions before the sequence start) become probabilities in place.
template <int NH>
__device__ __forceinline__ void window_probs(float (*sc)[64], int w, int warp, int lane) {
  if (warp < NH) {
    const float x0 = lane < w ? sc[warp][lane] : -INFINITY;
    const float x1 = lane + 32 < w ? sc[warp][lane + 32] : -INFINITY;
    const float m = warp_max(fmaxf(x0, x1));   // finite: the current position is always live
    const float e0 = lane < w ? expf(x0 - m) : 0.f;
    const float e1 = lane + 32 < w ? expf(x1 - m) : 0.f;
    const float iz = 1.0f / warp_sum(e0 + e1);
    if (lane < w) sc[warp][lane] = e0 * iz;
    if (lane + 32 < w) sc[warp][lane + 32] = e1 * iz;
  }
}

// Window softmax and value sums for NH heads.  sc[h][0..w) holds the scores (-inf
// for positions before the sequence start).  Every warp reduces the maxima and sums
// itself (no single-warp phase, no extra barrier).  Thread layout: 16-byte column
// piece cp = tid % NPC, slot group sg = tid / NPC, slots sg, sg + NSG, ...; each thread
// accumulates p_h(slot) v(slot) over its pieces, the slot groups of a warp are added
// with shuffles, and each warp writes wsum[warp][h][...]; the caller adds the NW
// partial sums.  Window position jj sits in row (row0 + jj) mod wrap of stride RS.
// With PROBS, sc already holds the probabilities (window_probs).
template <typename Tin, int D, int NT, int NH, int RS = ring_row_elems<Tin, D>(), bool PROBS = false>
struct WindowValues {
  static constexpr int EPP = 16 / (int)sizeof(Tin);   // elements per 16-byte piece
  static constexpr int NPC = D / EPP;                 // pieces per row
  static_assert(NPC <= 32 && 32 % NPC == 0, "a warp holds whole slot groups");
  static constexpr int NSG = NT / NPC;                // slot groups
  static constexpr int NW = NT / 32;                  // warps (partial sums)
  __device__ __forceinline__ static void run(const float (*sc)[64], const Tin* rv_s, const float* vs,
                                             float (*wsum)[NH][D], int p, int w, int tid, int lane,
                                             int row0 = 0, int wrap = 64) {
    float mh[NH], izh[NH];   // unused when sc already holds probabilities (PROBS)
#pragma unroll
    for (int h = 0; h < NH && !PROBS; ++h) {
      const float x0 = lane < w ? sc[h][lane] : -INFINITY;
      const float x1 = lane + 32 < w ? sc[h][lane + 32] : -INFINITY;
      const float m = warp_max(fmaxf(x0, x1));
      const float z = warp_sum((lane < w ? expf(x0 - m) : 0.f) + (lane + 32 < w ? expf(x1 - m) : 0.f));
      mh[h] = m;
      izh[h] = 1.0f / z;
    }
    const int cp = tid % NPC, sg = tid / NPC;
    float2 acc[NH][EPP / 2];   // element pairs (packed multiply-adds)
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int e = 0; e < EPP / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
#pragma unroll
    for (int it = 0; it < (64 + NSG - 1) / NSG; ++it) {
      const int jj = sg + it * NSG;
      const int j = p - (w - 1) + jj;
      if (jj >= w || j < 0) continue;
      float x[EPP];
      if (j == p) {
#pragma unroll
        for (int e = 0; e < EPP; ++e) x[e] = vs[cp * EPP + e];
      } else {
        int row = row0 + jj;
        row = row >= wrap ? row - wrap : row;
        ld16_vals<Tin>(rv_s + row * RS + cp * EPP, x);
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float ph = PROBS ? sc[h][jj] : expf(sc[h][jj] - mh[h]) * izh[h];
        const float2 ph2 = make_float2(ph, ph);
#pragma unroll
        for (int e = 0; e < EPP / 2; ++e) acc[h][e] = ffma2(ph2, make_float2(x[2 * e], x[2 * e + 1]), acc[h][e]);
      }
    }
#pragma unroll
    for (int o = NPC; o < 32; o <<= 1)
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int e = 0; e < EPP / 2; ++e) {
          acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, o);
          acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, o);
        }
    if (lane < NPC) {
#pragma unroll
      for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int e = 0; e < EPP / 2; e += 2)
          *reinterpret_cast<float4*>(&wsum[tid >> 5][h][cp * EPP + 2 * e]) =
              make_float4(acc[h][e].x, acc[h][e].y, acc[h][e + 1].x, acc[h][e + 1].y);
    }
  }
};

template <typename Tin, int D>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_kernel(DecodeArgs a) {
  constexpr int NT = kDecodeThreads;
  constexpr int CQ = D / 4;          // column quads
  constexpr int RGN = NT / CQ;       // row groups
  constexpr int RPT = D / RGN;       // rows per thread
  constexpr int EPL = D / 32;
  using WV = WindowValues<Tin, D, NT, 1>;
  extern __shared__ __align__(16) unsigned char dsm[];
  Tin* rk_s = reinterpret_cast<Tin*>(dsm);          // [64][D]
  Tin* rv_s = rk_s + 64 * ring_row_elems<Tin, D>();  // [64][row]
  __shared__ __align__(16) float qs[D], ks[D], vs[D], fq[D], fk[D], gv[D];
  __shared__ float sc[1][64];
  __shared__ __align__(16) float part[RGN][D];
  __shared__ __align__(16) float wsum[WV::NW][1][D];
  __shared__ float gsh;

  const int Hq = a.Hq, Hkv = a.Hkv, w = a.w, G = Hq / Hkv;
  const int b = blockIdx.x / Hq, h = blockIdx.x % Hq, kv = h / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid % CQ, rg = tid / CQ;

  pdl_wait();
  pdl_launch_dependents();
  // 1. the state rows this thread updates: all loads in flight at once
  float* S = a.state + ((size_t)b * Hq + h) * D * D;
  float4 st[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) st[r] = ld_stream(S + (size_t)(rg * RPT + r) * D + 4 * cq);

  // 2. the window's ring slots (positions p-w+1 .. p-1) start towards shared memory;
  //    they are waited for only after the state has streamed back
  const int p = max(a.pos[b], 0);   // a negative position is read as 0
  Tin* ring = static_cast<Tin*>(a.ring);
  const Tin* rk = ring + (((size_t)b * Hkv + kv) * 2 + 0) * w * D;
  const Tin* rv = ring + (((size_t)b * Hkv + kv) * 2 + 1) * w * D;
  ring_to_smem<Tin, D, NT>(rk, rv, rk_s, rv_s, p, w, tid);
  asm volatile("cp.async.commit_group;" ::: "memory");
  const Tin* qrow = static_cast<const Tin*>(a.q) + ((size_t)b * Hq + h) * D;
  const Tin* krow = static_cast<const Tin*>(a.k) + ((size_t)b * Hkv + kv) * D;
  const Tin* vrow = static_cast<const Tin*>(a.v) + ((size_t)b * Hkv + kv) * D;
  if (tid < D) {
    qs[tid] = io<Tin>::ld(qrow + tid);
    ks[tid] = io<Tin>::ld(krow + tid);
    vs[tid] = io<Tin>::ld(vrow + tid);
  }
  __syncthreads();

  // 3. phi(k) with the gate, and phi(q)
  if (warp == 0) {
    float x[EPL], m = -INFINITY, sum = 0.f, z = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = ks[lane + 32 * j]; m = fmaxf(m, x[j]); sum += x[j]; }
    m = warp_max(m);
    sum = warp_sum(sum);
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
    z = warp_sum(z);
#pragma unroll
    for (int j = 0; j < EPL; ++j) fk[lane + 32 * j] = x[j] / z;
    if (lane == 0) gsh = expf(log_sigmoid(sum / (float)D));
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      gv[lane + 32 * j] = a.vector_gate ? expf(log_sigmoid(ks[lane + 32 * j])) : 0.f;
  } else if (warp == 1) {
    float x[EPL], m = -INFINITY, z = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = qs[lane + 32 * j]; m = fmaxf(m, x[j]); }
    m = warp_max(m);
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
    z = warp_sum(z);
#pragma unroll
    for (int j = 0; j < EPL; ++j) fq[lane + 32 * j] = x[j] / z;
  }
  __syncthreads();

  // 4. state update and readout on the streamed rows: the state goes back to memory
  //    before the window branch is computed
  {
    const float gs = gsh;
    const bool vg = a.vector_gate != 0;
    const float4 vv = *reinterpret_cast<const float4*>(vs + 4 * cq);
    const float2 v01 = make_float2(vv.x, vv.y), v23 = make_float2(vv.z, vv.w);
    float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int row = rg * RPT + r;
      const float kr = fk[row], qr = fq[row];
      const float g = vg ? gv[row] : gs;
      const float2 g2 = make_float2(g, g), k2 = make_float2(kr, kr), q2 = make_float2(qr, qr);
      const float2 x01 = ffma2(g2, make_float2(st[r].x, st[r].y), fmul2(k2, v01));
      const float2 x23 = ffma2(g2, make_float2(st[r].z, st[r].w), fmul2(k2, v23));
      a01 = ffma2(q2, x01, a01);
      a23 = ffma2(q2, x23, a23);
      st_stream(S + (size_t)row * D + 4 * cq, make_float4(x01.x, x01.y, x23.x, x23.y));
    }
    *reinterpret_cast<float4*>(&part[rg][4 * cq]) = make_float4(a01.x, a01.y, a23.x, a23.y);
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // 5. window scores from shared memory (slot jj covers position p - (w-1) + jj)
  window_scores<Tin, D, 1>(reinterpret_cast<const float(*)[D]>(qs), ks, rk_s, sc, p, w, tid);
  __syncthreads();
  // 6. window softmax and value sums
  WV::run(sc, rv_s, vs, wsum, p, w, tid, lane);
  __syncthreads();
  if (tid < D) {
    float grm = 0.f, swa = 0.f;
#pragma unroll
    for (int r = 0; r < RGN; ++r) grm += part[r][tid];
#pragma unroll
    for (int r = 0; r < WV::NW; ++r) swa += wsum[r][0][tid];
    Tin* orow = static_cast<Tin*>(a.out) + ((size_t)b * Hq + h) * D;
    io<Tin>::st(orow + tid, a.alpha * grm + (1.0f - a.alpha) * swa);
    if (h % G == 0) {
      Tin* wk = ring + (((size_t)b * Hkv + kv) * 2 + 0) * w * D + (size_t)(p % w) * D;
      Tin* wv = ring + (((size_t)b * Hkv + kv) * 2 + 1) * w * D + (size_t)(p % w) * D;
      wk[tid] = krow[tid];
      wv[tid] = vrow[tid];
    }
  }
}

__global__ void advance_pos_kernel(int32_t* pos, int B) {
  pdl_wait();   // every CTA of the decode kernel has read pos
  pdl_launch_dependents();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) pos[b] += 1;
}

}  // namespace liger

namespace liger {

// Decode over one state per (sequence, kv head): state [B, Hkv, d, d].  The q
// heads of a group read the same state -- prefill writes identical copies and
// a per-head decode keeps them identical -- so one CTA per (sequence, kv head)
// streams that state once, applies S <- g S + phi(k)^T v once, and forms
// o_h = alpha phi(q_h) S + (1 - alpha) window_h for each of the G heads.  The
// fp32 state traffic per step drops by G.
template <typename Tin, int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_kvshared_kernel(DecodeArgs a) {
  constexpr int NT = kDecodeThreads;
  constexpr int CQ = D / 4;
  constexpr int RGN = NT / CQ;
  constexpr int RPT = D / RGN;
  constexpr int EPL = D / 32;
  using WV = WindowValues<Tin, D, NT, G>;
  extern __shared__ __align__(16) unsigned char dsm[];
  Tin* rk_s = reinterpret_cast<Tin*>(dsm);          // [64][D]
  Tin* rv_s = rk_s + 64 * ring_row_elems<Tin, D>();  // [64][row]
  __shared__ __align__(16) float qs[G][D], fq[G][D], ks[D], vs[D], fk[D];
  __shared__ float sc[G][64];
  __shared__ __align__(16) float part[RGN][G][D];
  __shared__ __align__(16) float wsum[WV::NW][G][D];
  __shared__ float gsh;

  const int Hkv = a.Hkv, w = a.w, Hq = a.Hq;
  const int b = blockIdx.x / Hkv, kv = blockIdx.x % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid % CQ, rg = tid / CQ;

  pdl_wait();
  pdl_launch_dependents();
  float* S = a.state + ((size_t)b * Hkv + kv) * D * D;
  float4 st[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) st[r] = ld_stream(S + (size_t)(rg * RPT + r) * D + 4 * cq);

  // the ring rows start towards shared memory; waited for after the state has streamed back
  const int p = max(a.pos[b], 0);
  Tin* ring = static_cast<Tin*>(a.ring);
  const Tin* rk = ring + (((size_t)b * Hkv + kv) * 2 + 0) * w * D;
  const Tin* rv = ring + (((size_t)b * Hkv + kv) * 2 + 1) * w * D;
  ring_to_smem<Tin, D, NT>(rk, rv, rk_s, rv_s, p, w, tid);
  asm volatile("cp.async.commit_group;" ::: "memory");
  const Tin* krow = static_cast<const Tin*>(a.k) + ((size_t)b * Hkv + kv) * D;
  const Tin* vrow = static_cast<const Tin*>(a.v) + ((size_t)b * Hkv + kv) * D;
  for (int idx = tid; idx < G * D; idx += NT) {
    const int hh = idx / D, e = idx % D;
    qs[hh][e] = io<Tin>::ld(static_cast<const Tin*>(a.q) + ((size_t)b * Hq + kv * G + hh) * D + e);
  }
  if (tid < D) {
    ks[tid] = io<Tin>::ld(krow + tid);
    vs[tid] = io<Tin>::ld(vrow + tid);
  }
  __syncthreads();

  // phi(k) with the gate (warp 0), phi(q_h) (warps 1..G)
  if (warp == 0) {
    float x[EPL], m = -INFINITY, sum = 0.f, z = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = ks[lane + 32 * j]; m = fmaxf(m, x[j]); sum += x[j]; }
    m = warp_max(m);
    sum = warp_sum(sum);
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
    z = warp_sum(z);
#pragma unroll
    for (int j = 0; j < EPL; ++j) fk[lane + 32 * j] = x[j] / z;
    if (lane == 0) gsh = expf(log_sigmoid(sum / (float)D));
  } else if (warp <= G) {
    const int hh = warp - 1;
    float x[EPL], m = -INFINITY, z = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = qs[hh][lane + 32 * j]; m = fmaxf(m, x[j]); }
    m = warp_max(m);
#pragma unroll
    for (int j = 0; j < EPL; ++j) { x[j] = expf(x[j] - m); z += x[j]; }
    z = warp_sum(z);
#pragma unroll
    for (int j = 0; j < EPL; ++j) fq[hh][lane + 32 * j] = x[j] / z;
  }
  __syncthreads();

  // state update once, readout for every head of the group; the state goes back to
  // memory before the window branch is computed
  {
    const float g = gsh;
    const float4 vv = *reinterpret_cast<const float4*>(vs + 4 * cq);
    const float2 g2 = make_float2(g, g), v01 = make_float2(vv.x, vv.y), v23 = make_float2(vv.z, vv.w);
    float2 a01[G], a23[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) a01[hh] = a23[hh] = make_float2(0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int row = rg * RPT + r;
      const float kr = fk[row];
      const float2 k2 = make_float2(kr, kr);
      const float2 x01 = ffma2(g2, make_float2(st[r].x, st[r].y), fmul2(k2, v01));
      const float2 x23 = ffma2(g2, make_float2(st[r].z, st[r].w), fmul2(k2, v23));
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float qr = fq[hh][row];
        const float2 q2 = make_float2(qr, qr);
        a01[hh] = ffma2(q2, x01, a01[hh]);
        a23[hh] = ffma2(q2, x23, a23[hh]);
      }
      st_stream(S + (size_t)row * D + 4 * cq, make_float4(x01.x, x01.y, x23.x, x23.y));
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
      *reinterpret_cast<float4*>(&part[rg][hh][4 * cq]) = make_float4(a01[hh].x, a01[hh].y, a23[hh].x, a23[hh].y);
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // window scores, head by head
  window_scores<Tin, D, G>(qs, ks, rk_s, sc, p, w, tid);
  __syncthreads();
  WV::run(sc, rv_s, vs, wsum, p, w, tid, lane);   // window softmax and value sums
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += NT) {
    const int hh = idx / D, e = idx % D;
    float grm = 0.f, swa = 0.f;
#pragma unroll
    for (int r = 0; r < RGN; ++r) grm += part[r][hh][e];
#pragma unroll
    for (int r = 0; r < WV::NW; ++r) swa += wsum[r][hh][e];
    Tin* orow = static_cast<Tin*>(a.out) + ((size_t)b * Hq + kv * G + hh) * D;
    io<Tin>::st(orow + e, a.alpha * grm + (1.0f - a.alpha) * swa);
  }
  if (tid < D) {
    Tin* wk = ring + (((size_t)b * Hkv + kv) * 2 + 0) * w * D + (size_t)(p % w) * D;
    Tin* wv = ring + (((size_t)b * Hkv + kv) * 2 + 1) * w * D + (size_t)(p % w) * D;
    wk[tid] = krow[tid];
    wv[tid] = vrow[tid];
  }
}

}  // namespace liger

namespace liger {
namespace kvs {

// Decode as a persistent stream.  One CTA per SM walks the units blockIdx.x,
// blockIdx.x + gridDim.x, ...: (sequence, kv head) with one state read out by the
// group's G heads (NH = G), or (sequence, q head) with a state per head (NH = 1,
// PER_HEAD; the group's heads read the same window ring, and the group's first
// head writes the step's key and value into it).  A producer warp moves each
// unit's fp32 state, its window ring (keys, then values, w slots each, in slot
// order) and the step's rows q_h (NH of them), k and v into one of two
// shared-memory stages by bulk copies, so that the next unit's bytes are in
// flight while eight consumer warps compute this one; one or two feature warps
// prepare each unit's feature maps and gates ahead of them.  The updated state goes
// back to HBM by bulk copies as soon as the consumers have written it, before
// they run the window branch.  Every wait is bounded; a wait that gives up
// records the timeout in the device error word and the CTA winds down with no
// copy in flight.

constexpr int kConsumers = 256;               // eight consumer warps
// feature warps: the key and half of the queries on one, the other queries on a second
template <int G>
constexpr int feature_warps() { return G >= 2 ? 2 : 1; }
template <int G>
constexpr int threads() { return kConsumers + 32 + 32 * feature_warps<G>(); }   // + producer, features
constexpr int kStages = 2;

template <typename Tin, int D, int G>   // G: heads read out per unit
struct Layout {
  static constexpr uint32_t STATE = D * D * 4;
  static constexpr uint32_t RING = 2 * 64 * D * sizeof(Tin);    // room for w = 64
  static constexpr uint32_t QKV = (G + 2) * D * sizeof(Tin);     // q_0 .. q_{G-1}, k, v
  static constexpr uint32_t STAGE = STATE + RING + QKV;
  static constexpr int CQ = D / 4;                  // column quads
  static constexpr int RGN = kConsumers / CQ;       // row groups
  static constexpr int RPT = D / RGN;               // rows per thread
  using WV = WindowValues<Tin, D, kConsumers, G, D, true>;
  static constexpr uint32_t PART = RGN * G * D * 4;              // readout partial sums
  static constexpr uint32_t WSUM = WV::NW * G * D * 4;           // window partial sums (same room)
  static constexpr uint32_t SCRATCH = PART > WSUM ? PART : WSUM;
  // per stage, written by the feature warps: phi(q_h) [G][D], q_h in fp32 [G][D], phi(k),
  // k and v in fp32, the per-row gates [D] each, the scalar gate
  // (q_h, k and v in fp32 are contiguous: one converted copy of the stage's rows)
  static constexpr uint32_t F_FQ = 0, F_FK = F_FQ + G * D * 4, F_GV = F_FK + D * 4;
  static constexpr uint32_t F_QF = F_GV + D * 4, F_KS = F_QF + G * D * 4, F_VS = F_KS + D * 4;
  static constexpr uint32_t F_G = F_VS + D * 4;
  static constexpr uint32_t FEAT = F_G + 16;
  static constexpr uint32_t OFF_SCRATCH = kStages * STAGE;
  static constexpr uint32_t OFF_FEAT = OFF_SCRATCH + SCRATCH;    // kStages feature buffers
  static constexpr uint32_t OFF_GRM = OFF_FEAT + kStages * FEAT; // [G][D] recurrent readout
  static constexpr uint32_t OFF_SC = OFF_GRM + G * D * 4;        // [G][64] window scores
  static constexpr uint32_t OFF_MISC = OFF_SC + G * 64 * 4;      // barriers, positions, abort
  static constexpr uint32_t BYTES = OFF_MISC + 128;
  static_assert(STAGE % 16 == 0 && STATE % 4096 == 0 && FEAT % 16 == 0, "16-byte pieces");
  static_assert(RGN * RPT == D && RPT >= 1, "row split");
};

// Whether the two stages fit one CTA's shared memory (fp32 rows at d = 128 do not).
template <typename Tin, int D, int G>
constexpr bool fits() {
  return Layout<Tin, D, G>::BYTES <= 227u * 1024u;
}

// A lane's EPL consecutive floats (EPL = 2 or 4) in one shared-memory access.
template <int EPL>
__device__ __forceinline__ void lane_slice_ld(const float* p, float* x) {
  if constexpr (EPL == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  } else {
    static_assert(EPL == 2, "d = 64 or 128");
    const float2 t = *reinterpret_cast<const float2*>(p);
    x[0] = t.x; x[1] = t.y;
  }
}
template <int EPL>
__device__ __forceinline__ void lane_slice_st(float* p, const float* x) {
  if constexpr (EPL == 4) *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  else *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}

struct Args {
  DecodeArgs d;
  int units;           // B * Hkv, or B * Hq per head
  uint32_t* err;       // device error word (timeouts)
  uint64_t wait_ns;    // give-up time of each wait
};

// Offsets (in elements) of one unit's rows.
struct UnitRows {
  size_t state, ring, q, kv;   // q: the first of the unit's q rows (also its first out row)
  bool writes_ring;
};
template <int G, bool PER_HEAD>
__device__ __forceinline__ UnitRows unit_rows(long u, int Hq, int Hkv, int D, int w) {
  UnitRows r;
  if (PER_HEAD) {
    const long b = u / Hq, h = u % Hq, grp = Hq / Hkv;
    const long kvi = b * Hkv + h / grp;
    r.state = (size_t)u * D * D;
    r.ring = (size_t)kvi * 2 * w * D;
    r.q = (size_t)u * D;
    r.kv = (size_t)kvi * D;
    r.writes_ring = h % grp == 0;
  } else {
    const long b = u / Hkv, kv = u % Hkv;
    r.state = (size_t)u * D * D;
    r.ring = (size_t)u * 2 * w * D;
    r.q = ((size_t)b * Hq + kv * G) * D;
    r.kv = (size_t)u * D;
    r.writes_ring = true;
  }
  return r;
}

template <typename Tin, int D, int G, bool PER_HEAD>
__global__ void __launch_bounds__(threads<G>(), 1) decode_stream_kernel(Args c) {
  static_assert(!PER_HEAD || G == 1, "a per-head unit reads out one head");
  using L = Layout<Tin, D, G>;
  using sm100::mbar_wait;
  extern __shared__ __align__(128) unsigned char sm[];
  float* grm = reinterpret_cast<float*>(sm + L::OFF_GRM);
  float(*sc)[64] = reinterpret_cast<float(*)[64]>(sm + L::OFF_SC);
  float(*part)[G][D] = reinterpret_cast<float(*)[G][D]>(sm + L::OFF_SCRATCH);
  float(*wsum)[G][D] = reinterpret_cast<float(*)[G][D]>(sm + L::OFF_SCRATCH);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::OFF_MISC);   // [2] ring and q/k/v loaded
  uint64_t* sdone = full + 2;                                        // [2] state updated in place
  uint64_t* cons = full + 4;                                         // [2] stage no longer read
  uint64_t* featb = full + 6;                                        // [2] stage's features written
  uint64_t* fullS = full + 8;                                        // [2] state loaded
  int* pos_s = reinterpret_cast<int*>(full + 10);                    // [2]
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(pos_s + 2);

  const DecodeArgs& a = c.d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hkv = a.Hkv, Hq = a.Hq, w = a.w;
  const uint32_t ring_bytes = 2u * (uint32_t)w * D * sizeof(Tin);
  auto stage = [&](int s) { return sm + (size_t)s * L::STAGE; };
  auto feat = [&](int s, uint32_t off) { return reinterpret_cast<float*>(sm + L::OFF_FEAT + s * L::FEAT + off); };
  constexpr int EPL = D / 32;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&sdone[s], kConsumers);
      sm100::mbar_init(&cons[s], kConsumers);
      sm100::mbar_init(&featb[s], 32 * feature_warps<G>());
      sm100::mbar_init(&fullS[s], 1);
    }
    *abort_flag = 0u;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  const sm100::WaitCtx wc{abort_flag, c.err, c.wait_ns};
  const int n_local = c.units > (int)blockIdx.x ? (c.units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == kConsumers / 32) {
    // ---------------------------------------------------------------- producer
    if (lane != 0) return;
    // the state part of a stage is reloaded as soon as the previous unit's state has
    // left it (mid-unit); the ring and q/k/v part once the consumers release the stage
    auto issue_state = [&](int i) {
      const int s = i % kStages;
      const long u = (long)blockIdx.x + (long)i * gridDim.x;
      const float* S = a.state + unit_rows<G, PER_HEAD>(u, Hq, Hkv, D, w).state;
      sm100::mbar_arrive_expect_tx(&fullS[s], L::STATE);
#pragma unroll
      for (int piece = 0; piece < 4; ++piece)
        sm100::bulk_load(stage(s) + piece * (L::STATE / 4), S + piece * (D * D / 4), L::STATE / 4, &fullS[s]);
    };
    auto issue = [&](int i) {
      const int s = i % kStages;
      const long u = (long)blockIdx.x + (long)i * gridDim.x;
      const UnitRows r = unit_rows<G, PER_HEAD>(u, Hq, Hkv, D, w);
      unsigned char* st = stage(s);
      pos_s[s] = max(a.pos[u / (PER_HEAD ? Hq : Hkv)], 0);   // a negative position is read as 0
      sm100::mbar_arrive_expect_tx(&full[s], ring_bytes + L::QKV);
      sm100::bulk_load(st + L::STATE, static_cast<const Tin*>(a.ring) + r.ring, ring_bytes, &full[s]);
      unsigned char* qkv = st + L::STATE + L::RING;
      sm100::bulk_load(qkv, static_cast<const Tin*>(a.q) + r.q, G * D * sizeof(Tin), &full[s]);
      sm100::bulk_load(qkv + G * D * sizeof(Tin), static_cast<const Tin*>(a.k) + r.kv, D * sizeof(Tin), &full[s]);
      sm100::bulk_load(qkv + (G + 1) * D * sizeof(Tin), static_cast<const Tin*>(a.v) + r.kv, D * sizeof(Tin),
                       &full[s]);
    };
    int issued = 0, issued_state = 0;   // units whose ring and q/k/v (state) copies are issued
    for (; issued < kStages && issued < n_local; ++issued, ++issued_state) {
      issue_state(issued);
      issue(issued);
    }
    for (int i = 0; i < n_local; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (uint32_t)(i / kStages) & 1u;
      if (!mbar_wait(&sdone[s], ph, wc, sm100::wsite(7, 1, i))) break;
      const long u = (long)blockIdx.x + (long)i * gridDim.x;
      float* S = a.state + (size_t)u * D * D;
#pragma unroll
      for (int piece = 0; piece < 4; ++piece)
        sm100::bulk_store(S + piece * (D * D / 4), stage(s) + piece * (L::STATE / 4), L::STATE / 4);
      sm100::bulk_commit();
      if (i + kStages < n_local) {
        sm100::bulk_wait_read_all();   // this unit's state has left the stage
        issue_state(issued_state++);
        if (!mbar_wait(&cons[s], ph, wc, sm100::wsite(7, 2, i))) break;
        issue(issued++);
      }
    }
    // never leave with copies in flight: the last load of each stage, then the stores
    volatile uint32_t never = 0u;
    const sm100::WaitCtx drain{&never, nullptr, c.wait_ns};
    for (int i = issued_state > kStages ? issued_state - kStages : 0; i < issued_state; ++i)
      mbar_wait(&fullS[i % kStages], (uint32_t)(i / kStages) & 1u, drain);
    for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
      mbar_wait(&full[i % kStages], (uint32_t)(i / kStages) & 1u, drain);
    sm100::bulk_wait_all();
    return;
  }

  if (warp > kConsumers / 32) {
    // ---------------------------------------------------------------- features
    // phi(k), the gate(s) and phi(q_h) of each unit, and fp32 copies of its q, k and v,
    // into the stage's feature buffer, one unit ahead of the consumers where the copies
    // allow.  Feature row 0 is the key (with the gates and the copy of v), rows 1..G the
    // queries; with two feature warps the first takes rows 0 .. G/2, the second the rest,
    // each converting the rows it reads.  The buffer of stage s is rewritten only after
    // the producer has reloaded stage s, i.e. after the consumers have released it.
    constexpr int EPP = 16 / (int)sizeof(Tin), PPR = D / EPP;
    auto feature_rows = [&](int s, auto r0c, auto r1c) {
      constexpr int R0 = decltype(r0c)::value, R1 = decltype(r1c)::value, NR = R1 - R0;
      constexpr int Q0 = R0 > 0 ? R0 : 1;   // first query row of this warp
      const Tin* qin = reinterpret_cast<const Tin*>(stage(s) + L::STATE + L::RING);
      float* rows = feat(s, L::F_QF);       // q rows, then k, then v (as in the stage)
      // fp32 copies, 16 bytes a step: this warp's query rows, and k and v with the key
      for (int pc = (Q0 - 1) * PPR + lane; pc < (R1 - 1) * PPR; pc += 32) {
        float xv[EPP];
        ld16_vals<Tin>(qin + pc * EPP, xv);
#pragma unroll
        for (int e = 0; e < EPP; e += 4)
          *reinterpret_cast<float4*>(rows + pc * EPP + e) = make_float4(xv[e], xv[e + 1], xv[e + 2], xv[e + 3]);
      }
      if (R0 == 0) {
        for (int pc = G * PPR + lane; pc < (G + 2) * PPR; pc += 32) {
          float xv[EPP];
          ld16_vals<Tin>(qin + pc * EPP, xv);
#pragma unroll
          for (int e = 0; e < EPP; e += 4)
            *reinterpret_cast<float4*>(rows + pc * EPP + e) = make_float4(xv[e], xv[e + 1], xv[e + 2], xv[e + 3]);
        }
      }
      __syncwarp();
      // one softmax over d per row, EPL consecutive elements per lane
      float x[NR][EPL], m[NR], z[NR], sum = 0.f;
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) {
        const int r = R0 + rr;
        const float* src = (r == 0 ? rows + G * D : rows + (r - 1) * D) + lane * EPL;
        m[rr] = -INFINITY;
        z[rr] = 0.f;
        lane_slice_ld<EPL>(src, x[rr]);
#pragma unroll
        for (int j = 0; j < EPL; ++j) m[rr] = fmaxf(m[rr], x[rr][j]);
      }
      if (R0 == 0) {
        if (PER_HEAD && a.vector_gate) {
          float* gv = feat(s, L::F_GV) + lane * EPL;
#pragma unroll
          for (int j = 0; j < EPL; ++j) gv[j] = expf(log_sigmoid(x[0][j]));
        }
#pragma unroll
        for (int j = 0; j < EPL; ++j) sum += x[0][j];
        sum = warp_sum(sum);
      }
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) m[rr] = warp_max(m[rr]);
#pragma unroll
      for (int rr = 0; rr < NR; ++rr)
#pragma unroll
        for (int j = 0; j < EPL; ++j) { x[rr][j] = expf(x[rr][j] - m[rr]); z[rr] += x[rr][j]; }
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) z[rr] = warp_sum(z[rr]);
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) {
        const int r = R0 + rr;
        float* dst = (r == 0 ? feat(s, L::F_FK) : feat(s, L::F_FQ) + (r - 1) * D) + lane * EPL;
        float y[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) y[j] = x[rr][j] / z[rr];
        lane_slice_st<EPL>(dst, y);
      }
      if (R0 == 0 && lane == 0) *feat(s, L::F_G) = expf(log_sigmoid(sum / (float)D));
    };
    constexpr int RSPLIT = feature_warps<G>() == 2 ? 1 + G / 2 : G + 1;   // rows of the first warp
    const int fw = warp - kConsumers / 32 - 1;
    for (int i = 0; i < n_local; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (uint32_t)(i / kStages) & 1u;
      if (!sm100::warp_all(mbar_wait(&full[s], ph, wc, sm100::wsite(8, 1 + fw, i)))) break;
      if (fw == 0) {
        feature_rows(s, std::integral_constant<int, 0>{}, std::integral_constant<int, RSPLIT>{});
      } else if constexpr (feature_warps<G>() == 2) {
        feature_rows(s, std::integral_constant<int, RSPLIT>{}, std::integral_constant<int, G + 1>{});
      }
      sm100::mbar_arrive(&featb[s]);   // every lane: its own writes are released
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int cq = tid % L::CQ, rg = tid / L::CQ;
  for (int i = 0; i < n_local; ++i) {
    const int s = i % kStages;
    const uint32_t ph = (uint32_t)(i / kStages) & 1u;
    const bool ok = mbar_wait(&featb[s], ph, wc, sm100::wsite(6, 1, i)) &&
                    mbar_wait(&fullS[s], ph, wc, sm100::wsite(6, 2, i));
    if (sm100::named_bar_or(1, kConsumers, !ok)) break;
    const long u = (long)blockIdx.x + (long)i * gridDim.x;
    const UnitRows ur = unit_rows<G, PER_HEAD>(u, Hq, Hkv, D, w);
    unsigned char* st = stage(s);
    float* Ss = reinterpret_cast<float*>(st);
    const Tin* rk = reinterpret_cast<const Tin*>(st + L::STATE);
    const Tin* rv = rk + (size_t)w * D;
    const Tin* kin = reinterpret_cast<const Tin*>(st + L::STATE + L::RING) + G * D;
    const Tin* vin = kin + D;
    const float* fq = feat(s, L::F_FQ);
    const float* qf = feat(s, L::F_QF);
    const float* fk = feat(s, L::F_FK);
    const float* ks = feat(s, L::F_KS);
    const float* vs = feat(s, L::F_VS);
    const float* gv = feat(s, L::F_GV);
    const int p = pos_s[s];

    // state update in place, readout for every head of the group; the producer sends
    // the state back as soon as every consumer has written its rows
    {
      const bool vgate = PER_HEAD && a.vector_gate;
      const float g = *feat(s, L::F_G);
      const float4 vv = *reinterpret_cast<const float4*>(vs + 4 * cq);
      const float2 v01 = make_float2(vv.x, vv.y), v23 = make_float2(vv.z, vv.w);
      float2 a01[G], a23[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) a01[hh] = a23[hh] = make_float2(0.f, 0.f);
      static_assert(L::RPT % 4 == 0, "rows in quads");
#pragma unroll
      for (int r4 = 0; r4 < L::RPT; r4 += 4) {
        const int row4 = rg * L::RPT + r4;
        const float4 k4 = *reinterpret_cast<const float4*>(fk + row4);   // phi(k) of four rows
        const float4 g4 = vgate ? *reinterpret_cast<const float4*>(gv + row4) : make_float4(g, g, g, g);
        float4 q4[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) q4[hh] = *reinterpret_cast<const float4*>(fq + hh * D + row4);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float4* sp = reinterpret_cast<float4*>(Ss + (size_t)(row4 + r) * D + 4 * cq);
          const float4 sv = *sp;
          const float kr = r == 0 ? k4.x : r == 1 ? k4.y : r == 2 ? k4.z : k4.w;
          const float gr = r == 0 ? g4.x : r == 1 ? g4.y : r == 2 ? g4.z : g4.w;
          const float2 k2 = make_float2(kr, kr), g2 = make_float2(gr, gr);
          const float2 x01 = ffma2(g2, make_float2(sv.x, sv.y), fmul2(k2, v01));
          const float2 x23 = ffma2(g2, make_float2(sv.z, sv.w), fmul2(k2, v23));
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float qr = r == 0 ? q4[hh].x : r == 1 ? q4[hh].y : r == 2 ? q4[hh].z : q4[hh].w;
            const float2 q2 = make_float2(qr, qr);
            a01[hh] = ffma2(q2, x01, a01[hh]);
            a23[hh] = ffma2(q2, x23, a23[hh]);
          }
          *sp = make_float4(x01.x, x01.y, x23.x, x23.y);
        }
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
        *reinterpret_cast<float4*>(&part[rg][hh][4 * cq]) = make_float4(a01[hh].x, a01[hh].y, a23[hh].x, a23[hh].y);
    }
    sm100::fence_proxy_async_smem();   // the rows written above are read by the bulk copy out
    sm100::mbar_arrive(&sdone[s]);

    // window scores on the ring in slot order (window position jj is slot (p+1+jj) mod w);
    // they read only this phase's inputs, so no barrier separates them from the update
    const int row0 = (p + 1) % w;
    window_scores<Tin, D, G, D>(reinterpret_cast<const float(*)[D]>(qf), ks, rk, sc, p, w, tid, row0, w);
    sm100::named_bar(1, kConsumers);
    // window softmax, one warp per head; the other warps add up the readout partial sums
    if (warp < G) {
      window_probs<G>(sc, w, warp, lane);
    } else {
      for (int idx = tid - 32 * G; idx < G * D; idx += kConsumers - 32 * G) {
        float t = 0.f;
#pragma unroll
        for (int r = 0; r < L::RGN; ++r) t += part[r][idx / D][idx % D];
        grm[idx] = t;
      }
    }
    sm100::named_bar(1, kConsumers);
    L::WV::run(sc, rv, vs, wsum, p, w, tid, lane, row0, w);   // window value sums
    sm100::named_bar(1, kConsumers);
    for (int idx = tid; idx < G * D; idx += kConsumers) {
      const int hh = idx / D, e = idx % D;
      float swa = 0.f;
#pragma unroll
      for (int r = 0; r < L::WV::NW; ++r) swa += wsum[r][hh][e];
      Tin* orow = static_cast<Tin*>(a.out) + ur.q + (size_t)hh * D;
      io<Tin>::st(orow + e, a.alpha * grm[idx] + (1.0f - a.alpha) * swa);
    }
    // the step's key and value replace the oldest slot of this unit's ring (no unit of
    // the step reads that slot: it holds the position that just left every window)
    constexpr int PC = D * (int)sizeof(Tin) / 16;   // 16-byte pieces per row
    if (ur.writes_ring && tid < 2 * PC) {
      const int which = tid / PC, piece = tid % PC;
      Tin* dst = static_cast<Tin*>(a.ring) + ur.ring + (size_t)which * w * D + (size_t)(p % w) * D;
      const Tin* src = which ? vin : kin;
      reinterpret_cast<uint4*>(dst)[piece] = reinterpret_cast<const uint4*>(src)[piece];
    }
    sm100::mbar_arrive(&cons[s]);
  }
}

}  // namespace kvs
}  // namespace liger
