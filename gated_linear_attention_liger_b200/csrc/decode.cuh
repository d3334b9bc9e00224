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
// slot; thread quarter qq takes the 16-byte pieces qq, qq+4, ... of the row
// (conflict-free on the padded rows), loads each key piece once for all heads and
// reduces with two shuffles.  qv[h] is head h's query row (fp32, 16-byte aligned).
// Needs blockDim >= 4 * w.
template <typename Tin, int D, int NH>
__device__ __forceinline__ void window_scores(const float (*qv)[D], const float* ks, const Tin* rk_s,
                                              float (*sc)[64], int p, int w, int tid) {
  constexpr int EPP = 16 / (int)sizeof(Tin);      // elements per 16-byte piece
  constexpr int NP = D / EPP;                     // pieces per row
  constexpr int RS = ring_row_elems<Tin, D>();
  const int jj = tid >> 2, qq = tid & 3;
  if (jj < 64) {   // all four lanes of a slot take part in the shuffles
    const int j = p - (w - 1) + jj;
    const bool live = jj < w && j >= 0;
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
          ld16_vals<Tin>(rk_s + jj * RS + pc * EPP, x);
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

// Window softmax and value sums for NH heads.  sc[h][0..w) holds the scores (-inf
// for positions before the sequence start).  Every warp reduces the maxima and sums
// itself (no single-warp phase, no extra barrier).  Thread layout: 16-byte column
// piece cp = tid % NPC, slot group sg = tid / NPC, slots sg, sg + NSG, ...; each thread
// accumulates p_h(slot) v(slot) over its pieces, the slot groups of a warp are added
// with shuffles, and each warp writes wsum[warp][h][...]; the caller adds the NW
// partial sums.
template <typename Tin, int D, int NT, int NH>
struct WindowValues {
  static constexpr int EPP = 16 / (int)sizeof(Tin);   // elements per 16-byte piece
  static constexpr int NPC = D / EPP;                 // pieces per row
  static_assert(NPC <= 32 && 32 % NPC == 0, "a warp holds whole slot groups");
  static constexpr int NSG = NT / NPC;                // slot groups
  static constexpr int NW = NT / 32;                  // warps (partial sums)
  __device__ __forceinline__ static void run(const float (*sc)[64], const Tin* rv_s, const float* vs,
                                             float (*wsum)[NH][D], int p, int w, int tid, int lane) {
    float mh[NH], izh[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const float x0 = lane < w ? sc[h][lane] : -INFINITY;
      const float x1 = lane + 32 < w ? sc[h][lane + 32] : -INFINITY;
      const float m = warp_max(fmaxf(x0, x1));
      const float z = warp_sum((lane < w ? expf(x0 - m) : 0.f) + (lane + 32 < w ? expf(x1 - m) : 0.f));
      mh[h] = m;
      izh[h] = 1.0f / z;
    }
    constexpr int RS = ring_row_elems<Tin, D>();
    const int cp = tid % NPC, sg = tid / NPC;
    float2 acc[NH][EPP / 2];   // element pairs (packed multiply-adds)
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int e = 0; e < EPP / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
    for (int jj = sg; jj < w; jj += NSG) {
      const int j = p - (w - 1) + jj;
      if (j < 0) continue;
      float x[EPP];
      if (j == p) {
#pragma unroll
        for (int e = 0; e < EPP; ++e) x[e] = vs[cp * EPP + e];
      } else {
        ld16_vals<Tin>(rv_s + jj * RS + cp * EPP, x);
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float ph = expf(sc[h][jj] - mh[h]) * izh[h];
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
