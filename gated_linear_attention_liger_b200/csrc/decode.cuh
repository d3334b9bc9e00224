// decode.cuh -- one decode step: a pure HBM stream over the fp32 states.
//
// One CTA per (sequence, q head).  Per step the dominant traffic is reading
// and writing that head's d x d fp32 state; each thread owns a 4-column slab
// of RPT key rows, issues all of its 128-bit loads before any arithmetic (the
// loads are in flight while the feature maps, gate and window are computed),
// then applies S <- g S + phi(k)^T v, accumulates phi(q) S and streams the rows
// back.  The 64-slot key/value ring of the window branch is small and read
// through L2 (the q heads of a group share it); the new key/value is taken
// from the step's inputs, and the group's first q head writes it to slot
// pos mod w, which no other CTA of the step reads.  The position counter is
// advanced by a second one-thread-per-sequence kernel so that no CTA can see
// it half-updated.
//
// Recurrence and hybrid: "Liger: Linearizing Large Language Models to Gated
// Recurrent Structures" (Paper-Notes page), sections 统一的门控线性循环框架 and
// Liger Attention; constant-memory decoding: same page, section 亮点与洞察.
#pragma once

#include "common.cuh"

namespace liger {

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
};

constexpr int kDecodeThreads = 256;

__device__ __forceinline__ float4 ld_stream(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(float* p, float4 x) {
  __stcs(reinterpret_cast<float4*>(p), x);
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(DecodeArgs a) {
  constexpr int NT = kDecodeThreads;
  constexpr int CQ = D / 4;          // column quads
  constexpr int RGN = NT / CQ;       // row groups
  constexpr int RPT = D / RGN;       // rows per thread
  constexpr int EPL = D / 32;
  constexpr int VG = NT / D;         // window-sum key groups
  __shared__ __align__(16) float qs[D], ks[D], vs[D], fq[D], fk[D];
  __shared__ float sc[64];
  __shared__ __align__(16) float part[RGN][D];
  __shared__ float wpart[VG][D];
  __shared__ float gsh;

  const int Hq = a.Hq, Hkv = a.Hkv, w = a.w, G = Hq / Hkv;
  const int b = blockIdx.x / Hq, h = blockIdx.x % Hq, kv = h / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid % CQ, rg = tid / CQ;

  float* S = a.state + ((size_t)b * Hq + h) * D * D;
  float4 st[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) st[r] = ld_stream(S + (size_t)(rg * RPT + r) * D + 4 * cq);

  const Tin* qrow = static_cast<const Tin*>(a.q) + ((size_t)b * Hq + h) * D;
  const Tin* krow = static_cast<const Tin*>(a.k) + ((size_t)b * Hkv + kv) * D;
  const Tin* vrow = static_cast<const Tin*>(a.v) + ((size_t)b * Hkv + kv) * D;
  Tin* ring = static_cast<Tin*>(a.ring);
  const Tin* rk = ring + (((size_t)b * Hkv + kv) * 2 + 0) * w * D;
  const Tin* rv = ring + (((size_t)b * Hkv + kv) * 2 + 1) * w * D;
  const int p = max(a.pos[b], 0);   // a negative position is read as 0
  if (tid < D) {
    qs[tid] = io<Tin>::ld(qrow + tid);
    ks[tid] = io<Tin>::ld(krow + tid);
    vs[tid] = io<Tin>::ld(vrow + tid);
  }
  __syncthreads();

  if (warp == 0) {            // phi(k) and the gate
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
  } else if (warp == 1) {     // phi(q)
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
  // window scores: slot jj covers position p - (w-1) + jj
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  for (int jj = warp; jj < w; jj += NT / 32) {
    const long j = (long)p - (w - 1) + jj;
    float dot = -INFINITY;
    if (j >= 0) {
      float acc = 0.f;
      if (j == p) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc = fmaf(qs[lane + 32 * e], ks[lane + 32 * e], acc);
      } else {
        const Tin* kr = rk + (size_t)(j % w) * D;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc = fmaf(qs[lane + 32 * e], io<Tin>::ld(kr + lane + 32 * e), acc);
      }
      dot = warp_sum(acc) * inv_sqrt_d;
    }
    if (lane == 0) sc[jj] = dot;
  }
  __syncthreads();
  if (warp == 0) {
    const float x0 = lane < w ? sc[lane] : -INFINITY;
    const float x1 = lane + 32 < w ? sc[lane + 32] : -INFINITY;
    const float m = warp_max(fmaxf(x0, x1));
    const float e0 = lane < w ? expf(x0 - m) : 0.f;
    const float e1 = lane + 32 < w ? expf(x1 - m) : 0.f;
    const float z = warp_sum(e0 + e1);
    if (lane < w) sc[lane] = e0 / z;
    if (lane + 32 < w) sc[lane + 32] = e1 / z;
  }
  __syncthreads();
  {  // window value sum, split over VG key groups
    const int e = tid % D, grp = tid / D;
    float acc = 0.f;
    for (int jj = grp; jj < w; jj += VG) {
      const long j = (long)p - (w - 1) + jj;
      if (j < 0) continue;
      const float vx = (j == p) ? vs[e] : io<Tin>::ld(rv + (size_t)(j % w) * D + e);
      acc = fmaf(sc[jj], vx, acc);
    }
    wpart[grp][e] = acc;
  }
  // state update and readout on the streamed rows
  const float g = gsh;
  const float4 vv = *reinterpret_cast<const float4*>(vs + 4 * cq);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int row = rg * RPT + r;
    const float kr = fk[row], qr = fq[row];
    float4 x = st[r];
    x.x = fmaf(g, x.x, kr * vv.x);
    x.y = fmaf(g, x.y, kr * vv.y);
    x.z = fmaf(g, x.z, kr * vv.z);
    x.w = fmaf(g, x.w, kr * vv.w);
    acc.x = fmaf(qr, x.x, acc.x);
    acc.y = fmaf(qr, x.y, acc.y);
    acc.z = fmaf(qr, x.z, acc.z);
    acc.w = fmaf(qr, x.w, acc.w);
    st_stream(S + (size_t)row * D + 4 * cq, x);
  }
  *reinterpret_cast<float4*>(&part[rg][4 * cq]) = acc;
  __syncthreads();
  if (tid < D) {
    float grm = 0.f, swa = 0.f;
#pragma unroll
    for (int r = 0; r < RGN; ++r) grm += part[r][tid];
#pragma unroll
    for (int r = 0; r < VG; ++r) swa += wpart[r][tid];
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
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) pos[b] += 1;
}

}  // namespace liger
