// decode.cuh -- one decode step: a pure HBM stream over the fp32 states.
//
// One CTA per (sequence, q head).  Per step the dominant traffic is reading
// and writing that head's d x d fp32 state.  Each thread owns a 4-column slab
// of RPT key rows and issues all of its 128-bit streaming loads first; in the
// same breath the CTA copies the window ring's keys and values (the valid
// slots only) into shared memory with cp.async, so every later step of the
// window branch reads shared memory and no warp waits on a chain of dependent
// global loads.  Then S <- g S + phi(k)^T v is applied to the registers,
// phi(q) S is accumulated, and the rows stream back.  The new key/value is
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

template <typename Tin, int D>
constexpr size_t decode_smem_bytes() {
  return sizeof(Tin) * 2 * 64 * D;   // window ring keys and values
}

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
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_kernel(DecodeArgs a) {
  constexpr int NT = kDecodeThreads;
  constexpr int CQ = D / 4;          // column quads
  constexpr int RGN = NT / CQ;       // row groups
  constexpr int RPT = D / RGN;       // rows per thread
  constexpr int EPL = D / 32;
  constexpr int VG = NT / D;         // window-sum key groups
  constexpr int ROWB = D * (int)sizeof(Tin);   // bytes of one ring row
  extern __shared__ __align__(16) unsigned char dsm[];
  Tin* rk_s = reinterpret_cast<Tin*>(dsm);          // [64][D]
  Tin* rv_s = rk_s + 64 * D;                         // [64][D]
  __shared__ __align__(16) float qs[D], ks[D], vs[D], fq[D], fk[D];
  __shared__ float sc[64];
  __shared__ __align__(16) float part[RGN][D];
  __shared__ float wpart[VG][D];
  __shared__ float gsh;

  const int Hq = a.Hq, Hkv = a.Hkv, w = a.w, G = Hq / Hkv;
  const int b = blockIdx.x / Hq, h = blockIdx.x % Hq, kv = h / G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = tid % CQ, rg = tid / CQ;

  // 1. the state rows this thread updates: all loads in flight at once
  float* S = a.state + ((size_t)b * Hq + h) * D * D;
  float4 st[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) st[r] = ld_stream(S + (size_t)(rg * RPT + r) * D + 4 * cq);

  // 2. the window's ring slots (positions p-w+1 .. p-1) into shared memory
  const int p = max(a.pos[b], 0);   // a negative position is read as 0
  Tin* ring = static_cast<Tin*>(a.ring);
  const Tin* rk = ring + (((size_t)b * Hkv + kv) * 2 + 0) * w * D;
  const Tin* rv = ring + (((size_t)b * Hkv + kv) * 2 + 1) * w * D;
  {
    constexpr int CPR = ROWB / 16;   // 16-byte pieces per row
    for (int idx = tid; idx < w * CPR * 2; idx += NT) {
      const int which = idx / (w * CPR);           // 0 keys, 1 values
      const int rem = idx % (w * CPR);
      const int jj = rem / CPR, piece = rem % CPR;
      const long j = (long)p - (w - 1) + jj;
      if (j < 0 || j == p) continue;
      const Tin* src = (which ? rv : rk) + (size_t)(j % w) * D;
      Tin* dst = (which ? rv_s : rk_s) + jj * D;
      cp_async16(reinterpret_cast<char*>(dst) + piece * 16, reinterpret_cast<const char*>(src) + piece * 16);
    }
  }
  const Tin* qrow = static_cast<const Tin*>(a.q) + ((size_t)b * Hq + h) * D;
  const Tin* krow = static_cast<const Tin*>(a.k) + ((size_t)b * Hkv + kv) * D;
  const Tin* vrow = static_cast<const Tin*>(a.v) + ((size_t)b * Hkv + kv) * D;
  if (tid < D) {
    qs[tid] = io<Tin>::ld(qrow + tid);
    ks[tid] = io<Tin>::ld(krow + tid);
    vs[tid] = io<Tin>::ld(vrow + tid);
  }
  cp_async_wait_all();
  __syncthreads();

  // 3. window scores from shared memory (slot jj covers position p - (w-1) + jj)
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  {
    float qv[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[e] = qs[lane + 32 * e];
    for (int jj = warp; jj < w; jj += NT / 32) {
      const long j = (long)p - (w - 1) + jj;
      float dot = -INFINITY;
      if (j >= 0) {
        const Tin* kr = (j == p) ? nullptr : rk_s + jj * D;
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e)
          acc = fmaf(qv[e], kr ? io<Tin>::ld(kr + lane + 32 * e) : ks[lane + 32 * e], acc);
        dot = warp_sum(acc) * inv_sqrt_d;
      }
      if (lane == 0) sc[jj] = dot;
    }
  }
  // 4. phi(k) with the gate, and phi(q)
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
  // 5. window softmax
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
  // 6. window value sum, split over VG key groups
  {
    const int e = tid % D, grp = tid / D;
    float acc = 0.f;
    for (int jj = grp; jj < w; jj += VG) {
      const long j = (long)p - (w - 1) + jj;
      if (j < 0) continue;
      const float vx = (j == p) ? vs[e] : io<Tin>::ld(rv_s + jj * D + e);
      acc = fmaf(sc[jj], vx, acc);
    }
    wpart[grp][e] = acc;
  }
  // 7. state update and readout on the streamed rows
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
