// prefill_bwd.cuh -- gradient of the bf16 prefill on the sm_100a tensor cores.
//
// The pages give no backward pass; the linearisation fine-tune they describe
// (news article on Liger, section 軽量ファインチューニング: LoRA on the
// Q/K/V projections trained with next-token cross-entropy through this layer)
// needs one.  It is the derivative of the recurrence and hybrid of the
// Paper-Notes page (sections 统一的门控线性循环框架 and Liger Attention),
// evaluated chunk by chunk like the forward.  Within a chunk of n tokens with
// running log-gate sums b (b_C at its last token), entering state S and the
// gradient dS' of the state the chunk hands on:
//   A_ij  = e^{b_i - b_j} phi q_i . phi k_j  (j <= i),   G_ij = (alpha dO_i) . v_j  (j <= i)
//   d phi q_i = alpha e^{b_i} dO_i S^T + sum_j G_ij e^{b_i-b_j} phi k_j
//   d phi k_j = sum_i G_ij e^{b_i-b_j} phi q_i + e^{b_C-b_j} v_j dS'^T
//   dv_j      = sum_i A_ij alpha dO_i + e^{b_C-b_j} phi k_j dS'
//   dS        = e^{b_C} dS' + sum_i (e^{b_i} phi q_i)^T alpha dO_i
//   db_i      = alpha e^{b_i} phi q_i S . dO_i + sum_j A_ij G_ij - sum_i' A_i'i G_i'i
//               - e^{b_C-b_i} phi k_i dS' . v_i + [i last] <dS', S'>
// and d log g_t = sum_{i >= t in the chunk} db_i; the gate adds
// d log g_t sigmoid(-m_t) / d to every element of dk_t; the feature maps give
// dx = phi (d phi - <d phi, phi>).  The window branch's part is the backward
// of band-masked softmax attention.
//
// Launch sequence (one stream):
//   plan, seg_state        the forward's segment table, the per-chunk key images
//                          (e^{b_C-b_j} phi k_j, or phi k_j when the chunk's decay
//                          does not factor) and the running log-gate sums
//   chunk_incr             per (chunk, kv head): dS_c = Ktilde^T V and
//                          U_c = sum over the group's heads of (e^b phi Q)^T alpha dO
//   scan                   per (sequence, kv head): the state entering each chunk and
//                          the gradient of the state leaving it, as bf16 operand images
//   window                 per (chunk, q-head pair): the window branch's dq (kept in
//                          fp32), dk and dv (added into fp32 accumulators)
//   recurrent              per (chunk, q-head pair): the recurrent branch's dq (final,
//                          with the window part), d phi k, dv and the log-gate terms
//   finalize               per (token, kv head): dk and dv
// The initial state (when given) and its gradient are one per (sequence, kv head),
// the form in which the recurrence carries it.
#pragma once

#include "prefill_tc.cuh"

namespace liger {
namespace bwd {

using namespace liger::sm100;
using tc::C;
using tc::ROWS;
using tc::kmajor_off;
using tc::kFactorFloor;

struct BwdParams {
  tc::DevParams f;       // forward tables: segments, key images, gate sums, error word, sizes
  const void* k;         // [NT][Hkv][D] bf16 keys
  const void* dout;      // [NT][Hq][D] bf16
  const float* dfs;      // [n][Hq][D][D] gradient of the final state, or null
  const float* s0;       // [n][Hkv][D][D] initial state, or null
  float* ds0;            // [n][Hkv][D][D] its gradient (out), or null
  float* dS;             // [slots][Hkv][D][D] state increment of each chunk (from a zero start)
  float* U;              // [slots][Hkv][D][D] state-gradient increment of each chunk
  char* Himg;            // [slots][Hkv] bf16 D x D image: the state entering the chunk
  char* DHimg;           // [slots][Hkv] bf16 image: the gradient of the state leaving it
  float* dq_acc;         // [NT][Hq][D] the window branch's dq
  float* dphik;          // [NT][Hkv][D] gradient of phi(k), summed over the group's heads
  float* dkw;            // [NT][Hkv][D] the window branch's dk
  float* dv_acc;         // [NT][Hkv][D]
  float* dlg;            // [NT][Hkv] gradient of the log gate
  void* dq;              // [NT][Hq][D] bf16 (out)
  void* dk;              // [NT][Hkv][D] bf16 (out)
  void* dv;              // [NT][Hkv][D] bf16 (out)
};

// Byte offset of element (r, c) in a D x D bf16 image: rows r, 64-column blocks of
// D rows x 128 bytes, 128-byte swizzle (the layout of an MMA operand tile).
template <int D>
__device__ __forceinline__ uint32_t img_off(int r, int c) {
  return (uint32_t)(c >> 6) * (D * 128) + sw128(r, (c & 63) >> 3) + (uint32_t)((c & 7) << 1);
}

// The chunk a CTA of a (slot, kv head) grid works on; false when the slot is unused.
struct ChunkRef {
  int seg, c, t0, nv, kv;
  size_t ci;   // (slot, kv head) index
  bool first;  // the chunk starts its sequence
};
__device__ __forceinline__ bool chunk_ref(const tc::DevParams& p, int slot, int kv, ChunkRef& r) {
  const int seg = slot / p.L, c = slot % p.L;
  if (seg >= *p.n_segs) return false;
  const tc::SegInfo sg = p.segs[seg];
  const int nch = (sg.t_end - sg.t_begin + C - 1) / C;
  if (c >= nch) return false;
  r.seg = seg;
  r.c = c;
  r.t0 = sg.t_begin + c * C;
  r.nv = min(C, sg.t_end - r.t0);
  r.kv = kv;
  r.ci = (size_t)slot * p.Hkv + kv;
  r.first = r.t0 == sg.q0;
  return true;
}

// Bounded wait shorthand for the backward kernels (one role at a time, so a wait that
// gives up only has to leave the CTA consistently; every thread reaches the end).
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, const WaitCtx& w, uint32_t site) {
  return mbar_wait(bar, parity, w, site);
}

// ============================================================== per-chunk increments

template <int D>
struct IncrSmem {
  static constexpr uint32_t KV = C * D * 2, QB = ROWS * D * 2;
  static constexpr uint32_t IMG = 0, V0 = IMG + KV, Q0 = V0 + KV, DO0 = Q0 + QB, FQ = DO0 + QB;
  static constexpr uint32_t SMALL = FQ + QB;
  static constexpr uint32_t BYTES = SMALL + 1024 + 1024;
};

// Grid (slots * Hkv), 160 threads: warps 0-3 one row (2 * token + head) each, warp 4
// lane 0 issues the copies and the MMAs.
template <int D>
__global__ void __launch_bounds__(160, 1)
    chunk_incr_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
                      const __grid_constant__ CUtensorMap tmv, BwdParams bp) {
  griddep_wait_and_release();
  const tc::DevParams& p = bp.f;
  using L = IncrSmem<D>;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::SMALL);
  uint64_t* ld_img = bars;       // image, gate sums, values
  uint64_t* ld_q = bars + 1;     // a pair's q and dO
  uint64_t* mma_bar = bars + 2;
  uint64_t* drain = bars + 3;    // every MMA finished (before TMEM is freed)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never = tmem_slot + 2;
  float* bsh = reinterpret_cast<float*>(smem + L::SMALL + 64);   // [64]

  ChunkRef cr;
  if (!chunk_ref(p, blockIdx.x / p.Hkv, blockIdx.x % p.Hkv, cr)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv, npairs = G / 2;
  const bool issuer = warp == 4 && lane == 0;
  if (threadIdx.x == 0) {
    mbar_init(ld_img, 1); mbar_init(ld_q, 1); mbar_init(mma_bar, 1); mbar_init(drain, 1);
    *abort_flag = 0u;
    *never = 0u;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err, p.wait_ns};
  auto load_pair = [&](int pr) {
    mbar_arrive_expect_tx(ld_q, 2 * L::QB);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) {
      tma_load_3d(smem + L::Q0 + kb * ROWS * 128, &tmq, ld_q, kb * 64, cr.kv * G + 2 * pr, cr.t0);
      tma_load_3d(smem + L::DO0 + kb * ROWS * 128, &tmdo, ld_q, kb * 64, cr.kv * G + 2 * pr, cr.t0);
    }
  };
  if (issuer) {
    mbar_arrive_expect_tx(ld_img, L::KV + L::KV + C * 4);
    bulk_load(smem + L::IMG, p.kimg + cr.ci * L::KV, L::KV, ld_img);
    bulk_load(bsh, p.bimg + cr.ci * C, C * 4, ld_img);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) tma_load_3d(smem + L::V0 + kb * C * 128, &tmv, ld_img, kb * 64, cr.kv, cr.t0);
    load_pair(0);
  }
  bool ok = bwait(ld_img, 0, wc, wsite(3, 1, 0));
  const float bC = bsh[C - 1];
  const bool fast = bC >= kFactorFloor;
  if (!fast && threadIdx.x < 128) {   // exact mode: the image holds phi(k); scale it to Ktilde
    const int j = threadIdx.x >> 1, h = threadIdx.x & 1;
    const float sc = __expf(bC - bsh[j]);
#pragma unroll
    for (int c8 = 0; c8 < D / 16; ++c8) {
      const uint32_t off = kmajor_off(j, h * (D / 2) + c8 * 8, C * 128);
      float x[8];
      tc::ld_chunk8(smem + L::IMG, off, x);
#pragma unroll
      for (int q = 0; q < 8; ++q) x[q] *= sc;
      tc::st_chunk8(smem + L::IMG, off, x);
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (issuer && ok) {   // dS_c = Ktilde^T V  (M = D rows of the key dim; D = 64 duplicates rows)
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(128, D, 1, 1);
    const uint32_t lbo_a = D == 128 ? C * 128 : 0;
#pragma unroll
    for (int kk = 0; kk < C / 16; ++kk)
      mma_bf16_ss(tmem, sdesc_sw128(smem_u32(smem + L::IMG) + kk * 2048, lbo_a, 1024),
                  sdesc_sw128(smem_u32(smem + L::V0) + kk * 2048, C * 128, 1024), idesc, kk > 0);
  }
  const float alpha = p.alpha;
  int pairs_issued = 1;
  for (int pr = 0; pr < npairs; ++pr) {
    ok = bwait(ld_q, pr & 1, wc, wsite(3, 2, pr)) && ok;
    if (threadIdx.x < 128) {
      // row = 2 * token + head: alpha e^{b_i} phi(q) (bf16), zero past the valid tokens
      const int row = threadIdx.x, i = row >> 1;
      const char* qb = smem + L::Q0;
      float m = -INFINITY;
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) m = fmaxf(m, bf16x8_max(*reinterpret_cast<const uint4*>(qb + kmajor_off(row, c8 * 8, ROWS * 128))));
      float z = 0.f;
      constexpr float kL2e = 1.4426950408889634f;
      const float ml = m * kL2e;
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) {
        float x[8];
        tc::ld_chunk8(qb, kmajor_off(row, c8 * 8, ROWS * 128), x);
#pragma unroll
        for (int q = 0; q < 8; ++q) z += ex2(fmaf(x[q], kL2e, -ml));
      }
      const float sc = i < cr.nv ? alpha * __expf(bsh[i]) / z : 0.f;
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint32_t off = kmajor_off(row, c8 * 8, ROWS * 128);
        float x[8];
        tc::ld_chunk8(qb, off, x);
#pragma unroll
        for (int q = 0; q < 8; ++q) x[q] = sc * ex2(fmaf(x[q], kL2e, -ml));
        tc::st_chunk8(smem + L::FQ, off, x);
      }
      fence_proxy_async_smem();
    }
    __syncthreads();
    if (issuer && ok) {   // U_c += (alpha e^b phi Q)^T dO: M = D (key dim), N = D, K = 128 rows
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, D, 1, 1);
      const uint32_t lbo_a = D == 128 ? ROWS * 128 : 0;
#pragma unroll
      for (int kk = 0; kk < ROWS / 16; ++kk)
        mma_bf16_ss(tmem + 128, sdesc_sw128(smem_u32(smem + L::FQ) + kk * 2048, lbo_a, 1024),
                    sdesc_sw128(smem_u32(smem + L::DO0) + kk * 2048, ROWS * 128, 1024), idesc,
                    (pr > 0 || kk > 0) ? 1u : 0u);
      mma_commit(mma_bar);
    }
    ok = bwait(mma_bar, pr & 1, wc, wsite(2, 1, pr)) && ok;   // the tiles may be overwritten
    tc_fence_after();
    if (issuer && ok && pr + 1 < npairs) {
      load_pair(pr + 1);
      pairs_issued = pr + 2;
    }
  }
  if (issuer) {   // never leave with copies in flight
    const WaitCtx dw{never, nullptr, p.wait_ns};
    mbar_wait(ld_img, 0, dw);
    mbar_wait(ld_q, (pairs_issued - 1) & 1, dw);
  }
  // both accumulators to global, one key-dim row per thread
  if (threadIdx.x < 128 && warp_all(ok && !*abort_flag)) {
    const int r = threadIdx.x;
    const uint32_t lb = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      float* dst = (which == 0 ? bp.dS : bp.U) + (cr.ci * D + (r < D ? r : 0)) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float v[32];
        tmem_ld32(lb + which * 128 + c0, v);
        tmem_wait_ld();
        if (r < D) {
#pragma unroll
          for (int u = 0; u < 32; u += 4) *reinterpret_cast<float4*>(dst + c0 + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
        }
      }
    }
  }
  if (issuer) mma_commit(drain);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    mbar_wait(drain, 0, WaitCtx{never, nullptr, p.wait_ns});
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ============================================================== window branch

template <int D>
struct WinSmem {
  static constexpr uint32_t QB = ROWS * D * 2;          // 128 rows x D
  static constexpr uint32_t KB = 2 * C * D * 2;         // 128 keys x D: [previous | current]
  static constexpr uint32_t TB = ROWS * 2 * C * 2;      // 128 rows x 128 keys
  static constexpr uint32_t Q0 = 0, DO0 = Q0 + QB, K0 = DO0 + QB, V0 = K0 + KB, DSW = V0 + KB, PW = DSW + TB;
  static constexpr uint32_t SMALL = PW + TB;
  static constexpr uint32_t BYTES = SMALL + 1024 + 1024;
};

// Adds `v` into global fp32 memory without returning the old value.
__device__ __forceinline__ void red_add(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
// Adds four consecutive fp32 (16-byte aligned) in one instruction.
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// Per (chunk, q-head pair): rows 2 * token + head against keys [previous chunk | current
// chunk].  Grid (slots * Hq / 2), 160 threads: warps 0-3 one row each, warp 4 lane 0
// issues copies and MMAs.
template <int D>
__global__ void __launch_bounds__(160, 1)
    bwd_window_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
                      const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv, BwdParams bp) {
  griddep_wait_and_release();
  const tc::DevParams& p = bp.f;
  using L = WinSmem<D>;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::SMALL);
  uint64_t* ld = bars;
  uint64_t* mma1 = bars + 1;
  uint64_t* mma2 = bars + 2;
  uint64_t* drain = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never = tmem_slot + 2;

  const int npairs = p.Hq / 2;
  ChunkRef cr;
  const int G = p.Hq / p.Hkv;
  const int pair = blockIdx.x % npairs, h0 = 2 * pair;
  if (!chunk_ref(p, blockIdx.x / npairs, h0 / G, cr)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool issuer = warp == 4 && lane == 0;
  if (threadIdx.x == 0) {
    mbar_init(ld, 1); mbar_init(mma1, 1); mbar_init(mma2, 1); mbar_init(drain, 1);
    *abort_flag = 0u;
    *never = 0u;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err, p.wait_ns};
  if (issuer) {
    mbar_arrive_expect_tx(ld, 2 * L::QB + 2 * L::KB);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) {
      tma_load_3d(smem + L::Q0 + kb * ROWS * 128, &tmq, ld, kb * 64, h0, cr.t0);
      tma_load_3d(smem + L::DO0 + kb * ROWS * 128, &tmdo, ld, kb * 64, h0, cr.t0);
      // previous chunk's keys and values in rows 0-63 (coordinates before the sequence
      // start or the tensor read as zeros and are masked), the chunk's own in rows 64-127
      for (int half = 0; half < 2; ++half) {
        const int tok = cr.t0 + (half - 1) * C;
        tma_load_3d(smem + L::K0 + kb * (2 * C * 128) + half * C * 128, &tmk, ld, kb * 64, cr.kv, tok);
        tma_load_3d(smem + L::V0 + kb * (2 * C * 128) + half * C * 128, &tmv, ld, kb * 64, cr.kv, tok);
      }
    }
  }
  bool ok = bwait(ld, 0, wc, wsite(3, 1, 0));
  if (issuer && ok) {   // Ss = Q [Kp|Kc]^T, dOV = dO [Vp|Vc]^T (N = 128 keys)
    tc_fence_after();
    const uint32_t id = idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t ao = (kk >> 2) * (ROWS * 128) + (kk & 3) * 32, bo = (kk >> 2) * (2 * C * 128) + (kk & 3) * 32;
      mma_bf16_ss(tmem, sdesc_sw128(smem_u32(smem + L::Q0) + ao, 16, 1024),
                  sdesc_sw128(smem_u32(smem + L::K0) + bo, 16, 1024), id, kk > 0);
      mma_bf16_ss(tmem + 128, sdesc_sw128(smem_u32(smem + L::DO0) + ao, 16, 1024),
                  sdesc_sw128(smem_u32(smem + L::V0) + bo, 16, 1024), id, kk > 0);
    }
    mma_commit(mma1);
  }
  ok = bwait(mma1, 0, wc, wsite(2, 1, 0)) && ok;
  tc_fence_after();
  if (threadIdx.x < 128) {
    const int row = threadIdx.x, i = row >> 1;
    const uint32_t lb = tmem + ((uint32_t)(warp * 32) << 16);
    const bool live = i < cr.nv && ok;
    // band: keys x in [i+1, i+64] of [previous | current]; no previous keys in a
    // sequence's first chunk
    const int xlo = max(i + 1, cr.first ? C : 0), xhi = i + C;
    const float sl2 = 1.4426950408889634f / sqrtf((float)D);
    const float beta = 1.f - p.alpha;
    float P[2 * C];
#pragma unroll
    for (int x = 0; x < 2 * C; x += 32) tmem_ld32(lb + x, P + x);
    tmem_wait_ld();
    float m = -INFINITY;
#pragma unroll
    for (int x = 0; x < 2 * C; ++x) {
      P[x] = (x >= xlo && x <= xhi) ? P[x] * sl2 : -INFINITY;
      m = fmaxf(m, P[x]);
    }
    float l = 0.f;
#pragma unroll
    for (int x = 0; x < 2 * C; ++x) { P[x] = ex2(P[x] - m); l += P[x]; }
    const float il = live ? 1.f / l : 0.f;   // rows past the chunk's tokens add nothing
#pragma unroll
    for (int x = 0; x < 2 * C; ++x) P[x] *= il;
    // D_i = sum_x P dP with dP = beta dO . v_x
    float Dsum = 0.f;
#pragma unroll
    for (int x0 = 0; x0 < 2 * C; x0 += 32) {
      float g[32];
      tmem_ld32(lb + 128 + x0, g);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u) Dsum += P[x0 + u] * g[u];
    }
    Dsum *= beta;
    // dS = P (dP - D) / sqrt(d) and beta P, bf16 rows of the two key tiles
    const float isd = 1.f / sqrtf((float)D);
#pragma unroll
    for (int x0 = 0; x0 < 2 * C; x0 += 32) {
      float g[32];
      tmem_ld32(lb + 128 + x0, g);
      tmem_wait_ld();
#pragma unroll
      for (int u8 = 0; u8 < 32; u8 += 8) {
        float ds[8], pw[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float pv = P[x0 + u8 + q];
          ds[q] = pv * (beta * g[u8 + q] - Dsum) * isd;
          pw[q] = beta * pv;
        }
        const uint32_t off = kmajor_off(row, x0 + u8, ROWS * 128);
        tc::st_chunk8(smem + L::DSW, off, ds);
        tc::st_chunk8(smem + L::PW, off, pw);
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (issuer && ok) {
    tc_fence_after();
    // dq_win = dS [Kp|Kc] (M = 128 rows, N = D, K = 128 keys; keys tile MN-major)
    const uint32_t id_q = idesc_bf16(128, D, 0, 1);
#pragma unroll
    for (int kk = 0; kk < 2 * C / 16; ++kk)
      mma_bf16_ss(tmem + 256, sdesc_sw128(smem_u32(smem + L::DSW) + (kk >> 2) * (ROWS * 128) + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(smem_u32(smem + L::K0) + kk * 2048, 2 * C * 128, 1024), id_q, kk > 0);
    // dk_win = dS^T Q and dv_win = (beta P)^T dO with the keys on the lanes: M = 128 keys
    // (A = the key tiles, MN-major), N = D, K = 128 rows
    const uint32_t id_t = idesc_bf16(128, D, 1, 1);
#pragma unroll
    for (int kk = 0; kk < ROWS / 16; ++kk) {
      mma_bf16_ss(tmem, sdesc_sw128(smem_u32(smem + L::DSW) + kk * 2048, ROWS * 128, 1024),
                  sdesc_sw128(smem_u32(smem + L::Q0) + kk * 2048, ROWS * 128, 1024), id_t, kk > 0);
      mma_bf16_ss(tmem + 128, sdesc_sw128(smem_u32(smem + L::PW) + kk * 2048, ROWS * 128, 1024),
                  sdesc_sw128(smem_u32(smem + L::DO0) + kk * 2048, ROWS * 128, 1024), id_t, kk > 0);
    }
    mma_commit(mma2);
  }
  ok = bwait(mma2, 0, wc, wsite(2, 2, 0)) && ok;
  tc_fence_after();
  if (threadIdx.x < 128 && warp_all(ok && !*abort_flag)) {
    const int row = threadIdx.x, i = row >> 1, hh = row & 1;
    const uint32_t lb = tmem + ((uint32_t)(warp * 32) << 16);
    // the window part of dq, kept in fp32 for the recurrent kernel
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float v[32];
      tmem_ld32(lb + 256 + c0, v);
      tmem_wait_ld();
      if (i < cr.nv) {
        float* dst = bp.dq_acc + ((size_t)(cr.t0 + i) * p.Hq + h0 + hh) * D + c0;
#pragma unroll
        for (int u = 0; u < 32; u += 4) *reinterpret_cast<float4*>(dst + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
      }
    }
    // key side: lane = key x of [previous | current], columns = its d-vector.  The TMEM
    // loads are warp-collective: every lane takes them, only live keys add.
    const int x = row;
    const bool key_ok = x < C ? !cr.first : (x - C) < cr.nv;
    const size_t base = key_ok ? ((size_t)(cr.t0 + x - C) * p.Hkv + cr.kv) * D : 0;
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
      float* dst = (which == 0 ? bp.dkw : bp.dv_acc) + base;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float v[32];
        tmem_ld32(lb + which * 128 + c0, v);
        tmem_wait_ld();
        if (key_ok) {
#pragma unroll
          for (int u = 0; u < 32; u += 4) red_add4(dst + c0 + u, v[u], v[u + 1], v[u + 2], v[u + 3]);
        }
      }
    }
  }
  if (issuer) {
    mma_commit(drain);
    mbar_wait(ld, 0, WaitCtx{never, nullptr, p.wait_ns});   // never leave with copies in flight
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    mbar_wait(drain, 0, WaitCtx{never, nullptr, p.wait_ns});
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== recurrent branch

template <int D>
struct RecSmem {
  static constexpr uint32_t QB = ROWS * D * 2, KVB = C * D * 2, SB = D * D * 2, TB = ROWS * C * 2;
  static constexpr uint32_t Q0 = 0, DO0 = Q0 + QB, IMG = DO0 + QB, V0 = IMG + KVB, H0 = V0 + KVB;  // H0: then Qr
  static constexpr uint32_t DH0 = H0 + (SB > QB ? SB : QB), GM = DH0 + SB, AT = GM + TB;
  static constexpr uint32_t SMALL = AT + TB;
  static constexpr uint32_t BYTES = SMALL + 2048 + 1024;
};

template <int D>
__global__ void __launch_bounds__(160, 1)
    bwd_recurrent_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
                         const __grid_constant__ CUtensorMap tmv, BwdParams bp) {
  griddep_wait_and_release();
  const tc::DevParams& p = bp.f;
  using L = RecSmem<D>;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::SMALL);
  uint64_t* ld = bars;
  uint64_t* mma1 = bars + 1;
  uint64_t* mma2 = bars + 2;
  uint64_t* mma3 = bars + 3;
  uint64_t* drain = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never = tmem_slot + 2;
  float* bsh = reinterpret_cast<float*>(smem + L::SMALL + 64);    // [64] running log-gate sums
  float* colsum = bsh + 64;                                        // [64] sum_i A_ij G_ij (this pair)
  float* dbt = colsum + 64;                                        // [64] db per token (this pair)
  float* red = dbt + 64;                                           // [4] <dS', S> partials, [4] sum_j E_j

  const int npairs = p.Hq / 2;
  const int G = p.Hq / p.Hkv;
  const int pair = blockIdx.x % npairs, h0 = 2 * pair;
  ChunkRef cr;
  if (!chunk_ref(p, blockIdx.x / npairs, h0 / G, cr)) return;
  const bool pair_first = h0 % G == 0;   // adds the terms of the group-summed state gradient
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool issuer = warp == 4 && lane == 0;
  if (threadIdx.x == 0) {
    mbar_init(ld, 1); mbar_init(mma1, 1); mbar_init(mma2, 1); mbar_init(mma3, 1); mbar_init(drain, 1);
    *abort_flag = 0u;
    *never = 0u;
    fence_mbar_init();
  }
  if (threadIdx.x < 64) { colsum[threadIdx.x] = 0.f; dbt[threadIdx.x] = 0.f; }
  if (threadIdx.x < 8) red[threadIdx.x] = 0.f;
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err, p.wait_ns};
  if (issuer) {
    mbar_arrive_expect_tx(ld, 2 * L::QB + 2 * L::KVB + C * 4 + (pair_first ? 2 : 1) * L::SB);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) {
      tma_load_3d(smem + L::Q0 + kb * ROWS * 128, &tmq, ld, kb * 64, h0, cr.t0);
      tma_load_3d(smem + L::DO0 + kb * ROWS * 128, &tmdo, ld, kb * 64, h0, cr.t0);
      tma_load_3d(smem + L::V0 + kb * C * 128, &tmv, ld, kb * 64, cr.kv, cr.t0);
    }
    bulk_load(smem + L::IMG, p.kimg + cr.ci * L::KVB, L::KVB, ld);
    bulk_load(bsh, p.bimg + cr.ci * C, C * 4, ld);
    bulk_load(smem + L::H0, bp.Himg + cr.ci * L::SB, L::SB, ld);
    if (pair_first) bulk_load(smem + L::DH0, bp.DHimg + cr.ci * L::SB, L::SB, ld);
  }
  bool ok = bwait(ld, 0, wc, wsite(3, 1, 0));
  if (issuer && ok) {
    tc_fence_after();
    // X = dO S^T (N = D; S as the K-major image) and G' = dO Vc^T (N = 64)
    const uint32_t id_x = idesc_bf16(128, D, 0, 0), id_g = idesc_bf16(128, C, 0, 0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t ao = (kk >> 2) * (ROWS * 128) + (kk & 3) * 32;
      const uint64_t a = sdesc_sw128(smem_u32(smem + L::DO0) + ao, 16, 1024);
      mma_bf16_ss(tmem, a, sdesc_sw128(smem_u32(smem + L::H0) + (kk >> 2) * (D * 128) + (kk & 3) * 32, 16, 1024),
                  id_x, kk > 0);
      mma_bf16_ss(tmem + 128, a, sdesc_sw128(smem_u32(smem + L::V0) + (kk >> 2) * (C * 128) + (kk & 3) * 32, 16, 1024),
                  id_g, kk > 0);
    }
    mma_commit(mma1);
  }
  const float bC = bsh[C - 1];
  const bool fast = bC >= kFactorFloor;
  const float alpha = p.alpha;
  constexpr float kL2e = 1.4426950408889634f;
  // <dS', S> over the whole image (both bf16, same layout), before S's buffer is reused
  if (pair_first && threadIdx.x < 128) {
    float acc = 0.f;
    for (int c16 = threadIdx.x; c16 < D * D / 8; c16 += 128) {
      float a[8], b[8];
      tc::ld_chunk8(smem + L::H0, c16 * 16, a);
      tc::ld_chunk8(smem + L::DH0, c16 * 16, b);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc = fmaf(a[q], b[q], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) red[warp] = acc;
  }
  __syncthreads();   // every thread is done reading S's buffer before Qr overwrites it
  ok = bwait(mma1, 0, wc, wsite(2, 1, 0)) && ok;
  tc_fence_after();
  const int row = threadIdx.x, i = row >> 1, hh = row & 1;
  const uint32_t lb = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const bool live = threadIdx.x < 128 && i < cr.nv && ok;
  float g[C];        // G_ij = alpha dO_i . v_j, causal, zero for rows past the tokens
  float term1 = 0.f; // alpha e^{b_i} phi q_i . X_i
  float zq = 1.f, mq = 0.f;
  if (threadIdx.x < 128) {
    const char* qb = smem + L::Q0;
    mq = -INFINITY;
#pragma unroll
    for (int c8 = 0; c8 < D / 8; ++c8) mq = fmaxf(mq, bf16x8_max(*reinterpret_cast<const uint4*>(qb + kmajor_off(row, c8 * 8, ROWS * 128))));
    mq *= kL2e;
    zq = 0.f;
#pragma unroll
    for (int c8 = 0; c8 < D / 8; ++c8) {
      float x[8];
      tc::ld_chunk8(qb, kmajor_off(row, c8 * 8, ROWS * 128), x);
#pragma unroll
      for (int q = 0; q < 8; ++q) zq += ex2(fmaf(x[q], kL2e, -mq));
    }
    const float izq = 1.f / zq;
    const float bi = bsh[i];
    const float rq = fast ? __expf(bi - bC) : 1.f;   // row factor folded into Qr in factored mode
    // Qr = phi(q) (times e^{b_i - b_C} in factored mode) over S's buffer; phi(q) . X on the way
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float xv[32];
      tmem_ld32(lb + c0, xv);
      tmem_wait_ld();
#pragma unroll
      for (int u8 = 0; u8 < 32; u8 += 8) {
        const uint32_t off = kmajor_off(row, c0 + u8, ROWS * 128);
        float x[8];
        tc::ld_chunk8(qb, off, x);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          x[q] = ex2(fmaf(x[q], kL2e, -mq)) * izq;
          term1 = fmaf(x[q], xv[u8 + q], term1);
          x[q] *= rq;
        }
        tc::st_chunk8(smem + L::H0, off, x);
      }
    }
    term1 = live ? alpha * __expf(bi) * term1 : 0.f;
    float gv[C];
    tmem_ld32(lb + 128, gv);
    tmem_ld32(lb + 128 + 32, gv + 32);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < C; ++j) g[j] = (live && j <= i) ? alpha * gv[j] : 0.f;
    // GM = G (times e^{b_i - b_j} when the decay does not factor), bf16 [row][j]
#pragma unroll
    for (int j8 = 0; j8 < C; j8 += 8) {
      float x[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) x[q] = fast ? g[j8 + q] : g[j8 + q] * __expf(bi - bsh[j8 + q]);
      tc::st_chunk8(smem + L::GM, kmajor_off(row, j8, ROWS * 128), x);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (issuer && ok) {   // A' = Qr Ktilde^T (factored: A itself; exact: phi q . phi k)
    tc_fence_after();
    const uint32_t id_a = idesc_bf16(128, C, 0, 0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      mma_bf16_ss(tmem + 192, sdesc_sw128(smem_u32(smem + L::H0) + (kk >> 2) * (ROWS * 128) + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(smem_u32(smem + L::IMG) + (kk >> 2) * (C * 128) + (kk & 3) * 32, 16, 1024), id_a, kk > 0);
    mma_commit(mma2);
  }
  ok = bwait(mma2, 0, wc, wsite(2, 2, 0)) && ok;
  tc_fence_after();
  float rowsum = 0.f;
  if (threadIdx.x < 128) {
    float av[C];
    tmem_ld32(lb + 192, av);
    tmem_ld32(lb + 192 + 32, av + 32);
    tmem_wait_ld();
    const float bi = bsh[i];
#pragma unroll
    for (int j = 0; j < C; ++j) {
      float a = (live && j <= i) ? av[j] : 0.f;
      if (!fast) a *= __expf(bi - bsh[j]);
      av[j] = a;
      rowsum = fmaf(a, g[j], rowsum);
    }
#pragma unroll
    for (int j8 = 0; j8 < C; j8 += 8) {
      float x[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) x[q] = alpha * av[j8 + q];
      tc::st_chunk8(smem + L::AT, kmajor_off(row, j8, ROWS * 128), x);
    }
    fence_proxy_async_smem();
    // column sums over the pair's rows: a reduce-scatter across the warp (each exchange
    // halves the columns a lane holds; lane l ends with columns 2 l and 2 l + 1), then
    // shared atomics across the warps
#pragma unroll
    for (int j = 0; j < C; ++j) av[j] *= g[j];
    static_assert(C == 64, "two columns per lane at the end");
#pragma unroll
    for (int half = C / 2, mask = 16; half >= 2; half >>= 1, mask >>= 1) {
      const bool up = (lane & mask) != 0;   // this lane keeps the upper half of its columns
#pragma unroll
      for (int k = 0; k < half; ++k) {
        const float keep = up ? av[k + half] : av[k];
        const float send = up ? av[k] : av[k + half];
        av[k] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
      }
    }
    atomicAdd(&colsum[2 * lane], av[0]);
    atomicAdd(&colsum[2 * lane + 1], av[1]);
  }
  tc_fence_before();
  __syncthreads();
  if (issuer && ok) {
    tc_fence_after();
    // d phi q (recurrent part) = GM Img (N = D, K = 64 keys; the image MN-major)
    const uint32_t id_q = idesc_bf16(128, D, 0, 1);
#pragma unroll
    for (int kk = 0; kk < C / 16; ++kk)
      mma_bf16_ss(tmem + 128, sdesc_sw128(smem_u32(smem + L::GM) + kk * 32, 16, 1024),
                  sdesc_sw128(smem_u32(smem + L::IMG) + kk * 2048, C * 128, 1024), id_q, kk > 0);
    // key side with the keys on the lanes: M = 128 over the 64 keys (LBO 0 repeats them;
    // lanes 64-127 are not read), N = D, K = 128 rows
    const uint32_t id_t = idesc_bf16(128, D, 1, 1);
#pragma unroll
    for (int kk = 0; kk < ROWS / 16; ++kk) {
      // d phi k (the group's rows) = GM^T Qr
      mma_bf16_ss(tmem + 256, sdesc_sw128(smem_u32(smem + L::GM) + kk * 2048, 0, 1024),
                  sdesc_sw128(smem_u32(smem + L::H0) + kk * 2048, ROWS * 128, 1024), id_t, kk > 0);
      // dv (the group's rows) = (alpha A)^T dO
      mma_bf16_ss(tmem + 384, sdesc_sw128(smem_u32(smem + L::AT) + kk * 2048, 0, 1024),
                  sdesc_sw128(smem_u32(smem + L::DO0) + kk * 2048, ROWS * 128, 1024), id_t, kk > 0);
    }
    mma_commit(mma3);
  }
  ok = bwait(mma3, 0, wc, wsite(2, 3, 0)) && ok;
  tc_fence_after();
  if (threadIdx.x < 128 && warp_all(ok && !*abort_flag)) {
    const float bi = bsh[i];
    // dq = phi q (d phi q - <d phi q, phi q>) + the window part
    const float rq = fast ? __expf(bi - bC) : 1.f;
    const float eb = alpha * __expf(bi);
    const char* qb = smem + L::Q0;
    const float izq = 1.f / zq;
    float dot = 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float xv[32], mv[32];
      tmem_ld32(lb + c0, xv);
      tmem_ld32(lb + 128 + c0, mv);
      tmem_wait_ld();
#pragma unroll
      for (int u8 = 0; u8 < 32; u8 += 8) {
        float x[8];
        tc::ld_chunk8(qb, kmajor_off(row, c0 + u8, ROWS * 128), x);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float ph = ex2(fmaf(x[q], kL2e, -mq)) * izq;
          dot = fmaf(ph, fmaf(eb, xv[u8 + q], rq * mv[u8 + q]), dot);
        }
      }
    }
    const size_t o = ((size_t)(cr.t0 + i) * p.Hq + h0 + hh) * D;
    __nv_bfloat16* dq = static_cast<__nv_bfloat16*>(bp.dq);
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float xv[32], mv[32];
      tmem_ld32(lb + c0, xv);
      tmem_ld32(lb + 128 + c0, mv);
      tmem_wait_ld();
      if (live) {
#pragma unroll
        for (int u8 = 0; u8 < 32; u8 += 8) {
          float x[8];
          tc::ld_chunk8(qb, kmajor_off(row, c0 + u8, ROWS * 128), x);
          // the window part of dq: eight consecutive fp32 in two 16-byte loads
          const float4 wa = *reinterpret_cast<const float4*>(bp.dq_acc + o + c0 + u8);
          const float4 wb = *reinterpret_cast<const float4*>(bp.dq_acc + o + c0 + u8 + 4);
          const float wq[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 8; q += 2) {
            float y[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float ph = ex2(fmaf(x[q + e], kL2e, -mq)) * izq;
              const float dphi = fmaf(eb, xv[u8 + q + e], rq * mv[u8 + q + e]);
              y[e] = fmaf(ph, dphi - dot, wq[q + e]);
            }
            w[q / 2] = pack_bf16(y[0], y[1]);
          }
          *reinterpret_cast<uint4*>(dq + o + c0 + u8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();   // X and d phi q are read: their columns take the state-gradient terms
  if (pair_first && issuer && ok) {
    tc_fence_after();
    // v_j dS'^T (A = Vc K-major, B = dS' K-major) and Img_j dS' (A = Img K-major, B = dS'
    // MN-major); keys on the lanes, K = D
    const uint32_t id_kk = idesc_bf16(128, D, 0, 0), id_km = idesc_bf16(128, D, 0, 1);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      mma_bf16_ss(tmem, sdesc_sw128(smem_u32(smem + L::V0) + (kk >> 2) * (C * 128) + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(smem_u32(smem + L::DH0) + (kk >> 2) * (D * 128) + (kk & 3) * 32, 16, 1024), id_kk,
                  kk > 0);
      mma_bf16_ss(tmem + 128, sdesc_sw128(smem_u32(smem + L::IMG) + (kk >> 2) * (C * 128) + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(smem_u32(smem + L::DH0) + kk * 2048, D * 128, 1024), id_km, kk > 0);
    }
    mma_commit(mma1);   // (second phase of this barrier)
  }
  if (pair_first) {
    ok = bwait(mma1, 1, wc, wsite(2, 4, 0)) && ok;
    tc_fence_after();
  }
  if (threadIdx.x < 128 && warp_all(ok && !*abort_flag)) {
    // key j = this lane: d phi k and dv rows, and (once per kv head) the state terms.  The
    // TMEM loads are warp-collective: every lane takes them, only keys j < nv add.
    const int j = threadIdx.x;
    const bool jl = j < cr.nv;
    const float cj = __expf(bC - bsh[j & (C - 1)]);
    const size_t base = jl ? ((size_t)(cr.t0 + j) * p.Hkv + cr.kv) * D : 0;
    float es = 0.f;   // e^{b_C - b_j} phi k_j dS' . v_j
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float t1[32], t2[32], d2[32], d4[32];
      tmem_ld32(lb + 256 + c0, t1);
      tmem_ld32(lb + 384 + c0, t2);
      if (pair_first) {
        tmem_ld32(lb + c0, d2);
        tmem_ld32(lb + 128 + c0, d4);
      }
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        float dk = t1[u], dvv = t2[u];
        if (pair_first) {
          dk = fast ? cj * (dk + d2[u]) : dk + cj * d2[u];
          const float e4 = fast ? d4[u] : cj * d4[u];
          dvv += e4;
          // v_j[c] for c = c0 + u: element (j, c) of the values tile
          es = fmaf(e4, bf16_lo(*reinterpret_cast<const uint16_t*>(smem + L::V0 + kmajor_off(j & (C - 1), c0 + u, C * 128))), es);
        } else if (fast) {
          dk *= cj;
        }
        t1[u] = dk;
        t2[u] = dvv;
      }
      if (jl) {
#pragma unroll
        for (int u = 0; u < 32; u += 4) {
          red_add4(bp.dphik + base + c0 + u, t1[u], t1[u + 1], t1[u + 2], t1[u + 3]);
          red_add4(bp.dv_acc + base + c0 + u, t2[u], t2[u + 1], t2[u + 2], t2[u + 3]);
        }
      }
    }
    if (pair_first && jl) {
      atomicAdd(&dbt[j], -es);
      atomicAdd(&red[4], es);
    }
  }
  tc_fence_before();
  __syncthreads();
  // the log-gate gradient of the chunk's tokens: row terms of both heads, minus the column
  // sums, plus (once per kv head) the state terms; then suffix sums over the chunk
  if (threadIdx.x < 128 && ok) {
    const float both = term1 + rowsum + __shfl_xor_sync(0xffffffffu, term1 + rowsum, 1);
    if (hh == 0 && i < cr.nv) atomicAdd(&dbt[i], both - colsum[i]);
  }
  __syncthreads();
  if (threadIdx.x == 0 && ok && pair_first && cr.nv > 0) {
    // the last token's gate also scales the state it hands on:
    // <dS', S'> = e^{b_C} <dS', S> + sum_j E_j
    const float sds = red[0] + red[1] + red[2] + red[3];
    const float esum = red[4];
    atomicAdd(&dbt[cr.nv - 1], __expf(bC) * sds + esum);
  }
  __syncthreads();
  if (threadIdx.x < C && ok && threadIdx.x < cr.nv) {
    float acc = 0.f;
    for (int u = threadIdx.x; u < cr.nv; ++u) acc += dbt[u];
    red_add(bp.dlg + (size_t)(cr.t0 + threadIdx.x) * p.Hkv + cr.kv, acc);
  }
  if (issuer) {
    mma_commit(drain);
    mbar_wait(ld, 0, WaitCtx{never, nullptr, p.wait_ns});
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    mbar_wait(drain, 0, WaitCtx{never, nullptr, p.wait_ns});
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== scans

// Per (sequence, kv head), 1024 state elements per CTA (4 per thread): the state entering
// each chunk, h <- e^{b_C} h + dS_c, and from the last chunk back the gradient of the state
// leaving it, dh <- e^{b_C} dh + U_c; both written as bf16 operand images.  A sequence's
// chunks occupy consecutive slots.  Grid (n_seqs * Hkv, D * D / 1024), 256 threads.
template <int D>
__global__ void __launch_bounds__(256) bwd_scan_kernel(BwdParams bp) {
  griddep_wait_and_release();
  const tc::DevParams& p = bp.f;
  const int seq = blockIdx.x / p.Hkv, kv = blockIdx.x % p.Hkv;
  const int e = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (e >= D * D) return;
  const int r = e / D, c = e % D;
  const tc::SeqInfo si = p.seqs[seq];
  long q0, q1;
  seq_range(p.cu, seq, p.T, p.NT, &q0, &q1);
  // (never beyond the slots of the sequence's segments, even if the segment table failed)
  const int n_ch = (int)min((q1 - q0 + C - 1) / C, (long)si.n_seg * p.L);
  const size_t slot0 = (size_t)si.first_seg * p.L;
  const uint32_t ioff = img_off<D>(r, c);
  constexpr int kB = 8;   // chunks in flight
  auto store_img = [&](char* base, size_t ci, float4 x) {
    uint2 w;
    w.x = pack_bf16(x.x, x.y);
    w.y = pack_bf16(x.z, x.w);
    *reinterpret_cast<uint2*>(base + ci * (size_t)(D * D * 2) + ioff) = w;
  };
  const size_t mat = (size_t)D * D;
  // forward
  float4 h = bp.s0 ? *reinterpret_cast<const float4*>(bp.s0 + ((size_t)seq * p.Hkv + kv) * mat + e)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int f0 = 0; f0 < n_ch; f0 += kB) {
    float4 d[kB];
    float g[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (f0 + u < n_ch) {
        const size_t ci = (slot0 + f0 + u) * p.Hkv + kv;
        d[u] = __ldcs(reinterpret_cast<const float4*>(bp.dS + ci * mat + e));
        g[u] = __expf(p.bimg[ci * C + C - 1]);
      }
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (f0 + u < n_ch) {
        store_img(bp.Himg, (slot0 + f0 + u) * p.Hkv + kv, h);
        h = make_float4(fmaf(g[u], h.x, d[u].x), fmaf(g[u], h.y, d[u].y), fmaf(g[u], h.z, d[u].z),
                        fmaf(g[u], h.w, d[u].w));
      }
    }
  }
  // reverse: the final state's gradient summed over the group's q heads
  float4 dh = make_float4(0.f, 0.f, 0.f, 0.f);
  if (bp.dfs) {
    const int G = p.Hq / p.Hkv;
    for (int g = 0; g < G; ++g) {
      const float4 x = *reinterpret_cast<const float4*>(bp.dfs + ((size_t)seq * p.Hq + kv * G + g) * mat + e);
      dh = make_float4(dh.x + x.x, dh.y + x.y, dh.z + x.z, dh.w + x.w);
    }
  }
  for (int f0 = n_ch - 1; f0 >= 0; f0 -= kB) {
    float4 d[kB];
    float g[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (f0 - u >= 0) {
        const size_t ci = (slot0 + f0 - u) * p.Hkv + kv;
        d[u] = __ldcs(reinterpret_cast<const float4*>(bp.U + ci * mat + e));
        g[u] = __expf(p.bimg[ci * C + C - 1]);
      }
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (f0 - u >= 0) {
        store_img(bp.DHimg, (slot0 + f0 - u) * p.Hkv + kv, dh);
        dh = make_float4(fmaf(g[u], dh.x, d[u].x), fmaf(g[u], dh.y, d[u].y), fmaf(g[u], dh.z, d[u].z),
                         fmaf(g[u], dh.w, d[u].w));
      }
    }
  }
  if (bp.ds0) *reinterpret_cast<float4*>(bp.ds0 + ((size_t)seq * p.Hkv + kv) * mat + e) = dh;
}

// ============================================================== finalize

// dk = phi k (d phi k - <d phi k, phi k>) + dk_window + d log g sigmoid(-m) / D, dv; one
// warp per (token, kv head).  Grid (ceil(NT * Hkv / 8)), 256 threads.
template <int D>
__global__ void __launch_bounds__(256) bwd_finalize_kernel(BwdParams bp) {
  griddep_wait_and_release();
  const tc::DevParams& p = bp.f;
  const long unit = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (unit >= p.NT * p.Hkv) return;
  const int lane = threadIdx.x & 31;
  constexpr int E = D / 32;
  const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(bp.k);
  float x[E], m = -INFINITY, sum = 0.f;
#pragma unroll
  for (int u = 0; u < E; ++u) {
    x[u] = __bfloat162float(kin[unit * D + lane + 32 * u]);
    m = fmaxf(m, x[u]);
    sum += x[u];
  }
  m = warp_max(m);
  sum = warp_sum(sum);
  float z = 0.f;
#pragma unroll
  for (int u = 0; u < E; ++u) { x[u] = __expf(x[u] - m); z += x[u]; }
  z = warp_sum(z);
  const float iz = 1.f / z;
  float dp[E], dot = 0.f;
#pragma unroll
  for (int u = 0; u < E; ++u) {
    x[u] *= iz;
    dp[u] = bp.dphik[unit * D + lane + 32 * u];
    dot += dp[u] * x[u];
  }
  dot = warp_sum(dot);
  const float mean = sum / (float)D;
  // sigmoid(-mean) from the overflow-free log-sigmoid
  const float sgm = __expf(fminf(-mean, 0.f) - log1pf(__expf(-fabsf(mean))));
  const float gterm = bp.dlg[unit] * sgm / (float)D;
  __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(bp.dk);
  __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(bp.dv);
#pragma unroll
  for (int u = 0; u < E; ++u) {
    const long o = unit * D + lane + 32 * u;
    dk[o] = __float2bfloat16_rn(x[u] * (dp[u] - dot) + bp.dkw[o] + gterm);
    dv[o] = __float2bfloat16_rn(bp.dv_acc[o]);
  }
}

// ============================================================== host side

struct BwdLayout {
  tc::Plan pl;
  size_t off_dS, off_U, off_H, off_DH, off_dq, off_dphik, off_dkw, off_dv, off_dlg, total;
};

inline BwdLayout bwd_layout(int B, int Hq, int Hkv, long T, int d, int n_seqs, bool varlen) {
  BwdLayout L{};
  L.pl = tc::make_plan(B, Hq, Hkv, T, d, n_seqs, varlen);
  const long NT = varlen ? T : (long)B * T;
  const size_t units = (size_t)L.pl.n_seg_max * L.pl.L * Hkv;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = al(L.pl.total);
  L.off_dS = off;     off = al(off + units * d * d * 4);
  L.off_U = off;      off = al(off + units * d * d * 4);
  L.off_H = off;      off = al(off + units * d * d * 2);
  L.off_DH = off;     off = al(off + units * d * d * 2);
  L.off_dq = off;     off = al(off + (size_t)NT * Hq * d * 4);
  L.off_dphik = off;  off = al(off + (size_t)NT * Hkv * d * 4);
  L.off_dkw = off;    off = al(off + (size_t)NT * Hkv * d * 4);
  L.off_dv = off;     off = al(off + (size_t)NT * Hkv * d * 4);
  L.off_dlg = off;    off = al(off + (size_t)NT * Hkv * 4);
  L.total = off;
  return L;
}

inline size_t bwd_workspace_bytes(int B, int Hq, int Hkv, long T, int d, int n_seqs) {
  const BwdLayout a = bwd_layout(B, Hq, Hkv, T, d, B, false);
  const BwdLayout b = bwd_layout(1, Hq, Hkv, (long)B * T, d, n_seqs > 0 ? n_seqs : B, true);
  return a.total > b.total ? a.total : b.total;
}

struct BwdProblem {
  const void *q, *k, *v, *dout;
  const float *dfs, *s0;
  void *dq, *dk, *dv;
  float* ds0;
  const int32_t* cu;
  int B, Hq, Hkv;
  long T;
  int d, n_seqs;
  float alpha;
};

template <int D>
liger_status run_backward_d(const BwdProblem& pb, void* ws, cudaStream_t s, const tc::LaunchHooks& hk) {
  using tc::g_msg;
  const bool varlen = pb.cu != nullptr;
  const long NT = varlen ? pb.T : (long)pb.B * pb.T;
  const BwdLayout lay = bwd_layout(pb.B, pb.Hq, pb.Hkv, pb.T, D, pb.n_seqs, varlen);
  const tc::Plan& pl = lay.pl;
  char* w = static_cast<char*>(ws);
  BwdParams bp{};
  tc::PrefillProblem fp{pb.q, pb.k, pb.v, nullptr, nullptr, nullptr, pb.cu, pb.B, pb.Hq, pb.Hkv, pb.T, D, pb.n_seqs,
                        pb.alpha};
  bp.f = tc::fill_params(fp, w, pl, NT);
  bp.k = pb.k;
  bp.dout = pb.dout;
  bp.dfs = pb.dfs;
  bp.s0 = pb.s0;
  bp.ds0 = pb.ds0;
  bp.dS = reinterpret_cast<float*>(w + lay.off_dS);
  bp.U = reinterpret_cast<float*>(w + lay.off_U);
  bp.Himg = w + lay.off_H;
  bp.DHimg = w + lay.off_DH;
  bp.dq_acc = reinterpret_cast<float*>(w + lay.off_dq);
  bp.dphik = reinterpret_cast<float*>(w + lay.off_dphik);
  bp.dkw = reinterpret_cast<float*>(w + lay.off_dkw);
  bp.dv_acc = reinterpret_cast<float*>(w + lay.off_dv);
  bp.dlg = reinterpret_cast<float*>(w + lay.off_dlg);
  bp.dq = pb.dq;
  bp.dk = pb.dk;
  bp.dv = pb.dv;

  CUtensorMap mq, mdo, mk, mv;
  if (!tc::make_map(&mq, pb.q, D, pb.Hq, NT, 2) || !tc::make_map(&mdo, pb.dout, D, pb.Hq, NT, 2) ||
      !tc::make_map(&mk, pb.k, D, pb.Hkv, NT, 1) || !tc::make_map(&mv, pb.v, D, pb.Hkv, NT, 1)) {
    g_msg = "cuTensorMapEncodeTiled failed (driver entry point missing or unsupported layout)";
    return LIGER_ERR_CUDA;
  }
  // the key-side accumulators start at zero
  const size_t acc0 = lay.off_dphik, acc1 = lay.total;
  if (cudaMemsetAsync(w + acc0, 0, acc1 - acc0, s) != cudaSuccess) {
    g_msg = "clearing the backward accumulators failed";
    return LIGER_ERR_CUDA;
  }
  cudaError_t e;
  auto fail_launch = [&](cudaError_t err) { g_msg = cudaGetErrorString(err); return LIGER_ERR_CUDA; };
  // forward tables: segments, key images, gate sums
  e = tc::launch_chained(tc::plan_kernel, dim3(1), dim3(32), 0, s, bp.f, reinterpret_cast<tc::SeqInfo*>(w + pl.off_seqs),
                         reinterpret_cast<tc::SegInfo*>(w + pl.off_segs), reinterpret_cast<int32_t*>(w + 8));
  hk.count(1);
  if (e != cudaSuccess) return fail_launch(e);
  auto set_smem = [&](auto kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess;
  };
  if (!set_smem(tc::seg_state_kernel<D>, tc::SegSmem<D>::BYTES) || !set_smem(chunk_incr_kernel<D>, IncrSmem<D>::BYTES) ||
      !set_smem(bwd_window_kernel<D>, WinSmem<D>::BYTES) || !set_smem(bwd_recurrent_kernel<D>, RecSmem<D>::BYTES)) {
    cudaGetLastError();
    g_msg = "cudaFuncSetAttribute failed for a backward kernel";
    return LIGER_ERR_CUDA;
  }
  e = tc::launch_chained(tc::seg_state_kernel<D>, dim3((unsigned)pl.n_seg_max * pl.nsub * pb.Hkv), dim3(tc::kSegThreads),
                         tc::SegSmem<D>::BYTES, s, mk, mv, bp.f);
  hk.count(1);
  if (e != cudaSuccess) return fail_launch(e);
  const unsigned units = (unsigned)(pl.n_seg_max * pl.L);
  e = tc::launch_chained(chunk_incr_kernel<D>, dim3(units * pb.Hkv), dim3(160), IncrSmem<D>::BYTES, s, mq, mdo, mv, bp);
  hk.count(1);
  if (e != cudaSuccess) return fail_launch(e);
  e = tc::launch_chained(bwd_scan_kernel<D>, dim3((unsigned)(pb.n_seqs * pb.Hkv), (unsigned)(D * D / 1024)), dim3(256),
                         0, s, bp);
  hk.count(1);
  if (e != cudaSuccess) return fail_launch(e);
  hk.before_main(s);
  e = tc::launch_chained(bwd_window_kernel<D>, dim3(units * (pb.Hq / 2)), dim3(160), WinSmem<D>::BYTES, s, mq, mdo, mk,
                         mv, bp);
  hk.count(1);
  if (e != cudaSuccess) return fail_launch(e);
  e = tc::launch_chained(bwd_recurrent_kernel<D>, dim3(units * (pb.Hq / 2)), dim3(160), RecSmem<D>::BYTES, s, mq, mdo,
                         mv, bp);
  hk.after_main(s);
  hk.count(1);
  if (e != cudaSuccess) return fail_launch(e);
  const long fin_units = NT * pb.Hkv;
  e = tc::launch_chained(bwd_finalize_kernel<D>, dim3((unsigned)((fin_units + 7) / 8)), dim3(256), 0, s, bp);
  hk.count(1);
  if (e != cudaSuccess) return fail_launch(e);
  return LIGER_OK;
}

inline liger_status run_backward(const BwdProblem& pb, void* ws, cudaStream_t s, const tc::LaunchHooks& hk) {
  tc::g_msg = "";
  return pb.d == 64 ? run_backward_d<64>(pb, ws, s, hk) : run_backward_d<128>(pb, ws, s, hk);
}

}  // namespace bwd
}  // namespace liger
