// full_attn.cuh -- causal softmax attention on the sm_100a tensor cores (bf16).
//
// The standard attention layer of Liger's inter-layer hybrid: the news article
// on Liger (section ハイブリッドメカニズム) and the Paper-Notes page (section
// "Liger 整体架构") keep one full softmax attention layer after every seven
// Liger layers.  Per query head h with key/value head h / (Hq/Hkv):
//   o_t = sum_{j <= t} softmax_j(q_t . k_j / sqrt(d)) v_j      (causal, per sequence)
//
// One CTA per (128-token query block, q head, sequence), launched heaviest
// (latest) blocks first.  A TMA warp stages Q once and a 2-slot ring of
// 128-token key and value blocks; one thread issues the MMAs:
//   S_j = Q K_j^T   (M = 128 rows, N = 128 keys, fp32 in TMEM, two buffers)
//   O  += P_j V_j   (P_j bf16, written by the softmax warps into S_j's columns)
// Four softmax warps own one row each per thread: running maximum m and sum l
// (online softmax); the exponentials are taken against m, which is raised only
// when a block's maximum exceeds it by more than 2^8 (then the rows' O is
// rescaled in TMEM after the previous P.V has finished), so the exponentials
// stay below 2^8 and O is rarely touched.  The epilogue divides by l.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "liger_attn.h"
#include "sm100.cuh"

namespace liger {
namespace fa {

using namespace liger::sm100;

constexpr int BM = 128;                 // query rows (tokens) per CTA
constexpr int BN = 128;                 // keys per block
constexpr int kThreads = 192;           // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr float kRescaleLog2 = 8.f;     // raise the running maximum only beyond 2^8

struct Params {
  void* out;
  const int32_t* cu;     // [n + 1] or null
  long T;                // tokens per sequence, or the packed total
  int Hq, Hkv, n_qblk;   // n_qblk: query blocks per sequence in the grid (the longest)
  uint32_t* err;         // error word (timeouts) or null
  uint64_t wait_ns;
  float scale_log2;      // log2(e) / sqrt(d)
};

template <int D>
struct Smem {
  static constexpr uint32_t TILE = BM * D * 2;   // 128 rows x D bf16
  static constexpr uint32_t Q0 = 0;
  static constexpr uint32_t K0 = Q0 + TILE;      // 2 key slots
  static constexpr uint32_t V0 = K0 + 2 * TILE;  // 2 value slots
  static constexpr uint32_t SMALL = V0 + 2 * TILE;
  static constexpr uint32_t BYTES = SMALL + 256 + 1024;
};

// TMEM columns: S buffers at 0 and 128 (P_j packed into the first 64 columns of its
// buffer), O at 256.
constexpr uint32_t kColS0 = 0, kColO = 256;

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    full_attn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, Params p) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::SMALL);
  uint64_t* q_full = bars;          // [1]
  uint64_t* k_full = bars + 1;      // [2]
  uint64_t* k_empty = bars + 3;     // [2]
  uint64_t* v_full = bars + 5;      // [2]
  uint64_t* v_empty = bars + 7;     // [2]
  uint64_t* s_full = bars + 9;      // [2] S_j in its TMEM buffer
  uint64_t* p_ready = bars + 11;    // [2] P_j written (128 arrivals)
  uint64_t* pv_done = bars + 13;    // P_j V_j finished
  uint64_t* drain = bars + 14;      // every MMA of the CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never = tmem_slot + 2;

  // heaviest blocks first: blockIdx.x counts query blocks from the last one down
  const int qb = p.n_qblk - 1 - (int)blockIdx.x;
  const int h = blockIdx.y, seq = blockIdx.z;
  const int kv = h / (p.Hq / p.Hkv);
  const long NT = p.cu ? p.T : (long)gridDim.z * p.T;
  long q0, q1;
  seq_range(p.cu, seq, p.T, NT, &q0, &q1);
  const long len = q1 - q0;
  if ((long)qb * BM >= len) return;   // this sequence is shorter
  const int nblk = qb + 1;            // key blocks 0 .. qb (causal)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&p_ready[i], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    *never = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.err, p.wait_ns};

  if (warp == 4) {   // ---------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      auto load = [&](const CUtensorMap* m, char* dst, uint64_t* bar, int head, long tok) {
        mbar_arrive_expect_tx(bar, L::TILE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) tma_load_3d(dst + kb * BM * 128, m, bar, kb * 64, head, (int)tok);
      };
      load(&tmq, smem + L::Q0, q_full, h, q0 + (long)qb * BM);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&k_empty[s], ((j >> 1) - 1) & 1, wc, wsite(1, 1, j))) break;
        load(&tmk, smem + L::K0 + s * L::TILE, &k_full[s], kv, q0 + (long)j * BN);
        k_issued = j + 1;
        if (j >= 2 && !mbar_wait(&v_empty[s], ((j >> 1) - 1) & 1, wc, wsite(1, 2, j))) break;
        load(&tmv, smem + L::V0 + s * L::TILE, &v_full[s], kv, q0 + (long)j * BN);
        v_issued = j + 1;
      }
      const WaitCtx dw{never, nullptr, p.wait_ns};   // never leave with copies in flight
      mbar_wait(q_full, 0, dw);
      for (int j = (k_issued > 2 ? k_issued - 2 : 0); j < k_issued; ++j) mbar_wait(&k_full[j & 1], (j >> 1) & 1, dw);
      for (int j = (v_issued > 2 ? v_issued - 2 : 0); j < v_issued; ++j) mbar_wait(&v_full[j & 1], (j >> 1) & 1, dw);
    }
  } else if (warp == 5) {   // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(BM, BN, 0, 0);   // Q K^T: both K-major
      const uint32_t id_o = idesc_bf16(BM, D, 0, 1);    // P V: P from TMEM, V MN-major
      const uint32_t q_base = smem_u32(smem + L::Q0);
      bool ok = mbar_wait(q_full, 0, wc, wsite(2, 1, 0));
      auto issue_s = [&](int j) {
        const int s = j & 1;
        ok = ok && mbar_wait(&k_full[s], (j >> 1) & 1, wc, wsite(2, 2, j));
        if (!ok) return;
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + L::K0 + s * L::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_sw128(q_base + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(kb + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss(tmem + kColS0 + s * 128, a, b, id_s, kk > 0);
        }
        mma_commit(&s_full[s]);
        mma_commit(&k_empty[s]);
      };
      issue_s(0);
      if (nblk > 1) issue_s(1);
      for (int j = 0; j < nblk && ok; ++j) {
        const int s = j & 1;
        ok = ok && mbar_wait(&p_ready[s], (j >> 1) & 1, wc, wsite(2, 3, j));
        ok = ok && mbar_wait(&v_full[s], (j >> 1) & 1, wc, wsite(2, 4, j));
        if (!ok) break;
        tc_fence_after();
        const uint32_t vb = smem_u32(smem + L::V0 + s * L::TILE);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t b = sdesc_sw128(vb + kk * 2048, BN * 128, 1024);
          mma_bf16_ts(tmem + kColO, tmem + kColS0 + s * 128 + kk * 8, b, id_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(pv_done);
        mma_commit(&v_empty[s]);
        if (j + 2 < nblk) {
          // S_{j+2} reuses the buffer P_j was read from: wait until that product is done
          ok = ok && mbar_wait(pv_done, j & 1, wc, wsite(2, 5, j));
          issue_s(j + 2);
        }
      }
      mma_commit(drain);
    }
  } else {   // ---------------- softmax and epilogue (warps 0-3, thread = row)
    const int r = threadIdx.x;                    // query row in the block
    const long t = (long)qb * BM + r;             // its position in the sequence
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < nblk; ++j) {
      const int s = j & 1;
      const uint32_t sb = lane_base + kColS0 + s * 128;
      mbar_wait(&s_full[s], (j >> 1) & 1, wc, wsite(4, 1, j));
      tc_fence_after();
      // the row's 128 scores in registers (scaled to log2 units), masked on the diagonal block
      float x[BN];
#pragma unroll
      for (int c = 0; c < BN; c += 32) tmem_ld32(sb + c, x + c);
      tmem_wait_ld();
      const bool diag = j == qb;
      float bm = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        x[c] *= sl2;
        if (diag && c > r) x[c] = -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < BN; c += 2) bm = fmax3(bm, x[c], x[c + 1]);
      // raise the running maximum (and rescale this row's O and sum) only when the block's
      // maximum exceeds it by more than 2^8; decided per row, entered warp-wide
      const bool raise = bm > m + kRescaleLog2;
      if (__any_sync(0xffffffffu, raise)) {
        const float mn = raise ? bm : m;
        const float f = ex2(m - mn);   // 0 for the first block (m = -inf)
        if (j > 0) {
          // O holds the previous blocks' products: finish them, then rescale in TMEM
          mbar_wait(pv_done, (j - 1) & 1, wc, wsite(4, 2, j));
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            float o[32];
            tmem_ld32(lane_base + kColO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] *= f;
            tmem_st32(lane_base + kColO + c, o);
          }
          tmem_wait_st();
        }
        l *= f;
        m = mn;
      }
      const float2 nm2 = make_float2(-m, -m);
      float2 ls = make_float2(0.f, 0.f);
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        float2 y = fadd2(make_float2(x[c], x[c + 1]), nm2);
        y.x = ex2(y.x);
        y.y = ex2(y.y);
        ls = fadd2(ls, y);
        pk[c / 2] = pack_bf16(y.x, y.y);
      }
      l += ls.x + ls.y;
      // P_j over the first 64 columns of its S buffer (the scores there are in registers)
#pragma unroll
      for (int c = 0; c < BN / 2; c += 32) tmem_st32u(sb + c, pk + c);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_ready[s]);
    }
    // epilogue: O / l -> bf16 rows
    const bool live = mbar_wait(pv_done, (nblk - 1) & 1, wc, wsite(4, 3, nblk)) && !*abort_flag;
    tc_fence_after();
    const float il = 1.f / l;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + ((size_t)(q0 + t) * p.Hq + h) * D;
    const bool store = live && t < len;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      float o[32];
      tmem_ld32(lane_base + kColO + c, o);
      tmem_wait_ld();
      if (store) {
        uint32_t pw[16];
        const float2 il2 = make_float2(il, il);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float2 y = fmul2(make_float2(o[2 * u], o[2 * u + 1]), il2);
          pw[u] = pack_bf16(y.x, y.y);
        }
#pragma unroll
        for (int u = 0; u < 16; u += 4)
          *reinterpret_cast<uint4*>(orow + c + 2 * u) = make_uint4(pw[u], pw[u + 1], pw[u + 2], pw[u + 3]);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    mbar_wait(drain, 0, WaitCtx{never, nullptr, p.wait_ns});
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ============================================================== host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// A (d, head, token) bf16 tensor map with a (64, 1, 128) box and 128-byte swizzle.
inline bool make_map(EncodeTiledFn enc, CUtensorMap* m, const void* ptr, int d, int H, long NT) {
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)NT};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)BM};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace fa
}  // namespace liger
