// full_attn.cuh -- causal softmax attention on the sm_100a tensor cores (bf16).
//
// The standard attention layer of Liger's inter-layer hybrid: the news article
// on Liger (section ハイブリッドメカニズム) and the Paper-Notes page (section
// "Liger 整体架构") keep one full softmax attention layer after every seven
// Liger layers.  Per query head h with key/value head h / (Hq/Hkv):
//   o_t = sum_{j <= t} softmax_j(q_t . k_j / sqrt(d)) v_j      (causal, per sequence)
//
// One CTA per (pair of 128-token query blocks, q head, sequence), launched heaviest
// (latest) pairs first.  The two query tiles A and B take turns on the tensor pipe while
// each has its own softmax warpgroup, so one tile's softmax runs under the other
// tile's products.  A TMA warp stages both Q tiles once and a 2-slot ring of 128-token
// key and value blocks; one thread issues the MMAs:
//   S_t = Q_t K_j^T  (M = 128 rows, N = 128 keys, fp32 in TMEM, one buffer per tile)
//   O_t += P_t V_j   (P_t bf16, written by the tile's softmax warps over S_t's columns)
// Each softmax thread owns one row: running maximum m and sum l (online softmax); the
// exponentials are taken against m, which is raised only when a block's maximum exceeds
// it by more than 2^8 (then the rows' O is rescaled in TMEM after the previous P.V has
// finished), so the exponentials stay below 2^8 and O is rarely touched.  The epilogue
// divides by l.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "liger_attn.h"
#include "sm100.cuh"

namespace liger {
namespace fa {

using namespace liger::sm100;

constexpr int BM = 128;                 // query rows (tokens) per tile; two tiles per CTA
constexpr int BN = 128;                 // keys per block
constexpr int kThreads = 320;           // warps 0-3 softmax A, 4-7 softmax B, 8 TMA, 9 MMA
constexpr float kRescaleLog2 = 8.f;     // raise the running maximum only beyond 2^8
constexpr int kPolyPairs = 2;           // of every 8 column pairs off the diagonal: 2^x by polynomial

struct Params {
  void* out;
  const int32_t* cu;     // [n + 1] or null
  long T;                // tokens per sequence, or the packed total
  int Hq, Hkv, n_qblk;   // n_qblk: 128-token query blocks of the longest sequence
  uint32_t* err;         // error word (timeouts) or null
  uint64_t wait_ns;
  float scale_log2;      // log2(e) / sqrt(d)
};

template <int D>
struct Smem {
  static constexpr uint32_t TILE = BM * D * 2;   // 128 rows x D bf16
  static constexpr uint32_t Q0 = 0;              // 2 query tiles
  static constexpr uint32_t K0 = Q0 + 2 * TILE;  // 2 key slots
  static constexpr uint32_t V0 = K0 + 2 * TILE;  // 2 value slots
  static constexpr uint32_t SMALL = V0 + 2 * TILE;
  static constexpr uint32_t BYTES = SMALL + 256 + 1024;
};

// TMEM columns: the scores of tile t at 128 t (P_t packed into their first 64 columns),
// its output accumulator at 256 + 128 t.
constexpr uint32_t kColS0 = 0, kColO = 256;

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    full_attn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, Params p) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) char smem_raw[];
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::SMALL);
  uint64_t* q_full = bars;          // [1] both query tiles
  uint64_t* k_full = bars + 1;      // [2]
  uint64_t* k_empty = bars + 3;     // [2]
  uint64_t* v_full = bars + 5;      // [2]
  uint64_t* v_empty = bars + 7;     // [2]
  uint64_t* s_full = bars + 9;      // [tile] S_t of the current block in TMEM
  uint64_t* p_ready = bars + 11;    // [tile] P_t written (128 arrivals)
  uint64_t* pv_done = bars + 13;    // [tile] P_t V_j finished
  uint64_t* drain = bars + 15;      // every MMA of the CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* never = tmem_slot + 2;

  // heaviest pairs first: blockIdx.x counts query-block pairs from the last one down
  const int n_pair = (p.n_qblk + 1) / 2;
  const int pi = n_pair - 1 - (int)blockIdx.x;
  const int h = blockIdx.y, seq = blockIdx.z;
  const int kv = h / (p.Hq / p.Hkv);
  const long NT = p.cu ? p.T : (long)gridDim.z * p.T;
  long q0, q1;
  seq_range(p.cu, seq, p.T, NT, &q0, &q1);
  const long len = q1 - q0;
  if ((long)pi * 2 * BM >= len) return;   // this sequence is shorter
  // tile t holds query block 2 pi + t and sees key blocks 0 .. 2 pi + t (causal)
  const int nA = 2 * pi + 1, nB = 2 * pi + 2;   // key blocks of tiles A and B
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&p_ready[i], 128); mbar_init(&pv_done[i], 1);
    }
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

  if (warp == 8) {   // ---------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      auto load = [&](const CUtensorMap* m, char* dst, uint64_t* bar, int head, long tok) {
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) tma_load_3d(dst + kb * BM * 128, m, bar, kb * 64, head, (int)tok);
      };
      mbar_arrive_expect_tx(q_full, 2 * L::TILE);
      load(&tmq, smem + L::Q0, q_full, h, q0 + (long)(2 * pi) * BM);
      load(&tmq, smem + L::Q0 + L::TILE, q_full, h, q0 + (long)(2 * pi + 1) * BM);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nB; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&k_empty[s], ((j >> 1) - 1) & 1, wc, wsite(1, 1, j))) break;
        mbar_arrive_expect_tx(&k_full[s], L::TILE);
        load(&tmk, smem + L::K0 + s * L::TILE, &k_full[s], kv, q0 + (long)j * BN);
        k_issued = j + 1;
        if (j >= 2 && !mbar_wait(&v_empty[s], ((j >> 1) - 1) & 1, wc, wsite(1, 2, j))) break;
        mbar_arrive_expect_tx(&v_full[s], L::TILE);
        load(&tmv, smem + L::V0 + s * L::TILE, &v_full[s], kv, q0 + (long)j * BN);
        v_issued = j + 1;
      }
      const WaitCtx dw{never, nullptr, p.wait_ns};   // never leave with copies in flight
      mbar_wait(q_full, 0, dw);
      for (int j = (k_issued > 2 ? k_issued - 2 : 0); j < k_issued; ++j) mbar_wait(&k_full[j & 1], (j >> 1) & 1, dw);
      for (int j = (v_issued > 2 ? v_issued - 2 : 0); j < v_issued; ++j) mbar_wait(&v_full[j & 1], (j >> 1) & 1, dw);
    }
  } else if (warp == 9) {   // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(BM, BN, 0, 0);   // Q K^T: both K-major
      const uint32_t id_o = idesc_bf16(BM, D, 0, 1);    // P V: P from TMEM, V MN-major
      bool ok = mbar_wait(q_full, 0, wc, wsite(2, 1, 0));
      // S_t(j) = Q_t K_j^T.  Tile B is the later user of key block j: it releases the slot
      // (tile A has no block 2 pi + 1, so there B alone uses it).
      auto issue_s = [&](int t, int j) {
        const int s = j & 1;
        if (t == 0 || j >= nA) ok = ok && mbar_wait(&k_full[s], (j >> 1) & 1, wc, wsite(2, 2, j));
        if (!ok) return;
        tc_fence_after();
        const uint32_t qb = smem_u32(smem + L::Q0 + t * L::TILE);
        const uint32_t kb = smem_u32(smem + L::K0 + s * L::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_sw128(qb + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(kb + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss(tmem + kColS0 + t * 128, a, b, id_s, kk > 0);
        }
        mma_commit(&s_full[t]);
        if (t == 1) mma_commit(&k_empty[s]);
      };
      // O_t += P_t(j) V_j.  Tile B is the later user of value block j as well.
      auto issue_pv = [&](int t, int j) {
        const int s = j & 1;
        ok = ok && mbar_wait(&p_ready[t], j & 1, wc, wsite(2, 3 + t, j));
        if (t == 0 || j >= nA) ok = ok && mbar_wait(&v_full[s], (j >> 1) & 1, wc, wsite(2, 5, j));
        if (!ok) return;
        tc_fence_after();
        const uint32_t vb = smem_u32(smem + L::V0 + s * L::TILE);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t b = sdesc_sw128(vb + kk * 2048, BN * 128, 1024);
          mma_bf16_ts(tmem + kColO + t * 128, tmem + kColS0 + t * 128 + kk * 8, b, id_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&pv_done[t]);
        if (t == 1) mma_commit(&v_empty[s]);
      };
      // S_t(j + 1) lies over P_t(j): it goes out after P_t(j) V_j (the tensor pipe runs the
      // products in issue order)
      issue_s(0, 0);
      issue_s(1, 0);
      for (int j = 0; j < nB && ok; ++j) {
        if (j < nA) {
          issue_pv(0, j);
          if (j + 1 < nA) issue_s(0, j + 1);
        }
        issue_pv(1, j);
        if (j + 1 < nB) issue_s(1, j + 1);
      }
      mma_commit(drain);
    }
  } else {   // ---------------- softmax and epilogue: tile t = warp / 4, thread = row
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;                  // query row in the tile
    const long tok = (long)(2 * pi + t) * BM + r;     // its position in the sequence
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t sb = lane_base + kColS0 + t * 128, ob = lane_base + kColO + t * 128;
    const float sl2 = p.scale_log2;
    const int diag_blk = 2 * pi + t;
    float m = -INFINITY, l = 0.f;
    const int nb = t ? nB : nA;
    for (int j = 0; j < nb; ++j) {
      mbar_wait(&s_full[t], j & 1, wc, wsite(4, 1 + t, j));
      tc_fence_after();
      // the row's 128 scores in registers (scaled to log2 units), masked on the diagonal block
      float x[BN];
#pragma unroll
      for (int c = 0; c < BN; c += 32) tmem_ld32(sb + c, x + c);
      tmem_wait_ld();
      const bool diag = j == diag_blk;
      float bm = -INFINITY;
      if (diag) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c > r) x[c] = -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < BN; c += 2) bm = fmax3(bm, x[c], x[c + 1]);
      bm *= sl2;   // the scale is positive: the maximum of the scaled scores
      // raise the running maximum (and rescale this row's O and sum) only when the block's
      // maximum exceeds it by more than 2^8; decided per row, entered warp-wide
      const bool raise = bm > m + kRescaleLog2;
      if (__any_sync(0xffffffffu, raise)) {
        const float mn = raise ? bm : m;
        const float f = ex2(m - mn);   // 0 for the first block (m = -inf)
        if (j > 0) {
          // O holds the previous blocks' products: finish them, then rescale in TMEM
          mbar_wait(&pv_done[t], (j - 1) & 1, wc, wsite(4, 3 + t, j));
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            float o[32];
            tmem_ld32(ob + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] *= f;
            tmem_st32(ob + c, o);
          }
          tmem_wait_st();
        }
        l *= f;
        m = mn;
      }
      const float2 nm2 = make_float2(-m, -m), s2 = make_float2(sl2, sl2);
      float2 ls = make_float2(0.f, 0.f);
      // P over the first 64 columns of the tile's score buffer (the scores are in
      // registers), written eight columns at a time so that fewer values are live at once.
      // Off the diagonal block, kPolyPairs of every eight column pairs take 2^x from the
      // FMA pipes (exp2_poly2) instead of the special-function unit, the busier of the two
      // here; the diagonal block (with its masked -inf scores) stays on the unit.
      auto write_p = [&](auto poly) {
#pragma unroll
        for (int h4 = 0; h4 < 8; ++h4) {
          uint32_t pk[8];
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            float2 y = ffma2(make_float2(x[h4 * 16 + c], x[h4 * 16 + c + 1]), s2, nm2);
            if (decltype(poly)::value && c >= 16 - 2 * kPolyPairs) {
              y = exp2_poly2(y);
            } else {
              y.x = ex2(y.x);
              y.y = ex2(y.y);
            }
            ls = fadd2(ls, y);
            pk[c / 2] = pack_bf16(y.x, y.y);
          }
          tmem_st8u(sb + h4 * 8, pk);
        }
      };
      if (diag) write_p(std::false_type{});
      else write_p(std::true_type{});
      l += ls.x + ls.y;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_ready[t]);
    }
    // epilogue: O / l -> bf16 rows
    const bool live = warp_all(mbar_wait(&pv_done[t], (nb - 1) & 1, wc, wsite(4, 5 + t, nb)) &&
                               !*abort_flag);
    tc_fence_after();
    const float il = 1.f / l;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + ((size_t)(q0 + tok) * p.Hq + h) * D;
    const bool store = live && tok < len;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      float o[32];
      tmem_ld32(ob + c, o);
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
