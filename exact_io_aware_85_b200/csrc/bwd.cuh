// bwd.cuh — exact attention backward on B200 by recomputation.
//
// The forward pass keeps only O and the row logsumexp; the backward pass
// recomputes the score tiles from Q, K and that logsumexp instead of storing
// the N x N probabilities ("flash-attention-trading-models", section "Pase hacia
// atras": O(N) statistics, redundant arithmetic traded for the N^2 memory term).
// With P = exp(scale S - LSE) and D_q = sum_c dO_qc O_qc (= sum_k P_qk dP_qk):
//   dV = P^T dO,  dP = dO V^T,  dS = scale P o (dP - D),  dQ = dS K,  dK = dS^T Q.
//
// Three launches on the caller's stream:
//   bwd_pre   D, LSE*log2(e) into padded workspace rows, zero the fp32 dQ accumulator
//   bwd_main  one CTA per (128-key tile, batch*head): K_j, V_j stay in shared memory,
//             the CTA walks the query tiles (from the diagonal when causal);
//             tcgen05 MMAs: S^T = K Q^T, dP^T = V dO^T (into TMEM), then
//             dV += P^T dO (P^T from TMEM), dK += dS^T Q, dQ_i = dS K;
//             dV, dK accumulate in TMEM over the whole walk; each dQ_i tile is
//             added into the fp32 accumulator in global memory.
//   bwd_post  dQ accumulator -> bf16
//
// Warp roles in bwd_main (448 threads):
//   warps 0-7   gradient warps: thread = key row (TMEM lane); warps 0-3 own query
//               columns 0-63, warps 4-7 columns 64-127 of each tile
//   warps 8-11  dQ drain: TMEM -> fp32 reductions into global memory
//   warp 12     TMA producer (K_j, V_j once; Q_i, dO_i, LSE_i, D_i double-buffered)
//   warp 13     tcgen05.mma issuer and TMEM owner
// Tensor memory (fp32 columns): dV [0,d), dK [d,2d), S^T [2d,2d+128) with P^T
// (bf16) written over its first 64 columns, dP^T [2d+128,2d+256); dQ_i reuses the
// dP^T columns when d = 128 (the budget is full) and has its own when d = 64.
#pragma once
#include "sm100.cuh"

namespace fa {

// ---------------------------------------------------------------------------
// bwd_pre: one group of D/8 threads per query row (16-byte vectors)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse, float* __restrict__ lse2,
                                                         float* __restrict__ dvec, float* __restrict__ dq_acc, int N,
                                                         int Npad, long long rows_total) {
  constexpr int TPR = D / 8;  // threads per row
  const long long gtid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gtid / TPR;  // padded row index over BH * Npad
  const int part = static_cast<int>(gtid % TPR);
  if (row >= rows_total) return;
  const long long bh = row / Npad;
  const int n = static_cast<int>(row % Npad);
  float acc = 0.f;
  if (n < N) {
    const size_t base = (static_cast<size_t>(bh) * N + n) * D + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + base);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + base);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(pa[e]);
      const float2 y = __bfloat1622float2(pb[e]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, TPR);
  if (part == 0) {
    dvec[row] = acc;  // 0 on padding rows
    lse2[row] = n < N ? lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f : INFINITY;  // pad: P = 0
  }
  float4* z = reinterpret_cast<float4*>(dq_acc + static_cast<size_t>(row) * D + part * 8);
  z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// bwd_post: dQ accumulator (fp32, padded rows) times f -> bf16 (f is the
// softmax scale when the main pass accumulated dS / scale, 1 otherwise)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_post_kernel(const float* __restrict__ dq_acc,
                                                          __nv_bfloat16* __restrict__ dq, int N, int Npad,
                                                          long long vec_total, float f) {
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;  // one 8-element vector
  if (g >= vec_total) return;
  constexpr int VPR = D / 8;
  const long long row = g / VPR;  // unpadded row over BH * N
  const int part = static_cast<int>(g % VPR);
  const long long bh = row / N;
  const int n = static_cast<int>(row % N);
  const float4* src = reinterpret_cast<const float4*>(dq_acc + (static_cast<size_t>(bh) * Npad + n) * D + part * 8);
  const float4 a = src[0], b = src[1];
  uint4 w;
  w.x = pack_bf16x2(a.x * f, a.y * f);
  w.y = pack_bf16x2(a.z * f, a.w * f);
  w.z = pack_bf16x2(b.x * f, b.y * f);
  w.w = pack_bf16x2(b.z * f, b.w * f);
  *reinterpret_cast<uint4*>(dq + static_cast<size_t>(row) * D + part * 8) = w;
}

// ---------------------------------------------------------------------------
// bwd_main
// ---------------------------------------------------------------------------
struct BwdArgs {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* lse2;  // [BH, Npad] LSE * log2(e), +inf on padding rows
  const float* dvec;  // [BH, Npad] D, 0 on padding rows
  float* dq_acc;      // [BH, Npad, d]
  int N, Npad, BH, n_tiles;
  int group;         // query heads per key/value head (1 = multi-head attention)
  int BHkv;          // batch * key/value heads
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  int causal;
};

template <int D>
struct BwdCfg {
  static constexpr int TILE = 128 * D * 2;   // one 128 x D bf16 tile
  static constexpr int NBOX = D / 64;        // 128-byte swizzled column blocks
  static constexpr int BOX = 16384;          // 128 rows x 128 bytes
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;          // 2 stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;     // 2 stages
  static constexpr int OFF_DS = OFF_DO + 2 * TILE;    // dS^T, 128 keys x 128 queries bf16 (2 blocks)
  static constexpr int OFF_LSE = OFF_DS + 2 * BOX;    // 2 stages x 128 floats
  static constexpr int OFF_DV = OFF_LSE + 2 * 512;    // 2 stages x 128 floats
  static constexpr int OFF_BAR = OFF_DV + 2 * 512;
  static constexpr int SMEM_BYTES = OFF_BAR + 256;
  static constexpr uint32_t COL_DV = 0, COL_DK = D, COL_S = 2 * D, COL_DP = 2 * D + 128;
  static constexpr bool DQ_SHARES_DP = (2 * D + 256 + D > 512);
  static constexpr uint32_t COL_DQ = DQ_SHARES_DP ? COL_DP : 2 * D + 256;
  static constexpr int NTHREADS = 448;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// dst[0..1] += (lo, hi) (fp32) as one 8-byte reduction in the L2
__device__ __forceinline__ void red_add_v2(float* dst, float lo, float hi) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(dst), "f"(lo), "f"(hi) : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// 16-byte chunk c (0..7) of row r inside a 128-byte-swizzled block
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(448, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars + 0;
  uint64_t* bar_ld_full = bars + 1;   // [2]
  uint64_t* bar_ld_empty = bars + 3;  // [2]
  uint64_t* bar_s_full = bars + 5;
  uint64_t* bar_dp_full = bars + 6;
  uint64_t* bar_pds = bars + 7;
  uint64_t* bar_ds_free = bars + 8;
  uint64_t* bar_dq_full = bars + 9;
  uint64_t* bar_dq_free = bars + 10;
  uint64_t* bar_acc = bars + 11;
  uint64_t* bar_done = bars + 12;
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_sh = reinterpret_cast<volatile int*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  const int bh_kv = blockIdx.x % a.BHkv;  // key/value head
  const int j = blockIdx.x / a.BHkv;      // key tile; j = 0 (the longest walk when causal) first
  const int i0 = a.causal ? j : 0;
  const int spq = a.n_tiles - i0;         // query tiles per query head
  const int steps = spq * a.group;        // the walk covers every query head of the group
  // step t -> (query head, query tile)
  auto step_head = [&](int t) { return bh_kv * a.group + t / spq; };
  auto step_tile = [&](int t) { return i0 + t % spq; };

  // the swizzled TMA/UMMA layouts need a 1024-byte aligned base
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&g_fa_status, 0, 4 /*FA_ERR_CUDA*/ | (99 << 8));
    return;
  }
  if (warp == 13) {
    tmem_alloc(tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    *abort_sh = 0;
    mbar_init(bar_kv, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_ld_full + s, 1);
      mbar_init(bar_ld_empty + s, 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_pds, 256);
    mbar_init(bar_ds_free, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_free, 128);
    mbar_init(bar_acc, 1);
    mbar_init(bar_done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sh;

  if (warp == 12) {
    // ============================ producer ===================================
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar_kv, 2 * C::TILE);
      for (int b = 0; b < C::NBOX; ++b) {
        tma_load_3d(smem + C::OFF_K + b * C::BOX, &tmK, bar_kv, b * 64, j * 128, bh_kv);
        tma_load_3d(smem + C::OFF_V + b * C::BOX, &tmV, bar_kv, b * 64, j * 128, bh_kv);
      }
      int t = 0;
      for (; t < steps; ++t) {
        const int i = step_tile(t), hq = step_head(t);
        const int s = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        if (!mbar_wait(bar_ld_empty + s, ph ^ 1, abort_sh, 40)) break;
        mbar_arrive_expect_tx(bar_ld_full + s, 2 * C::TILE + 1024);
        for (int b = 0; b < C::NBOX; ++b) {
          tma_load_3d(smem + C::OFF_Q + s * C::TILE + b * C::BOX, &tmQ, bar_ld_full + s, b * 64, i * 128, hq);
          tma_load_3d(smem + C::OFF_DO + s * C::TILE + b * C::BOX, &tmDO, bar_ld_full + s, b * 64, i * 128, hq);
        }
        const size_t roff = static_cast<size_t>(hq) * a.Npad + static_cast<size_t>(i) * 128;
        bulk_load(smem + C::OFF_LSE + s * 512, a.lse2 + roff, 512, bar_ld_full + s);
        bulk_load(smem + C::OFF_DV + s * 512, a.dvec + roff, 512, bar_ld_full + s);
      }
      // teardown: let the copies in flight land
      mbar_wait_drain(bar_kv, 0, 100000000ull);
      for (int u = max(0, t - 2); u < t; ++u) mbar_wait_drain(bar_ld_full + (u & 1), (u >> 1) & 1, 100000000ull);
    }
  } else if (warp == 13) {
    // ============================ MMA issuer =================================
    if (lane == 0) {
      constexpr uint32_t id_ss = make_idesc(128, 128, kFmtBF16, 0, 0);      // S^T, dP^T
      constexpr uint32_t id_dv = make_idesc(128, D, kFmtBF16, 0, 1);        // dV (A from TMEM)
      constexpr uint32_t id_dk = make_idesc(128, D, kFmtBF16, 0, 1);        // dK
      constexpr uint32_t id_dq = make_idesc(128, D, kFmtBF16, 1, 1);        // dQ (A = dS, MN-major)
      const uint32_t k_addr = smem_u32(smem + C::OFF_K), v_addr = smem_u32(smem + C::OFF_V);
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q), do_addr = smem_u32(smem + C::OFF_DO);
      const uint32_t ds_addr = smem_u32(smem + C::OFF_DS);
      bool ok = mbar_wait(bar_kv, 0, abort_sh, 41);
      for (int t = 0; ok && t < steps; ++t) {
        const int s = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        if (!(ok = mbar_wait(bar_ld_full + s, ph, abort_sh, 42))) break;
        tc_fence_after();
        const uint32_t qa = q_addr + s * C::TILE, da = do_addr + s * C::TILE;
        // S^T = K_j Q_i^T    (M = 128 keys, N = 128 queries, K = d)
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::COL_S, make_sdesc_sw128(k_addr + off, 16, 1024), make_sdesc_sw128(qa + off, 16, 1024),
                 id_ss, k > 0);
        }
        mma_commit(bar_s_full);
        if (C::DQ_SHARES_DP && t > 0) {
          if (!(ok = mbar_wait(bar_dq_free, (t - 1) & 1, abort_sh, 43))) break;
          tc_fence_after();
        }
        // dP^T = V_j dO_i^T
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::COL_DP, make_sdesc_sw128(v_addr + off, 16, 1024), make_sdesc_sw128(da + off, 16, 1024),
                 id_ss, k > 0);
        }
        mma_commit(bar_dp_full);
        if (!(ok = mbar_wait(bar_pds, t & 1, abort_sh, 44))) break;
        tc_fence_after();
        // dV += P^T dO_i   (A = P^T from TMEM, K = 128 queries; B = dO_i MN-major)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tmem + C::COL_DV, tmem + C::COL_S + k * 8, make_sdesc_sw128(da + k * 2048, C::BOX, 1024), id_dv,
                 (t > 0 || k > 0) ? 1u : 0u);
        // dK += dS^T Q_i   (A = dS^T K-major in smem; B = Q_i MN-major)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::COL_DK, make_sdesc_sw128(ds_addr + off, 16, 1024),
                 make_sdesc_sw128(qa + k * 2048, C::BOX, 1024), id_dk, (t > 0 || k > 0) ? 1u : 0u);
        }
        if (!C::DQ_SHARES_DP && t > 0) {
          if (!(ok = mbar_wait(bar_dq_free, (t - 1) & 1, abort_sh, 45))) break;
          tc_fence_after();
        }
        // dQ_i = dS K_j     (A = dS: the dS^T buffer read MN-major; B = K_j MN-major)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + C::COL_DQ, make_sdesc_sw128(ds_addr + k * 2048, C::BOX, 1024),
                 make_sdesc_sw128(k_addr + k * 2048, C::BOX, 1024), id_dq, k > 0 ? 1u : 0u);
        mma_commit(bar_dq_full);
        mma_commit(bar_ld_empty + s);
        mma_commit(bar_ds_free);
      }
      if (ok) mma_commit(bar_acc);
      mma_commit(bar_done);
      mbar_wait_drain(bar_done, 0, 100000000ull);
    }
  } else if (warp >= 8) {
    // ============================ dQ drain ===================================
    const int r = threadIdx.x - 256;  // query row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    for (int t = 0; t < steps; ++t) {
      const int i = step_tile(t), hq = step_head(t);
      if (!mbar_wait(bar_dq_full, t & 1, abort_sh, 46)) break;
      tc_fence_after();
      float* dst = a.dq_acc + (static_cast<size_t>(hq) * a.Npad + static_cast<size_t>(i) * 128 + r) * D;
      const bool live = i * 128 + r < N;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + C::COL_DQ + ch * 32, v);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            atomicAdd(reinterpret_cast<float4*>(dst + ch * 32 + 4 * e),
                      make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                  __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3])));
        }
      }
      tc_fence_before();
      mbar_arrive(bar_dq_free);
    }
  } else {
    // ============================ gradient warps =============================
    const int half = warp >> 2;                  // query columns [64 half, 64 half + 64)
    const int r = threadIdx.x & 127;             // key row in tile == TMEM lane
    const int key = j * 128 + r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float c = a.scale_log2;
    bool ok = true;
    for (int t = 0; t < steps && ok; ++t) {
      const int i = step_tile(t);
      const int s = t & 1;
      const float* lse2 = reinterpret_cast<const float*>(smem + C::OFF_LSE + s * 512) + half * 64;
      const float* dv = reinterpret_cast<const float*>(smem + C::OFF_DV + s * 512) + half * 64;
      const int q0 = i * 128 + half * 64;
      const bool need_mask = (a.causal && i == j) || key >= N;
      if (!(ok = mbar_wait(bar_s_full, t & 1, abort_sh, 47))) break;
      tc_fence_after();
      float p[64];
      tmem_ld32(tmem + lane_base + C::COL_S + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
      tmem_ld32(tmem + lane_base + C::COL_S + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        float x = ex2_approx(fmaf(p[e], c, -lse2[e]));
        if (need_mask && (key >= N || (a.causal && key > q0 + e))) x = 0.f;
        p[e] = x;
      }
      // both halves have read S^T before P^T is written over its first 64 columns
      named_bar_sync(1, 256);
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
        tmem_st32(tmem + lane_base + C::COL_S + half * 32, pk);
      }
      if (!(ok = mbar_wait(bar_ds_free, (t & 1) ^ 1, abort_sh, 48))) break;
      if (!(ok = mbar_wait(bar_dp_full, t & 1, abort_sh, 49))) break;
      tc_fence_after();
      uint8_t* dsb = smem + C::OFF_DS + half * C::BOX;  // queries [64 half, +64) live in block `half`
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t dp[32];
        tmem_ld32(tmem + lane_base + C::COL_DP + half * 64 + h2 * 32, dp);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {  // 4 chunks of 8 queries
          uint4 w;
          uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int qi = h2 * 32 + cc * 8 + 2 * e;
            const float d0 = a.scale * p[qi] * (__uint_as_float(dp[cc * 8 + 2 * e]) - dv[qi]);
            const float d1 = a.scale * p[qi + 1] * (__uint_as_float(dp[cc * 8 + 2 * e + 1]) - dv[qi + 1]);
            wp[e] = pack_bf16x2(d0, d1);
          }
          *reinterpret_cast<uint4*>(dsb + sw128_off(r, h2 * 4 + cc)) = w;
        }
      }
      tmem_wait_st();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(bar_pds);
    }
    // ---- epilogue: dV (warps 0-3) and dK (warps 4-7) -> bf16 -------------------
    if (ok) ok = mbar_wait(bar_acc, 0, abort_sh, 50);
    if (ok) {
      tc_fence_after();
      const uint32_t col = half ? C::COL_DK : C::COL_DV;
      __nv_bfloat16* dst = (half ? a.dk : a.dv) + (static_cast<size_t>(bh_kv) * N + key) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + col + ch * 32, v);
        tmem_wait_ld();
        if (key < N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * v4 + 0]), __uint_as_float(v[8 * v4 + 1]));
            w.y = pack_bf16x2(__uint_as_float(v[8 * v4 + 2]), __uint_as_float(v[8 * v4 + 3]));
            w.z = pack_bf16x2(__uint_as_float(v[8 * v4 + 4]), __uint_as_float(v[8 * v4 + 5]));
            w.w = pack_bf16x2(__uint_as_float(v[8 * v4 + 6]), __uint_as_float(v[8 * v4 + 7]));
            d4[v4] = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// bwd_main at d = 128 with 128-query steps
// ---------------------------------------------------------------------------
// One CTA per (128-key tile, key/value head), K_j and V_j resident.  Each step
// takes 128 queries, so S^T, dP^T and dQ^T are N = 128 MMAs (a shared-memory
// MMA costs about the same ~110 cycles per 16-deep step at N = 64 as at N = 128,
// so this halves their cost per FLOP against 64-query steps).  Tensor memory
// holds one step (dV, dK, S^T, dP^T: all 512 columns), so the step's hand-offs
// are split finely enough that the tensor core stays busy:
//   S^T(t) -> [gradient warps: P]  dP^T(t) -> [gradient warps: dS]
//   dV(t) as soon as P^T is stored (while dS is computed), dK(t) once dS^T is
//   stored, dQ^T(t) into the dP^T columns (after dK has read dS^T there), then
//   S^T(t+1) while the drain warps empty dQ^T(t), then dP^T(t+1).
// The gradient warps read neither LSE nor D: the accumulators start from them.
// Before S^T(t) the drain warps fill the S^T columns with -LSE_q / scale (one
// row per key, every row the same) and before dP^T(t) the dP^T columns with
// -D_q, and the two MMAs accumulate onto them, so the gradient warps compute
// P = 2^(scale log2(e) acc) and dS = P acc' straight from tensor memory.  The
// softmax scale of dS is applied to dK in its epilogue and to dQ in the post
// pass.  dQ^T(t) is drained with coalesced fp32 reductions (a warp adds 32
// consecutive head-dimension entries of one query row).
// Warp roles (16 warps; registers per thread after setmaxnreg):
//   warps 0-7   gradient warps (136): thread = key row (TMEM lane); warps 0-3
//               queries 0-63 of the step, warps 4-7 queries 64-127
//   warps 8-11  dQ drain and accumulator set-up (152): thread = TMEM lane
//   warp  12    TMA producer, warp 13 MMA issuer and TMEM owner, 14-15 idle (88)
// Launched at 128 registers a thread: 2 x 128 x 136 + 128 x 152 + 128 x 88 =
// 65536 = 512 x 128, and 136 + 136 + 152 + 88 = 512 per sub-partition.
struct BwdQ128Cfg {
  static constexpr int D = 128;
  static constexpr int BOX = 16384;             // 128 rows x 128 bytes
  static constexpr int TILE = 2 * BOX;          // 128 rows x 128 bf16 columns
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int NST = 2;                 // Q/dO/LSE/D load stages
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + NST * TILE;
  static constexpr int OFF_DS = OFF_DO + NST * TILE;  // dS^T: 128 keys x 128 queries, two 64-query blocks
  static constexpr int OFF_LSE = OFF_DS + TILE;       // NST x 128 floats
  static constexpr int OFF_DV = OFF_LSE + NST * 512;  // NST x 128 floats
  static constexpr int OFF_BAR = OFF_DV + NST * 512;
  static constexpr int SMEM_BYTES = OFF_BAR + 256;
  static constexpr uint32_t COL_DV = 0, COL_DK = 128, COL_S = 256, COL_DP = 384;
  static constexpr int NTHREADS = 512;
  static constexpr int LAUNCH_REGS = 128, GRAD_REGS = 136, DRAIN_REGS = 152, OTHER_REGS = 88;
  // exponentials of P on the FMA pipe (exp2_fma2) for EXP_POLY of every 8 query
  // pairs.  Measured on the training workload (step TFLOP/s): 0 -> 813, 1 -> 818,
  // 2 -> 816, 3 -> 817.
  static constexpr int EXP_POLY = 1;
  static_assert(2 * 128 * GRAD_REGS + 128 * DRAIN_REGS + 128 * OTHER_REGS <= NTHREADS * LAUNCH_REGS,
                "register split");
  static_assert(2 * GRAD_REGS + DRAIN_REGS + OTHER_REGS <= 512, "registers per sub-partition");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__global__ void __launch_bounds__(512, 1)
    fa_bwd_main_q128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                            const BwdArgs a) {
  using C = BwdQ128Cfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars + 0;
  uint64_t* bar_ld_full = bars + 1;   // [NST]
  uint64_t* bar_ld_empty = bars + 3;  // [NST]
  uint64_t* bar_s_full = bars + 5;
  uint64_t* bar_dp_full = bars + 6;
  uint64_t* bar_p_ready = bars + 7;   // 256 arrivals: P^T stored, S^T read
  uint64_t* bar_ds_ready = bars + 8;  // 256 arrivals: dS^T stored (tensor and shared memory)
  uint64_t* bar_dq_full = bars + 9;   // dQ^T(t) complete (also: shared dS^T read)
  uint64_t* bar_dp_init = bars + 10;  // 128 arrivals: dQ^T(t-1) read out, -D(t) in the dP^T columns
  uint64_t* bar_s_free = bars + 15;   // dV(t) complete: the S^T columns may be refilled
  uint64_t* bar_s_init = bars + 16;   // 128 arrivals: -LSE(t) / scale in the S^T columns
  uint64_t* bar_acc = bars + 11;
  uint64_t* bar_done = bars + 12;
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_sh = reinterpret_cast<volatile int*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  const int bh_kv = blockIdx.x % a.BHkv;  // key/value head
  const int j = blockIdx.x / a.BHkv;      // key tile; j = 0 (the longest walk when causal) first
  const int i0 = a.causal ? j : 0;        // first query tile of 128
  const int spq = a.n_tiles - i0;         // query tiles per query head
  const int steps = spq * a.group;        // the walk covers every query head of the group
  auto step_head = [&](int t) { return bh_kv * a.group + t / spq; };
  auto step_tile = [&](int t) { return i0 + t % spq; };

  // the swizzled TMA/UMMA layouts need a 1024-byte aligned base (uniform: every
  // thread returns before any barrier)
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&g_fa_status, 0, 4 /*FA_ERR_CUDA*/ | (97 << 8));
    return;
  }
  if (warp == 13) {
    tmem_alloc(tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    *abort_sh = 0;
    mbar_init(bar_kv, 1);
    for (int b = 0; b < C::NST; ++b) {
      mbar_init(bar_ld_full + b, 1);
      mbar_init(bar_ld_empty + b, 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_p_ready, 256);
    mbar_init(bar_ds_ready, 256);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dp_init, 128);
    mbar_init(bar_s_free, 1);
    mbar_init(bar_s_init, 128);
    mbar_init(bar_acc, 1);
    mbar_init(bar_done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sh;

  if (warp >= 12) {
    setmaxnreg_to<C::LAUNCH_REGS, C::OTHER_REGS>();
    if (warp == 12 && lane == 0) {
      // ============================ producer ===================================
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar_kv, 2 * C::TILE);
      for (int b = 0; b < 2; ++b) {
        tma_load_3d(smem + C::OFF_K + b * C::BOX, &tmK, bar_kv, b * 64, j * 128, bh_kv);
        tma_load_3d(smem + C::OFF_V + b * C::BOX, &tmV, bar_kv, b * 64, j * 128, bh_kv);
      }
      int t = 0;
      for (; t < steps; ++t) {
        const int i = step_tile(t), hq = step_head(t);
        const int s = t % C::NST;
        const uint32_t ph = (t / C::NST) & 1;
        if (!mbar_wait_inl(bar_ld_empty + s, ph ^ 1, abort_sh, 80)) break;
        mbar_arrive_expect_tx(bar_ld_full + s, 2 * C::TILE + 1024);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(smem + C::OFF_Q + s * C::TILE + b * C::BOX, &tmQ, bar_ld_full + s, b * 64, i * 128, hq);
          tma_load_3d(smem + C::OFF_DO + s * C::TILE + b * C::BOX, &tmDO, bar_ld_full + s, b * 64, i * 128, hq);
        }
        const size_t roff = static_cast<size_t>(hq) * a.Npad + static_cast<size_t>(i) * 128;
        bulk_load(smem + C::OFF_LSE + s * 512, a.lse2 + roff, 512, bar_ld_full + s);
        bulk_load(smem + C::OFF_DV + s * 512, a.dvec + roff, 512, bar_ld_full + s);
      }
      mbar_wait_drain(bar_kv, 0, 100000000ull);
      for (int u = max(0, t - C::NST); u < t; ++u)
        mbar_wait_drain(bar_ld_full + u % C::NST, (u / C::NST) & 1, 100000000ull);
    } else if (warp == 13 && lane == 0) {
      // ============================ MMA issuer =================================
      constexpr uint32_t id_s = make_idesc(128, 128, kFmtBF16, 0, 0);  // S^T, dP^T: N = 128 queries
      constexpr uint32_t id_g = make_idesc(128, 128, kFmtBF16, 0, 1);  // dV, dK: B MN-major (d contiguous)
      constexpr uint32_t id_q = make_idesc(128, 128, kFmtBF16, 1, 1);  // dQ^T: A = K^T, B = dS^T, MN-major
      const uint32_t k_addr = smem_u32(smem + C::OFF_K), v_addr = smem_u32(smem + C::OFF_V);
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q), do_addr = smem_u32(smem + C::OFF_DO);
      const uint32_t ds_addr = smem_u32(smem + C::OFF_DS);
      // base descriptors, built once; each MMA adds its K-step's byte offset
      const uint64_t kd_k = make_sdesc_sw128(k_addr, 16, 1024);        // K, K-major (S^T)
      const uint64_t vd_k = make_sdesc_sw128(v_addr, 16, 1024);        // V, K-major (dP^T)
      const uint64_t kd_mn = make_sdesc_sw128(k_addr, C::BOX, 1024);   // K^T, MN-major (dQ^T)
      const uint64_t dsd_mn = make_sdesc_sw128(ds_addr, C::BOX, 1024); // dS^T, MN-major (dQ^T)
      bool ok = mbar_wait_inl(bar_kv, 0, abort_sh, 81);
      for (int t = 0; ok && t < steps; ++t) {
        const int st = t % C::NST;
        const uint32_t ph = t & 1;
        if (!(ok = mbar_wait_inl(bar_ld_full + st, (t / C::NST) & 1, abort_sh, 82))) break;
        tc_fence_after();
        const uint32_t qa = q_addr + st * C::TILE, da = do_addr + st * C::TILE;
        const uint64_t qd_k = make_sdesc_sw128(qa, 16, 1024), dod_k = make_sdesc_sw128(da, 16, 1024);
        const uint64_t qd_mn = make_sdesc_sw128(qa, C::BOX, 1024), dod_mn = make_sdesc_sw128(da, C::BOX, 1024);
        // S^T = -LSE/scale + K_j Q_i^T (M = 128 keys, N = 128 queries, K = d), onto
        // the drain warps' fill of the columns that dV(t-1) read last
        if (!(ok = mbar_wait_inl(bar_s_init, ph, abort_sh, 91))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::COL_S, sdesc_add(kd_k, off), sdesc_add(qd_k, off), id_s, 1u);
        }
        mma_commit(bar_s_full);
        // dP^T = -D + V_j dO_i^T, onto the fill that replaced dQ^T(t-1)
        if (!(ok = mbar_wait_inl(bar_dp_init, ph, abort_sh, 83))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k >> 2) * C::BOX + (k & 3) * 32;
          mma_ss(tmem + C::COL_DP, sdesc_add(vd_k, off), sdesc_add(dod_k, off), id_s, 1u);
        }
        mma_commit(bar_dp_full);
        // dV += P^T dO_i (M = 128 keys, N = 128 columns, K = 128 queries): P^T in
        // tensor memory, each 64-query half packed in the first 32 of its 64 columns
        if (!(ok = mbar_wait_inl(bar_p_ready, ph, abort_sh, 84))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tmem + C::COL_DV, tmem + C::COL_S + 64 * (k >> 2) + 8 * (k & 3), sdesc_add(dod_mn, k * 2048), id_g,
                 (t > 0 || k > 0) ? 1u : 0u);
        mma_commit(bar_s_free);  // P^T read: the S^T columns may be refilled
        // dK += dS^T Q_i (dS^T likewise over dP^T)
        if (!(ok = mbar_wait_inl(bar_ds_ready, ph, abort_sh, 85))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tmem + C::COL_DK, tmem + C::COL_DP + 64 * (k >> 2) + 8 * (k & 3), sdesc_add(qd_mn, k * 2048), id_g,
                 (t > 0 || k > 0) ? 1u : 0u);
        mma_commit(bar_ld_empty + st);  // Q_i, dO_i, LSE_i, D_i read by everything that needs them
        // dQ_i^T = K_j^T dS^T (M = 128 columns, N = 128 queries, K = 128 keys) into
        // the dP^T columns, after dK has read dS^T there
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + C::COL_DP, sdesc_add(kd_mn, k * 2048), sdesc_add(dsd_mn, k * 2048), id_q, k > 0 ? 1u : 0u);
        mma_commit(bar_dq_full);
      }
      if (ok) mma_commit(bar_acc);
      mma_commit(bar_done);
      mbar_wait_drain(bar_done, 0, 100000000ull);
    }
    tc_fence_before();
    named_bar_sync_all(1, C::NTHREADS);
    if (warp == 13) {
      __syncwarp();  // lane 0 issued the MMAs alone: reconverge for the warp-wide dealloc
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  } else if (warp >= 8) {
    setmaxnreg_to<C::LAUNCH_REGS, C::DRAIN_REGS>();
    // ============================ dQ drain and accumulator set-up ===========
    // Per step t: fill the S^T columns with -LSE(t)/scale once dV(t-1) has read
    // P^T there; read dQ^T(t-1) out of the dP^T columns (thread = head-dimension
    // column c, one value per query), fill them with -D(t), release them, and
    // only then add dQ^T(t-1) into the accumulator (the reductions queue behind
    // nothing that the next MMAs wait for).
    const int c = threadIdx.x - 256;  // TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float neg_inv_c = -1.0f / a.scale_log2;  // -LSE log2(e) / (scale log2(e)) = -LSE / scale
    bool ok = true;
    for (int t = 0; t <= steps && ok; ++t) {
      const bool fill = t < steps;
      const int st = t % C::NST;
      if (fill) {
        // -LSE(t)/scale into the S^T columns once dV(t-1) has read P^T(t-1)
        if (!(ok = mbar_wait_inl(bar_ld_full + st, (t / C::NST) & 1, abort_sh, 92))) break;
        if (t >= 1 && !(ok = mbar_wait_inl(bar_s_free, (t - 1) & 1, abort_sh, 93))) break;
        tc_fence_after();
        const float4* l4p = reinterpret_cast<const float4*>(smem + C::OFF_LSE + st * 512);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {  // 16 columns (queries) per store
          uint32_t w[16];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 l4 = l4p[4 * ch + e4];
            w[4 * e4 + 0] = __float_as_uint(l4.x * neg_inv_c);
            w[4 * e4 + 1] = __float_as_uint(l4.y * neg_inv_c);
            w[4 * e4 + 2] = __float_as_uint(l4.z * neg_inv_c);
            w[4 * e4 + 3] = __float_as_uint(l4.w * neg_inv_c);
          }
          tmem_st16(tmem + lane_base + C::COL_S + 16 * ch, w);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_s_init);
      }
      uint32_t v[128];
      if (t >= 1) {
        if (!(ok = mbar_wait_inl(bar_dq_full, (t - 1) & 1, abort_sh, 86))) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          tmem_ld32(tmem + lane_base + C::COL_DP + 32 * ch, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * ch]));
        tmem_wait_ld();
      }
      if (fill) {
        const float4* d4p = reinterpret_cast<const float4*>(smem + C::OFF_DV + st * 512);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t w[16];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 d4 = d4p[4 * ch + e4];
            w[4 * e4 + 0] = __float_as_uint(-d4.x);
            w[4 * e4 + 1] = __float_as_uint(-d4.y);
            w[4 * e4 + 2] = __float_as_uint(-d4.z);
            w[4 * e4 + 3] = __float_as_uint(-d4.w);
          }
          tmem_st16(tmem + lane_base + C::COL_DP + 16 * ch, w);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      if (fill) mbar_arrive(bar_dp_init);
      if (t >= 1) {
        const int i = step_tile(t - 1), hq = step_head(t - 1);
        // lane pairs (c even, c + 1): the even lane adds columns c, c + 1 of the
        // even queries, the odd lane those of the odd queries, 8 bytes at a time
        // (half the reduction instructions of one 4-byte add per query; training
        // step 817 -> 833 TFLOP/s)
        const int c0 = c & ~1;
        float* dst = a.dq_acc + (static_cast<size_t>(hq) * a.Npad + static_cast<size_t>(i) * 128) * C::D + c0;
        const bool odd = (c & 1) != 0;
#pragma unroll
        for (int q2 = 0; q2 < 64; ++q2) {
          const float give = __uint_as_float(odd ? v[2 * q2] : v[2 * q2 + 1]);
          const float got = __shfl_xor_sync(0xffffffffu, give, 1);
          const int q = 2 * q2 + (odd ? 1 : 0);
          const float mine = __uint_as_float(odd ? v[2 * q2 + 1] : v[2 * q2]);
          const float lo = odd ? got : mine, hi = odd ? mine : got;
          red_add_v2(dst + static_cast<size_t>(q) * C::D, lo, hi);
        }
      }
    }
    tc_fence_before();
    named_bar_sync_all(1, C::NTHREADS);
  } else {
    setmaxnreg_to<C::LAUNCH_REGS, C::GRAD_REGS>();
    // ============================ gradient warps =============================
    const int half = warp >> 2;       // queries [64 half, 64 half + 64) of each step
    const int r = threadIdx.x & 127;  // key row in tile == TMEM lane
    const int key = j * 128 + r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float cl = a.scale_log2;
    bool ok = true;
    for (int t = 0; t < steps && ok; ++t) {
      const int i = step_tile(t);
      const uint32_t ph = t & 1;
      const int q0 = i * 128 + half * 64;
      const bool need_mask = (a.causal && q0 < j * 128 + 128) || key >= N;
      // ---- P = exp2(scale log2(e) (S^T - LSE / scale)) for 64 queries; P^T to TMEM
      if (!(ok = mbar_wait_inl(bar_s_full, ph, abort_sh, 87))) break;
      tc_fence_after();
      float p[64];
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        float* ps = p + 32 * sub;
        tmem_ld32(tmem + lane_base + C::COL_S + 64 * half + 32 * sub, *reinterpret_cast<uint32_t(*)[32]>(ps));
        tmem_wait_ld();
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const float2 x = fmul2(make_float2(ps[2 * e2], ps[2 * e2 + 1]), make_float2(cl, cl));
          if ((e2 & 7) < C::EXP_POLY) {
            const float2 pp = exp2_fma2(x);
            ps[2 * e2] = pp.x;
            ps[2 * e2 + 1] = pp.y;
          } else {
            ps[2 * e2] = ex2_approx(x.x);
            ps[2 * e2 + 1] = ex2_approx(x.y);
          }
        }
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (key >= N || (a.causal && key > q0 + 32 * sub + e)) ps[e] = 0.f;
        }
        // P^T (bf16, two per column) into columns 16 sub .. 16 sub + 15 of this
        // half: their fp32 scores have been read already
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pw[e] = pack_bf16x2(ps[2 * e], ps[2 * e + 1]);
        tmem_st16(tmem + lane_base + C::COL_S + 64 * half + 16 * sub, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_ready);
      // ---- dS / scale = P (dP - D); dS^T to TMEM (A of dK) and shared memory (B of dQ^T)
      if (!(ok = mbar_wait_inl(bar_dp_full, ph, abort_sh, 88))) break;
      tc_fence_after();
      // the shared dS^T buffer was last read by dQ(t-1)
      if (t >= 1 && !(ok = mbar_wait_inl(bar_dq_full, ph ^ 1, abort_sh, 89))) break;
      uint8_t* db = smem + C::OFF_DS + half * C::BOX;  // this half's 64-query block
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        uint32_t dp[32];
        tmem_ld32(tmem + lane_base + C::COL_DP + 64 * half + 32 * sub, dp);
        tmem_wait_ld();
        uint32_t dw[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {  // the dP^T accumulator started from -D
          const float* ps = p + 32 * sub + 2 * e2;
          const float2 g = fmul2(make_float2(ps[0], ps[1]),
                                 make_float2(__uint_as_float(dp[2 * e2]), __uint_as_float(dp[2 * e2 + 1])));
          dw[e2] = pack_bf16x2(g.x, g.y);
        }
        tmem_st16(tmem + lane_base + C::COL_DP + 64 * half + 16 * sub, dw);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {  // 16-byte chunk 4 sub + cc (8 queries) of row r
          const uint32_t off = sw128_off(r, 4 * sub + cc);
          *reinterpret_cast<uint4*>(db + off) = make_uint4(dw[4 * cc], dw[4 * cc + 1], dw[4 * cc + 2], dw[4 * cc + 3]);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(bar_ds_ready);
    }
    // ---- epilogue: dV (warps 0-3) and dK (warps 4-7) -> bf16 -------------------
    if (ok) ok = mbar_wait_inl(bar_acc, 0, abort_sh, 90);
    if (ok) {
      tc_fence_after();
      const uint32_t col = half ? C::COL_DK : C::COL_DV;
      const float f = half ? a.scale : 1.0f;  // dK = scale dS^T Q: the MMAs used dS / scale
      __nv_bfloat16* dst = (half ? a.dk : a.dv) + (static_cast<size_t>(bh_kv) * N + key) * C::D;
#pragma unroll
      for (int ch = 0; ch < C::D / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + col + ch * 32, v);
        tmem_wait_ld();
        if (key < N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(
                pack_bf16x2(__uint_as_float(v[8 * v4 + 0]) * f, __uint_as_float(v[8 * v4 + 1]) * f),
                pack_bf16x2(__uint_as_float(v[8 * v4 + 2]) * f, __uint_as_float(v[8 * v4 + 3]) * f),
                pack_bf16x2(__uint_as_float(v[8 * v4 + 4]) * f, __uint_as_float(v[8 * v4 + 5]) * f),
                pack_bf16x2(__uint_as_float(v[8 * v4 + 6]) * f, __uint_as_float(v[8 * v4 + 7]) * f));
        }
      }
    }
    tc_fence_before();
    named_bar_sync_all(1, C::NTHREADS);
  }
}

}  // namespace fa
