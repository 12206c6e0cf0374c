// bwd256.cuh — bwd_main at head dim 256 on CTA pairs ("FlashAttention (IT)",
// section "FlashAttention-2 (2023)": heads up to 256 wide; the backward of
// "flash-attention-trading-models", "Pase hacia atrás": the score tiles are
// recomputed from the saved logsumexp).
//
// At d = 256 the fp32 dK and dV of one 128-key tile take all 512 tensor-memory
// columns, so one CTA cannot hold both next to the score tiles.  Two CTAs of a
// cluster share the key tile and split the work by role instead of recomputing
// the contractions over d in both:
//   rank 0 (scores):   S^T = K Q_i^T, P^T = exp(S^T - LSE) -> sent to rank 1;
//                      dK += dS^T Q_i and dQ_i[:, 0:128] = dS K[:, 0:128]
//                      with dS^T received from rank 1.
//   rank 1 (gradient): dP^T = V dO_i^T; with P^T received from rank 0,
//                      dS^T = P^T (dP^T - D) * scale -> sent to rank 0;
//                      dV += P^T dO_i and dQ_i[:, 128:256] = dS K[:, 128:256].
// Each rank issues 10.5 MFLOP of MMAs per 64-query step, where one CTA per
// 128-column slice recomputing S^T and dP^T issues 14.7.  The exchanged tiles
// (128 keys x 64 queries bf16, 16 KB each way per step) are written by the
// gradient warps into a local buffer and move into the peer's buffer by
// shared-to-shared bulk copies, counted in bytes on the peer's barriers: one
// 4 KB copy per 32 key rows, issued as soon as the two warps that own those
// rows have written them, and awaited on the other side by the two warps that
// own the same rows (measured: one 16 KB copy took about 3,200 cycles from
// issue to arrival; with 16-byte remote stores instead, the storing threads
// stalled 2,000-4,800 cycles on the fence and arrival that publish them).  The consumer returns the buffer with a
// tensor-core commit that arrives on the sender's barrier (tcgen05.commit to
// the peer: a signal, no data).
//
// Both ranks have the same shared-memory layout (region contents by rank):
//   A   64 KB  K (rank 0) / V (rank 1), resident, 4 swizzled 128 x 64 boxes
//   K1  32 KB  rank 1: K[:, 128:256], resident (the A side of its dQ slice)
//   X   2 x 32 KB stages: dO_i (rank 1), 64 rows x 256 columns; rank 0 keeps
//       Q_i in three stages that start at K1 (it has no K1 of its own)
//   P   2 x 16 KB  P^T written and sent (rank 0) / received (rank 1)
//   DS  2 x 16 KB  dS^T received (rank 0) / written and sent (rank 1)
//   ROW 3 x 256 B  LSE * log2(e) (rank 0) / D (rank 1) of the step's 64 queries,
//       one per load stage
// Tensor memory (each rank): dK or dV [0, 256), S^T or dP^T buffers at 256 and
// 320, dQ^T slice buffers at 384 and 448 (64 columns each).  The dQ^T slices
// have columns of their own so that S^T(t+2) / dP^T(t+2) wait only for the
// gradient warps to have read step t, not for step t's exchange to return.
// Two threads issue MMAs: the front issuer (S^T or dP^T of step t, which need
// only a loaded stage and a drained buffer) and the back issuer (dK or dV and
// the dQ^T slice of step u, which wait on the peer).  With one issuer in program
// order, the next step's load would hold up the exchange of the current one.
#pragma once
#include "bwd.cuh"

namespace fa {

struct BwdPairCfg {
  static constexpr int DK = 256;
  static constexpr int KV_BOX = 16384;       // 128 rows x 64 columns bf16, 128-byte swizzle
  static constexpr int Q_BOX = 8192;         // 64 rows x 64 columns
  static constexpr int X_TILE = 4 * Q_BOX;   // 64 rows x 256 columns
  static constexpr int OP_TILE = 16384;      // 128 keys x 64 queries bf16 (one swizzled block)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_K1 = OFF_A + 4 * KV_BOX;
  static constexpr int OFF_X = OFF_K1 + 2 * KV_BOX;
  static constexpr int OFF_P = OFF_X + 2 * X_TILE;
  static constexpr int OFF_DS = OFF_P + 2 * OP_TILE;
  static constexpr int OFF_ROW = OFF_DS + 2 * OP_TILE;
  static constexpr int OFF_BAR = OFF_ROW + 3 * 256;
  static constexpr int SMEM_BYTES = OFF_BAR + 512;
  static constexpr uint32_t COL_G = 0, COL_S = 256, COL_Q = 384;  // dK / dV; S^T / dP^T and dQ^T buffer b at +64 b
  static constexpr int NTHREADS = 480;
  static constexpr int QUARTER = OP_TILE / 4;  // 32 key rows of an exchanged tile
  // load stages of Q (rank 0, from OFF_K1) and dO (rank 1, from OFF_X)
  static constexpr int NST0 = 3, NST1 = 2;
  static_assert(OFF_K1 + NST0 * X_TILE == OFF_P && OFF_X + NST1 * X_TILE == OFF_P, "stage regions");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// grid.x = 2 x (128-key tiles) x (batch * key/value heads), clusters of 2
// along x: the two CTAs of a cluster take the same key tile.
// Warps 0-7 gradient (2 per TMEM lane quarter: key row x query half), 8-11 dQ
// drain, 12 producer, 13 front MMA issuer, 14 back MMA issuer.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(480, 1)
    fa_bwd_main_pair256_kernel(const __grid_constant__ CUtensorMap tmQ64, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO64,
                               const BwdArgs a) {
  using C = BwdPairCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars + 0;
  uint64_t* bar_ld_full = bars + 1;     // [3] X stage loaded
  uint64_t* bar_ld_empty = bars + 4;    // [3] X stage read by both issuers' MMAs (2 arrivals)
  uint64_t* bar_mma_full = bars + 7;    // [2] S^T / dP^T of the step in TMEM
  uint64_t* bar_xchg_free = bars + 9;   // [2] the peer has consumed the tile this rank sent from buffer b
  uint64_t* bar_local_free = bars + 11; // [2] rank 1: dQ^T has read dS^T buffer b
  uint64_t* bar_dq_full = bars + 13;    // [2]
  uint64_t* bar_dq_free = bars + 15;    // [2] (128 arrivals)
  uint64_t* bar_acc = bars + 17;
  uint64_t* bar_done = bars + 18;       // both issuers' MMAs complete (2 arrivals)
  uint64_t* bar_xchg_full = bars + 19;  // [2][4] rows 32q.. of the peer's tile arrived (dS^T on rank 0, P^T on rank 1)
  uint64_t* bar_ready = bars + 27;      // [2][4] rows 32q.. of the tile to send are written (64 arrivals)
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(bars + 35);
  volatile int* abort_sh = reinterpret_cast<volatile int*>(bars + 36);

  const uint32_t rank = cluster_ctarank();  // 0: scores side, 1: gradient side
  const uint32_t peer = rank ^ 1u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N;
  const int pair = blockIdx.x >> 1;
  const int bh_kv = pair % a.BHkv;        // key/value head
  const int j = pair / a.BHkv;            // key tile of 128
  const int n_q = (N + 63) >> 6;          // query tiles of 64
  const int i0 = a.causal ? 2 * j : 0;
  const int spq = n_q - i0;               // query tiles per query head (>= 1)
  const int steps = spq * a.group;        // the walk covers every query head of the group
  auto step_head = [&](int t) { return bh_kv * a.group + t / spq; };
  auto step_tile = [&](int t) { return i0 + t % spq; };
  const int nst = rank == 0 ? C::NST0 : C::NST1;
  uint8_t* const xbase = smem + (rank == 0 ? C::OFF_K1 : C::OFF_X);

  // both CTAs of the pair see the same layout, so both leave here or neither
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
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar_ld_full + s, 1);
      mbar_init(bar_ld_empty + s, 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_mma_full + b, 1);
      for (int q = 0; q < 4; ++q) {
        mbar_init(bar_xchg_full + 4 * b + q, 1);
        mbar_init(bar_ready + 4 * b + q, 64);
      }
      mbar_init(bar_xchg_free + b, 1);
      mbar_init(bar_local_free + b, 1);
      mbar_init(bar_dq_full + b, 1);
      mbar_init(bar_dq_free + b, 128);
    }
    mbar_init(bar_acc, 1);
    mbar_init(bar_done, 2);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  // the peer's barriers exist before any arrival, copy or commit reaches them
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sh;

  if (warp == 12) {
    // ============================ producer ===================================
    if (lane == 0) {
      const CUtensorMap* m_a = rank == 0 ? &tmK : &tmV;
      const CUtensorMap* m_x = rank == 0 ? &tmQ64 : &tmDO64;
      const float* rowsrc = rank == 0 ? a.lse2 : a.dvec;
      tma_prefetch_desc(m_a);
      tma_prefetch_desc(m_x);
      mbar_arrive_expect_tx(bar_kv, (rank == 0 ? 4 : 6) * C::KV_BOX);
      for (int b = 0; b < 4; ++b) tma_load_3d(smem + C::OFF_A + b * C::KV_BOX, m_a, bar_kv, b * 64, j * 128, bh_kv);
      if (rank == 1)
        for (int b = 0; b < 2; ++b)
          tma_load_3d(smem + C::OFF_K1 + b * C::KV_BOX, &tmK, bar_kv, (2 + b) * 64, j * 128, bh_kv);
      int t = 0;
      for (; t < steps; ++t) {
        const int i = step_tile(t), hq = step_head(t);
        const int s = t % nst;
        if (!mbar_wait(bar_ld_empty + s, ((t / nst) & 1) ^ 1, abort_sh, 120)) break;
        mbar_arrive_expect_tx(bar_ld_full + s, C::X_TILE + 256);
        for (int b = 0; b < 4; ++b)
          tma_load_3d(xbase + s * C::X_TILE + b * C::Q_BOX, m_x, bar_ld_full + s, b * 64, i * 64, hq);
        bulk_load(smem + C::OFF_ROW + s * 256, rowsrc + static_cast<size_t>(hq) * a.Npad + static_cast<size_t>(i) * 64,
                  256, bar_ld_full + s);
      }
      mbar_wait_drain(bar_kv, 0, 100000000ull);
      for (int u = max(0, t - nst); u < t; ++u) mbar_wait_drain(bar_ld_full + u % nst, (u / nst) & 1, 100000000ull);
    }
  } else if (warp == 13 || warp == 14) {
    // ============================ MMA issuers ================================
    constexpr uint32_t id_s = make_idesc(128, 64, kFmtBF16, 0, 0);   // S^T, dP^T: N = 64 queries, K = 256
    constexpr uint32_t id_g = make_idesc(128, 256, kFmtBF16, 0, 1);  // dK, dV: N = 256 columns, K = 64 queries
    constexpr uint32_t id_q = make_idesc(128, 64, kFmtBF16, 1, 1);   // dQ^T slice: A = K^T, B = dS^T, MN-major
    const uint32_t a_addr = smem_u32(smem + C::OFF_A), x_addr = smem_u32(xbase);
    if (warp == 13 && lane == 0) {
      // ---- front: S^T(t) = K Q_t^T (rank 0) or dP^T(t) = V dO_t^T (rank 1) ----
      bool ok = mbar_wait(bar_kv, 0, abort_sh, 121);
      for (int t = 0; ok && t < steps; ++t) {
        const int b = t & 1, s = t % nst;
        if (!(ok = mbar_wait(bar_ld_full + s, (t / nst) & 1, abort_sh, 122))) break;
        // the buffer held step t-2, which the gradient warps have read once all
        // four row quarters of it are marked written
        for (int q = 0; t >= 2 && q < 4 && ok; ++q) ok = mbar_wait(bar_ready + 4 * b + q, ((t >> 1) & 1) ^ 1, abort_sh, 123);
        if (!ok) break;
        tc_fence_after();
        // M = 128 keys, N = 64 queries, K = 256
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t aa = a_addr + (k >> 2) * C::KV_BOX + (k & 3) * 32;
          const uint32_t xb = x_addr + s * C::X_TILE + (k >> 2) * C::Q_BOX + (k & 3) * 32;
          mma_ss(tmem + C::COL_S + 64 * b, make_sdesc_sw128(aa, 16, 1024), make_sdesc_sw128(xb, 16, 1024), id_s,
                 k > 0);
        }
        mma_commit(bar_mma_full + b);
        mma_commit(bar_ld_empty + s);  // one of the stage's two readers
      }
      mma_commit(bar_done);
      mbar_wait_drain(bar_done, 0, 100000000ull);
    } else if (warp == 14 && lane == 0) {
      // ---- back: dK or dV and the dQ^T slice of step u, after the exchange ----
      const uint32_t p_addr = smem_u32(smem + C::OFF_P), ds_addr = smem_u32(smem + C::OFF_DS);
      // K columns of this rank's dQ slice: K[:, 0:128] (boxes 0, 1 of A) or K1
      const uint32_t kq_addr = rank == 0 ? a_addr : smem_u32(smem + C::OFF_K1);
      const uint16_t peer_mask = static_cast<uint16_t>(1u << peer);
      bool ok = mbar_wait(bar_kv, 0, abort_sh, 124);
      for (int u = 0; ok && u < steps; ++u) {
        const int ub = u & 1, su = u % nst;
        const uint32_t uph = (u >> 1) & 1;
        const uint32_t xu = x_addr + su * C::X_TILE;
        const uint32_t dsu = ds_addr + ub * C::OP_TILE;
        if (rank == 0) {
          // dS^T(u) from the peer
          for (int q = 0; q < 4 && ok; ++q) ok = mbar_wait_cluster(bar_xchg_full + 4 * ub + q, uph, abort_sh, 126);
          if (!ok) break;
          tc_fence_after();
          // dK += dS^T Q_u   (A = dS^T, 128 keys x 64 queries K-major; B = Q_u MN-major, N = 256)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss(tmem + C::COL_G, make_sdesc_sw128(dsu + k * 32, 16, 1024),
                   make_sdesc_sw128(xu + k * 2048, C::Q_BOX, 1024), id_g, (u > 0 || k > 0) ? 1u : 0u);
          mma_commit(bar_ld_empty + su);  // the stage's other reader
          // dQ_u[:, 0:128]^T = K[:, 0:128]^T dS^T   (M = 128 columns, N = 64 queries, K = 128 keys),
          // once the drain warps have emptied the buffer of dQ^T(u-2)
          if (u >= 2 && !(ok = mbar_wait(bar_dq_free + ub, uph ^ 1, abort_sh, 137))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tmem + C::COL_Q + 64 * ub, make_sdesc_sw128(kq_addr + k * 2048, C::KV_BOX, 1024),
                   make_sdesc_sw128(dsu + k * 2048, C::KV_BOX, 1024), id_q, k > 0 ? 1u : 0u);
          mma_commit(bar_dq_full + ub);
          mma_commit_cluster(bar_xchg_free + ub, peer_mask);  // dS^T(u) consumed
        } else {
          // P^T(u) from the peer
          for (int q = 0; q < 4 && ok; ++q) ok = mbar_wait_cluster(bar_xchg_full + 4 * ub + q, uph, abort_sh, 127);
          if (!ok) break;
          tc_fence_after();
          const uint32_t pu = p_addr + ub * C::OP_TILE;
          // dV += P^T dO_u   (A = P^T K-major, B = dO_u MN-major, N = 256)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss(tmem + C::COL_G, make_sdesc_sw128(pu + k * 32, 16, 1024),
                   make_sdesc_sw128(xu + k * 2048, C::Q_BOX, 1024), id_g, (u > 0 || k > 0) ? 1u : 0u);
          for (int q = 0; q < 4 && ok; ++q) ok = mbar_wait(bar_ready + 4 * ub + q, uph, abort_sh, 128);
          if (!ok) break;
          tc_fence_after();
          // the stage's other reader: dV(u), and the gradient warps have read D
          // from the stage's row slot
          mma_commit(bar_ld_empty + su);
          // P^T(u) consumed: by dV(u) (this commit) and by the gradient warps (bar_ready)
          mma_commit_cluster(bar_xchg_free + ub, peer_mask);
          // dQ_u[:, 128:256]^T = K[:, 128:256]^T dS^T
          if (u >= 2 && !(ok = mbar_wait(bar_dq_free + ub, uph ^ 1, abort_sh, 137))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tmem + C::COL_Q + 64 * ub, make_sdesc_sw128(kq_addr + k * 2048, C::KV_BOX, 1024),
                   make_sdesc_sw128(dsu + k * 2048, C::KV_BOX, 1024), id_q, k > 0 ? 1u : 0u);
          mma_commit(bar_dq_full + ub);
          mma_commit(bar_local_free + ub);
        }
      }
      if (ok) mma_commit(bar_acc);
      mma_commit(bar_done);
      mbar_wait_drain(bar_done, 0, 100000000ull);
    }
  } else if (warp >= 8) {
    // ============================ dQ drain ===================================
    const int c = threadIdx.x - 256;  // column of this rank's dQ slice == TMEM lane of dQ^T
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    for (int t = 0; t < steps; ++t) {
      const int b = t & 1;
      const int i = step_tile(t), hq = step_head(t);
      if (!mbar_wait(bar_dq_full + b, (t >> 1) & 1, abort_sh, 135)) break;
      tc_fence_after();
      uint32_t v[64];
      tmem_ld32(tmem + lane_base + C::COL_Q + 64 * b, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld32(tmem + lane_base + C::COL_Q + 64 * b + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar_dq_free + b);
      float* dst = a.dq_acc + (static_cast<size_t>(hq) * a.Npad + static_cast<size_t>(i) * 64) * C::DK + rank * 128 + c;
#pragma unroll
      for (int q = 0; q < 64; ++q) atomicAdd(dst + static_cast<size_t>(q) * C::DK, __uint_as_float(v[q]));
    }
  } else {
    // ============================ gradient warps =============================
    const int half = warp >> 2;       // queries [32 half, 32 half + 32) of each 64-query step
    const int r = threadIdx.x & 127;  // key row in tile == TMEM lane
    const int key = j * 128 + r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float cl = a.scale_log2;
    bool ok = true;
    for (int t = 0; t < steps && ok; ++t) {
      const int i = step_tile(t);
      const int b = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      const float4* row4 = reinterpret_cast<const float4*>(smem + C::OFF_ROW + (t % nst) * 256) + half * 8;
      if (!(ok = mbar_wait(bar_mma_full + b, ph, abort_sh, 129))) break;
      tc_fence_after();
      float x[32];
      tmem_ld32(tmem + lane_base + C::COL_S + 64 * b + half * 32, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
      tmem_wait_ld();
      uint32_t w[16];
      if (rank == 0) {
        // P = exp2(S scale log2(e) - LSE log2(e)); masked keys (causal, past N) give 0
        const int q0 = i * 64 + half * 32;
        const bool need_mask = (a.causal && q0 < j * 128 + 128) || key >= N;
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 l4 = row4[e4];
          const float2 x01 = ffma2(make_float2(x[4 * e4], x[4 * e4 + 1]), make_float2(cl, cl), make_float2(-l4.x, -l4.y));
          const float2 x23 = ffma2(make_float2(x[4 * e4 + 2], x[4 * e4 + 3]), make_float2(cl, cl),
                                   make_float2(-l4.z, -l4.w));
          x[4 * e4] = ex2_approx(x01.x);
          x[4 * e4 + 1] = ex2_approx(x01.y);
          x[4 * e4 + 2] = ex2_approx(x23.x);
          x[4 * e4 + 3] = ex2_approx(x23.y);
        }
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (key >= N || (a.causal && key > q0 + e)) x[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
        // P^T buffer b was sent at step t-2: the peer has consumed that copy
        if (t >= 2 && !(ok = mbar_wait(bar_xchg_free + b, ph ^ 1, abort_sh, 130))) break;
        uint8_t* dst = smem + C::OFF_P + b * C::OP_TILE;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          *reinterpret_cast<uint4*>(dst + sw128_off(r, half * 4 + cc)) =
              make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
        fence_proxy_async_smem();  // read by the bulk copy
        tc_fence_before();         // S^T(t) has been read: S^T(t+2) may overwrite it
      } else {
        // dS = P (dP - D) scale, with P^T from rank 0 (bf16, this row's 32 queries)
        if (!(ok = mbar_wait_cluster(bar_xchg_full + 4 * b + (warp & 3), ph, abort_sh, 131))) break;
        const uint8_t* prow = smem + C::OFF_P + b * C::OP_TILE;
        float p[32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(prow + sw128_off(r, half * 4 + cc));
          const uint32_t vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv[e]));
            p[8 * cc + 2 * e] = f.x;
            p[8 * cc + 2 * e + 1] = f.y;
          }
        }
        const float2 sc2 = make_float2(a.scale, a.scale);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 d4 = row4[e4];
          const float2 g01 = fmul2(fmul2(make_float2(p[4 * e4], p[4 * e4 + 1]),
                                         fadd2(make_float2(x[4 * e4], x[4 * e4 + 1]), make_float2(-d4.x, -d4.y))),
                                   sc2);
          const float2 g23 = fmul2(fmul2(make_float2(p[4 * e4 + 2], p[4 * e4 + 3]),
                                         fadd2(make_float2(x[4 * e4 + 2], x[4 * e4 + 3]), make_float2(-d4.z, -d4.w))),
                                   sc2);
          w[2 * e4] = pack_bf16x2(g01.x, g01.y);
          w[2 * e4 + 1] = pack_bf16x2(g23.x, g23.y);
        }
        // dS^T buffer b was sent at step t-2 and read by dQ^T(t-2)
        if (t >= 2) {
          if (!(ok = mbar_wait(bar_xchg_free + b, ph ^ 1, abort_sh, 132))) break;
          if (!(ok = mbar_wait(bar_local_free + b, ph ^ 1, abort_sh, 133))) break;
        }
        // dS^T(t): the B operand of this rank's dQ^T slice, and sent for dK
        uint8_t* dst = smem + C::OFF_DS + b * C::OP_TILE;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          *reinterpret_cast<uint4*>(dst + sw128_off(r, half * 4 + cc)) =
              make_uint4(w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
        fence_proxy_async_smem();  // read by the tensor core and the bulk copy
        tc_fence_before();         // dP^T(t) has been read: dP^T(t+2) may overwrite it
      }
      // rows 32 (warp % 4) .. + 31 of the tile (both query halves) go to the peer
      // once the two warps that own them have written them
      const int qr = warp & 3;
      mbar_arrive(bar_ready + 4 * b + qr);
      int sent = 1;
      if (warp < 4 && lane == 0) {
        sent = mbar_wait(bar_ready + 4 * b + qr, ph, abort_sh, 136);
        if (sent) {
          uint8_t* src = smem + (rank == 0 ? C::OFF_P : C::OFF_DS) + b * C::OP_TILE + qr * C::QUARTER;
          const uint32_t pbar = peer_smem(bar_xchg_full + 4 * b + qr, peer);
          mbar_arrive_expect_tx_peer(pbar, C::QUARTER);
          bulk_copy_to_peer(peer_smem(src, peer), src, C::QUARTER, pbar);
        }
      }
      // the whole warp leaves together (the loop's tensor-memory loads are warp-wide)
      if (!__shfl_sync(0xffffffffu, sent, 0)) ok = false;
    }
    // ---- epilogue: dK (rank 0) or dV (rank 1), 128 columns per query half ----
    if (ok) ok = mbar_wait(bar_acc, 0, abort_sh, 134);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dst = (rank == 0 ? a.dk : a.dv) + (static_cast<size_t>(bh_kv) * N + key) * C::DK + half * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + C::COL_G + half * 128 + ch * 32, v);
        tmem_wait_ld();
        if (key < N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            d4[v4] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * v4 + 0]), __uint_as_float(v[8 * v4 + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * v4 + 2]), __uint_as_float(v[8 * v4 + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * v4 + 4]), __uint_as_float(v[8 * v4 + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * v4 + 6]), __uint_as_float(v[8 * v4 + 7])));
        }
      }
    }
  }

  // The peer's last two returns of this rank's sent buffers are still owed
  // (earlier ones were awaited before each reuse); collect them so that no
  // arrival reaches this CTA after it has left.
  if (warp == 12 && lane == 0) {
    for (int u = max(0, steps - 2); u < steps; ++u)
      mbar_wait_drain(bar_xchg_free + (u & 1), (u >> 1) & 1, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  // neither CTA leaves while the other may still copy into it or signal it
  cluster_sync_all();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
