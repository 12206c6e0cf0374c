// fwd.cuh — exact attention forward on B200: TMA + tcgen05 + TMEM, warp-specialised.
//
// Algorithm ("flash-attention-trading-models", sections "El algoritmo de atencion
// flash" and "La recurrencia de softmax en linea"; "FlashAttention (IT)", "Tiling",
// "Calcolo online del Softmax", "Fusione delle operazioni"): split Q into row tiles
// of 128 and K, V into column tiles of 128; for each Q tile visit the K/V tiles,
// keep the running row max m and running sum l, rescale the partial O when m grows,
// never write S or P to device memory, and normalise O once at the end (the
// deferred rescale of FlashAttention-2, same page, section "FA2").
//
// One CTA owns two Q tiles (256 query rows) of one (batch, head) and runs on its
// own SM.  Warp roles (FlashAttention-3's producer/consumer split, same page,
// section "FA3", re-cast for tcgen05):
//   warps 0-3  softmax for Q tile 0   (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax for Q tile 1
//   warp  8    TMA producer: Q0, Q1 once, then K_j and V_j through a ring
//   warp  9    tcgen05.mma issuer (one thread) and TMEM owner
//   warps 10-11 no role (they complete the third warpgroup, whose registers
//              go to the softmax warpgroups)
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0,128)   S0 = Q0 K_j^T   (P0 is written over its first columns as bf16)
//   [128,256) S1 = Q1 K_j^T   (P1 likewise)
//   [256,256+D) O0, then O1   (fp32 accumulators)
// The MMA thread interleaves the two tiles so that the tensor core works on one
// tile while the softmax warps work on the other (FA3 "interleaved matmul and
// softmax"):  S0(j+1) is issued right after PV0(j), before waiting for P1(j).
// Every tcgen05.commit covers all earlier MMAs of the thread, so the arrival of
// "S_i(j) ready" also means "PV_i(j-1) done": the softmax warps may then rescale
// O_i in TMEM before handing P_i(j) back.
//
// Causal masking ("flash-attention-trading-models", section on causal masking):
// key tiles wholly in the future of a Q tile are never loaded or multiplied;
// the diagonal tile and the ragged last key tile are masked element-wise.
#pragma once
#include <type_traits>

#include "sm100.cuh"

namespace fa {

template <typename T>
struct ElemTraits;
template <>
struct ElemTraits<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr uint32_t kFmt = kFmtBF16;
};
template <>
struct ElemTraits<float> {
  static constexpr int kBytes = 4;
  static constexpr uint32_t kFmt = kFmtTF32;
};
// E4M3 codes (the full FP8 forward): kind::f8f6f4 MMAs
template <>
struct ElemTraits<uint8_t> {
  static constexpr int kBytes = 1;
  static constexpr uint32_t kFmt = kFmtE4M3;
};

struct FwdArgs {
  void* o;
  float* lse;
  int N;          // sequence length
  int BH;         // batch * heads
  int nblk;       // ceil(N / 256): CTAs per (batch, head)
  float scale_log2;  // softmax scale * log2(e)
  float p_scale;     // static scale S of the E4M3 P-cast (1 otherwise)
  int causal;
  int kv_order;      // 0: key tiles 0..T-1, 1: T-1..0
  unsigned long long* stats;
  int n_sink;
  // full FP8 operands only: dequantisation scales of the E4M3 codes
  const float* sq;  // [BH, nqb] per 128-row block of Q
  const float* sk;  // [B*H_kv, nqb] per 128-row block of K
  const float* sv;  // [BH] per head of V
  int nqb;          // ceil(N / 128)
  int group;        // query heads per key/value head (1 = multi-head attention)
};

template <typename T, int D, bool FP8P>
struct FwdCfg {
  static constexpr int EB = ElemTraits<T>::kBytes;
  // swizzled row of a TMA box: 128 bytes, or 64 for E4M3 at d = 64 (a whole row,
  // with the 64-byte swizzle)
  static constexpr int ROW_BYTES = D * EB < 128 ? D * EB : 128;
  static constexpr bool SW64 = ROW_BYTES == 64;
  static constexpr int BOX_COLS = ROW_BYTES / EB;      // elements in one swizzled row
  static constexpr int NBOX = D / BOX_COLS;            // TMA boxes across the head dim
  static constexpr int BOX_BYTES = 128 * ROW_BYTES;    // 128 rows
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;  // one 128 x D tile
  static constexpr int KSTEP = 32 / EB;                // K elements per MMA (32 bytes)
  static constexpr int KSTEPS_PER_BOX = BOX_COLS / KSTEP;
  static constexpr int NK_QK = D / KSTEP;              // MMAs for one S tile
  static constexpr int NK_PV = 128 / KSTEP;            // MMAs for one PV tile
  static constexpr int NSTAGE = (TILE_BYTES <= 16384) ? 3 : 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NSTAGE * TILE_BYTES;
  // bf16 at d = 64: P goes to shared memory and PV is a shared-memory x
  // shared-memory MMA.  With N = d = 64 an MMA reading A from tensor memory
  // takes ~151 cycles per 16-deep step against ~108 from shared memory (at
  // N = 128, d = 128, tensor memory is the faster, ~73).
  static constexpr bool PV_SS = (EB == 2) && (D == 64) && !FP8P;
  // Exponentials on the FMA pipe (exp2_fma2) for 2 of every 8 key pairs of a
  // bf16 tile at d = 64, the rest on the MUFU: there the MUFU is the busier pipe
  // (one exponential per 128 FLOP of MMA against one per 256 at d = 128).
  // Measured: 595 -> 616 TFLOP/s on the trading-day workload; 3 of 8 spill;
  // at d = 128 any share is slower.
  static constexpr int EXP_POLY = (EB == 2 && !FP8P && D == 64) ? 2 : 0;
  // E4M3 operands: the MMAs run at twice the bf16 rate, so the exponentials
  // weigh twice as much; 2 of every 8 groups of 4 keys on the FMA pipe.
  // Measured on the prefill shape: 1155 -> 1187 TFLOP/s; 3 of 8 1177, 4 of 8 1101.
  static constexpr int EXP_POLY_E4M3 = EB == 1 ? 2 : 0;
  static constexpr int P_BYTES = 128 * 128 * 2;  // one 128 x 128 bf16 P tile: two 64-key boxes
  static constexpr int OFF_P = OFF_V + NSTAGE * TILE_BYTES;
  static constexpr int SMEM_BYTES = OFF_P + (PV_SS ? 2 * P_BYTES : 0) + 1024;  // + alignment slack
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  // Three warpgroups: two softmax warpgroups and one for the producer and MMA
  // warps (two of its warps have no role).  Launched at 168 registers a thread
  // (12 warps on 4 sub-partitions), the third warpgroup gives registers back and
  // the softmax warpgroups take them: 8 x 32 x 216 + 4 x 32 x 72 = 64512 =
  // 384 x 168, and 2 x 32 x 216 + 32 x 72 = 16128 <= 16384 per sub-partition.
  static constexpr int NTHREADS = 384;
  static constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 216, OTHER_REGS = 72;
  static_assert(8 * 32 * SOFTMAX_REGS + 4 * 32 * OTHER_REGS <= NTHREADS * LAUNCH_REGS, "register split");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(COL_O1 + D <= 512, "tensor memory budget");
  static_assert(ROW_BYTES == 128 || (SW64 && EB == 1), "the 64-byte rows are E4M3 only");
};

// FP8P: P is cast to E4M3 before PV (bf16 operands); COUNT: FP8P that also
// counts the P' values that flushed to zero.
template <typename T, int D, bool FP8P, bool COUNT = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, const FwdArgs a) {
  using C = FwdCfg<T, D, FP8P>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_q, bar_kf[C::NSTAGE], bar_ke[C::NSTAGE], bar_vf[C::NSTAGE], bar_ve[C::NSTAGE];
  __shared__ uint64_t bar_s[2], bar_p[2], bar_o[2], bar_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work decode: heaviest query blocks first when causal -----------------
  const int N = a.N;
  // CTAs in flight should share K/V through L2: blocks are issued in groups of
  // kHeadGroup heads (all query blocks of the group, heaviest first when causal),
  // so the resident working set is a few heads' K/V instead of one per SM.
  constexpr int kHeadGroup = 8;
  const int group = blockIdx.x / (kHeadGroup * a.nblk);
  const int heads_in_group = min(kHeadGroup, a.BH - group * kHeadGroup);
  const int r_in_group = blockIdx.x - group * kHeadGroup * a.nblk;
  const int bh = group * kHeadGroup + r_in_group % heads_in_group;
  int qblk = r_in_group / heads_in_group;
  // grouped-query attention: query head bh reads key/value head bh / group (the
  // query heads of one key/value head are adjacent, so they run side by side and
  // share its tiles through L2)
  const int bh_kv = bh / a.group;
  if (a.causal) qblk = a.nblk - 1 - qblk;
  const int m0 = qblk * 256;
  const int n_kv = (N + 127) >> 7;
  const int qt0 = m0 >> 7;
  const bool valid0 = m0 < N, valid1 = m0 + 128 < N;
  const int kv_end0 = valid0 ? (a.causal ? min(n_kv, qt0 + 1) : n_kv) : 0;
  const int kv_end1 = valid1 ? (a.causal ? min(n_kv, qt0 + 2) : n_kv) : 0;
  const int n_steps = max(kv_end0, kv_end1);
  const int rev = a.kv_order;

  // ---- setup ---------------------------------------------------------------
  if (warp == 9) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(&bar_q, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_ke[s], 1);
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_p[i], 128);
      mbar_init(&bar_o[i], 1);
    }
    mbar_init(&bar_done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // Each warpgroup sets its register budget at the top of its own branch and the
  // branches never rejoin: each ends at its own arrival on the teardown barrier.
  if (warp >= 8) {
  setmaxnreg_dec<C::OTHER_REGS>();
  if (warp == 8) {
    // ======================= TMA producer ===================================
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if constexpr (C::EB == 2) tma_prefetch_desc(&tmO);
      mbar_arrive_expect_tx(&bar_q, (valid1 ? 2 : 1) * C::TILE_BYTES);
      for (int b = 0; b < C::NBOX; ++b) {
        tma_load_3d(smem + C::OFF_Q + b * C::BOX_BYTES, &tmQ, &bar_q, b * C::BOX_COLS, m0, bh);
        if (valid1)
          tma_load_3d(smem + C::OFF_Q + C::TILE_BYTES + b * C::BOX_BYTES, &tmQ, &bar_q, b * C::BOX_COLS, m0 + 128,
                      bh);
      }
      for (int t = 0; t < n_steps; ++t) {
        const int j = rev ? n_steps - 1 - t : t;
        const int s = t % C::NSTAGE;
        const uint32_t ph = (t / C::NSTAGE) & 1;
        if (!mbar_wait(&bar_ke[s], ph ^ 1, &abort_sh, 1)) break;
        mbar_arrive_expect_tx(&bar_kf[s], C::TILE_BYTES);
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_3d(smem + C::OFF_K + s * C::TILE_BYTES + b * C::BOX_BYTES, &tmK, &bar_kf[s], b * C::BOX_COLS,
                      j * 128, bh_kv);
        if (!mbar_wait(&bar_ve[s], ph ^ 1, &abort_sh, 2)) break;
        mbar_arrive_expect_tx(&bar_vf[s], C::TILE_BYTES);
        for (int b = 0; b < C::NBOX; ++b)
          tma_load_3d(smem + C::OFF_V + s * C::TILE_BYTES + b * C::BOX_BYTES, &tmV, &bar_vf[s], b * C::BOX_COLS,
                      j * 128, bh_kv);
      }
      // teardown: let every issued copy land before the CTA can exit
      const int first = max(0, n_steps - C::NSTAGE);
      for (int t = first; t < n_steps; ++t) {
        const int s = t % C::NSTAGE;
        const uint32_t ph = (t / C::NSTAGE) & 1;
        mbar_wait_drain(&bar_kf[s], ph, 100000000ull);
        mbar_wait_drain(&bar_vf[s], ph, 100000000ull);
      }
    }
  } else if (warp == 9) {
    // ======================= tcgen05.mma issuer =============================
    // Lane 0 alone issues MMAs and commits.  With fp32 operands the whole warp
    // follows the control flow (all lanes round the operand tiles); otherwise the
    // other lanes stay out of it: lanes spinning on the next barrier beside the
    // issuing lane measurably slow its MMA issue.
    constexpr bool kWarpWide = C::EB == 4;
    if (kWarpWide || lane == 0) {
      const bool leader = lane == 0;
      // every lane waits (each gets the acquire), then the warp agrees on the outcome
      auto warp_wait = [&](uint64_t* bar, uint32_t parity, volatile int* ab, int site) {
        if constexpr (kWarpWide)
          return __all_sync(0xffffffffu, mbar_wait(bar, parity, ab, site));
        else
          return mbar_wait(bar, parity, ab, site);
      };
      constexpr uint32_t idesc_s = make_idesc(128, 128, ElemTraits<T>::kFmt, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc(128, D, ElemTraits<T>::kFmt, 0, 1);
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
      const uint32_t k_addr = smem_u32(smem + C::OFF_K);
      const uint32_t v_addr = smem_u32(smem + C::OFF_V);
      int pv_count[2] = {0, 0};
      const int kv_end[2] = {kv_end0, kv_end1};

      auto issue_s = [&](int i, int s) {
        const uint32_t qa = q_addr + i * C::TILE_BYTES;
        const uint32_t ka = k_addr + s * C::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < C::NK_QK; ++k) {
          const uint32_t off = (k / C::KSTEPS_PER_BOX) * C::BOX_BYTES + (k % C::KSTEPS_PER_BOX) * 32;
          // K-major, 8-row groups 8 rows x ROW_BYTES apart
          const uint64_t ad = C::SW64 ? make_sdesc_sw64(qa + off, 16, 512) : make_sdesc_sw128(qa + off, 16, 1024);
          const uint64_t bd = C::SW64 ? make_sdesc_sw64(ka + off, 16, 512) : make_sdesc_sw128(ka + off, 16, 1024);
          if (!leader) continue;
          if constexpr (C::EB == 2)
            mma_ss(tmem + (i ? C::COL_S1 : C::COL_S0), ad, bd, idesc_s, k > 0);
          else if constexpr (C::EB == 1)
            mma_ss_f8(tmem + (i ? C::COL_S1 : C::COL_S0), ad, bd, idesc_s, k > 0);
          else
            mma_ss_tf32(tmem + (i ? C::COL_S1 : C::COL_S0), ad, bd, idesc_s, k > 0);
        }
        if (leader) mma_commit(&bar_s[i]);
      };
      auto issue_pv = [&](int i, int s) {
        const uint32_t va = v_addr + s * C::TILE_BYTES;
        const uint32_t pcol = tmem + (i ? C::COL_S1 : C::COL_S0);
        const uint32_t ocol = tmem + (i ? C::COL_O1 : C::COL_O0);
        const uint32_t pa = smem_u32(smem + C::OFF_P) + i * C::P_BYTES;
#pragma unroll
        for (int k = 0; k < C::NK_PV; ++k) {
          // V is the MN-major B operand: 128B swizzle (bf16, E4M3), 64B swizzle (E4M3 at
          // d = 64: N = 64 codes fill one row) or the 32-byte-atom 128B swizzle (tf32,
          // whose only MN-major layout), K rows ROW_BYTES apart.
          const uint32_t vk = va + k * C::KSTEP * C::ROW_BYTES;
          const uint64_t bd = C::EB == 4 ? make_sdesc_sw128_32b(vk, C::BOX_BYTES, 512)
                              : C::SW64  ? make_sdesc_sw64(vk, C::BOX_BYTES, 512)
                                         : make_sdesc_sw128(vk, C::BOX_BYTES, 1024);
          const uint32_t acc = (pv_count[i] > 0 || k > 0) ? 1u : 0u;
          if (!leader) continue;
          if constexpr (C::PV_SS)
            mma_ss(ocol, make_sdesc_sw128(pa + (k >> 2) * (C::P_BYTES / 2) + (k & 3) * 32, 16, 1024), bd, idesc_pv,
                   acc);
          else if constexpr (C::EB == 2)
            mma_ts(ocol, pcol + k * 8, bd, idesc_pv, acc);
          else if constexpr (C::EB == 1)
            mma_ts_f8(ocol, pcol + k * 8, bd, idesc_pv, acc);
          else
            mma_ts_tf32(ocol, pcol + k * 8, bd, idesc_pv, acc);
        }
        pv_count[i]++;
        if (leader && pv_count[i] == kv_end[i]) mma_commit(&bar_o[i]);
      };
      // fp32 inputs: the tensor core reads the top 19 bits of each operand
      // (truncation); Q and K are rounded to tf32 to nearest-even in place first,
      // so that the scores, and with them the logsumexp, carry no truncation bias.
      auto round_tile_tf32 = [&](uint32_t byte_off, int nbytes) {
        if constexpr (C::EB == 4) {
          uint4* p = reinterpret_cast<uint4*>(smem + byte_off);
          for (int idx = lane; idx < nbytes / 16; idx += 32) {
            uint4 w = p[idx];
            w.x = (w.x + 0xFFFu + ((w.x >> 13) & 1u)) & 0xFFFFE000u;
            w.y = (w.y + 0xFFFu + ((w.y >> 13) & 1u)) & 0xFFFFE000u;
            w.z = (w.z + 0xFFFu + ((w.z >> 13) & 1u)) & 0xFFFFE000u;
            w.w = (w.w + 0xFFFu + ((w.w >> 13) & 1u)) & 0xFFFFE000u;
            p[idx] = w;
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
      };

      bool ok = warp_wait(&bar_q, 0, &abort_sh, 3);
      if (ok) round_tile_tf32(C::OFF_Q, (valid1 ? 2 : 1) * C::TILE_BYTES);
      if (ok && n_steps > 0) {
        const int j0 = rev ? n_steps - 1 : 0;
        ok = warp_wait(&bar_kf[0], 0, &abort_sh, 4);
        if (ok) {
          round_tile_tf32(C::OFF_K, C::TILE_BYTES);
          tc_fence_after();
          if (j0 < kv_end0) issue_s(0, 0);
          if (j0 < kv_end1) issue_s(1, 0);
          if (leader) mma_commit(&bar_ke[0]);
        }
      }
      for (int t = 0; ok && t < n_steps; ++t) {
        const int j = rev ? n_steps - 1 - t : t;
        const int s = t % C::NSTAGE;
        const uint32_t ph = (t / C::NSTAGE) & 1;
        const bool has_next = t + 1 < n_steps;
        const int jn = rev ? n_steps - 2 - t : t + 1;
        const int sn = (t + 1) % C::NSTAGE;
        const uint32_t phn = ((t + 1) / C::NSTAGE) & 1;
        bool kn_ready = false;
        if (!(ok = warp_wait(&bar_vf[s], ph, &abort_sh, 5))) break;
        if (j < kv_end0) {
          if (!(ok = warp_wait(&bar_p[0], pv_count[0] & 1, &abort_sh, 6))) break;
          tc_fence_after();
          issue_pv(0, s);
        }
        if (has_next && jn < kv_end0) {
          if (!(ok = warp_wait(&bar_kf[sn], phn, &abort_sh, 7))) break;
          kn_ready = true;
          round_tile_tf32(C::OFF_K + sn * C::TILE_BYTES, C::TILE_BYTES);
          tc_fence_after();
          issue_s(0, sn);
        }
        if (j < kv_end1) {
          if (!(ok = warp_wait(&bar_p[1], pv_count[1] & 1, &abort_sh, 8))) break;
          tc_fence_after();
          issue_pv(1, s);
        }
        if (leader) mma_commit(&bar_ve[s]);
        if (has_next) {
          if (jn < kv_end1) {
            if (!kn_ready) {
              if (!(ok = warp_wait(&bar_kf[sn], phn, &abort_sh, 9))) break;
              round_tile_tf32(C::OFF_K + sn * C::TILE_BYTES, C::TILE_BYTES);
              tc_fence_after();
            }
            issue_s(1, sn);
          }
          if (leader) mma_commit(&bar_ke[sn]);
        }
      }
      // teardown: every MMA of this thread must be finished before TMEM is freed
      if (leader) {
        mma_commit(&bar_done);
        mbar_wait_drain(&bar_done, 0, 100000000ull);
      }
      if constexpr (kWarpWide) __syncwarp();
    }
  }
  // teardown of the third warpgroup: once every warp has arrived, no MMA or TMEM
  // access is in flight and warp 9 frees the tensor memory
  tc_fence_before();
  named_bar_sync_all(1, C::NTHREADS);
  if (warp == 9) {
    __syncwarp();  // reconverge after the barrier for the warp-wide dealloc
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  } else {
    setmaxnreg_inc<C::SOFTMAX_REGS>();
    // ======================= softmax warpgroups =============================
    const int i = warp >> 2;                       // Q tile
    const int r = threadIdx.x & 127;               // row in tile == TMEM lane
    const int row = m0 + 128 * i + r;              // query index
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_base + (i ? C::COL_S1 : C::COL_S0);
    const uint32_t tO = tmem + lane_base + (i ? C::COL_O1 : C::COL_O0);
    const int kv_end = i ? kv_end1 : kv_end0;
    const int qt = qt0 + i;
    // E4M3 operands carry block scales: the score factor of tile j is
    // scale*log2(e) * sq[query block] * sk[key block j]
    const float c_base = C::EB == 1 ? a.scale_log2 * a.sq[static_cast<size_t>(bh) * a.nqb + qt] : a.scale_log2;
    const int bh_k = bh_kv;  // key-side scales are per key/value head
    // With a P-cast (FP8P or E4M3 operands) the exponent carries log2(S): the
    // exps give q = S p directly, l sums q, and the epilogue divides by it.
    constexpr bool kCast = FP8P || C::EB == 1;
    // With the flush counting (more ALU work per key) 1 of every 8 key pairs on
    // the FMA pipe pays: sink workload 1013 -> 1026 TFLOP/s; without it (1146 ->
    // 1103) and in the plain bf16 forward at d = 128 (1112 -> 1084) it does not.
    constexpr int kExpPoly = COUNT ? 1 : C::EXP_POLY;
    const float lg2S = kCast ? log2f(a.p_scale) : 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    uint32_t nf_sink = 0, nf_non = 0;  // COUNT: P' that did not flush, per key class
    int cnt = 0;
    bool ok = true;
    if (kv_end > 0) {
      for (int t = 0; t < n_steps; ++t) {
        const int j = rev ? n_steps - 1 - t : t;
        if (j >= kv_end) continue;
        const float c = C::EB == 1 ? c_base * a.sk[static_cast<size_t>(bh_k) * a.nqb + j] : c_base;
        if (!(ok = mbar_wait_inl(&bar_s[i], cnt & 1, &abort_sh, 10 + i))) break;
        tc_fence_after();
        float sv[128];
        // first half of the row, then the second half streams in while the
        // first half's max is formed
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
        const int kbase = j * 128;
        const bool masked_tile = kbase + 128 > N || (a.causal && j == qt);
        const int lim = a.causal ? min(N - 1, row) : N - 1;  // last admissible key
        if (masked_tile) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (kbase + cc > lim) sv[cc] = -INFINITY;
        }
        // row max as 8 independent chains of 3-input max (a single 128-long chain
        // would be pure latency)
        float mx8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = fmax3(sv[u], sv[u + 8], sv[u + 16]);
#pragma unroll
        for (int cc = 24; cc < 56; cc += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u) mx8[u] = fmax3(mx8[u], sv[cc + u], sv[cc + 8 + u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = fmaxf(mx8[u], sv[56 + u]);
        tmem_wait_ld();
        if (masked_tile) {
#pragma unroll
          for (int cc = 64; cc < 128; ++cc)
            if (kbase + cc > lim) sv[cc] = -INFINITY;
        }
#pragma unroll
        for (int cc = 64; cc < 128; cc += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u) mx8[u] = fmax3(mx8[u], sv[cc + u], sv[cc + 8 + u]);
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        float m_new = fmaxf(m_run, mx * c);
        // Lazy rescale: keep the old max while the growth stays within 2^8 (exps stay
        // <= 256, safe in bf16/fp32).  The FP8 P-cast needs the exact running max.
        if (!FP8P && m_new - m_run <= 8.0f) m_new = m_run;
        const float alpha = ex2_approx(m_run - m_new);
        const bool rescale = cnt > 0 && __any_sync(0xffffffffu, m_new != m_run);
        l_run *= alpha;
        m_run = m_new;
        const float neg_m = lg2S - m_run;
        // 4 independent pairs of partial row sums (packed fp32x2 adds)
        float2 rs4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 c2 = make_float2(c, c), nm2 = make_float2(neg_m, neg_m);
        // COUNT, tiles that hold sink keys: the P' of keys < n_sink that did not
        // flush, counted apart before the main pass (the same fma, ex2 and cast
        // as there, so the same values); the main pass counts every key.
        uint32_t nf_part = 0;
        if constexpr (COUNT) {
          if (kbase < a.n_sink && row < N) {
#pragma unroll
            for (int cc = 0; cc < 128; ++cc) {
              if (kbase + cc < a.n_sink) {
                const float qv = ex2_approx(fmaf(sv[cc], c, neg_m));
                uint16_t e8;
                asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(e8) : "f"(0.f), "f"(qv));
                nf_part += (e8 & 0xFFu) ? 1u : 0u;
              }
            }
          }
        }
        uint32_t nf_tile = 0;
        if constexpr (C::EB == 1) {
          // P' = E4M3(S p), four codes per 32-bit TMEM column (the PV MMA's A operand)
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 x01 = ffma2(make_float2(sv[4 * e], sv[4 * e + 1]), c2, nm2);
            const float2 x23 = ffma2(make_float2(sv[4 * e + 2], sv[4 * e + 3]), c2, nm2);
            float2 s01, s23;  // S p
            if ((e & 7) < C::EXP_POLY_E4M3) {
              s01 = exp2_fma2(x01);
              s23 = exp2_fma2(x23);
            } else {
              s01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
              s23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
            }
            rs4[e & 3] = fadd2(rs4[e & 3], fadd2(s01, s23));
            uint16_t lo, hi;
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(s01.y), "f"(s01.x));
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(s23.y), "f"(s23.x));
            pk[e] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
          }
          tmem_st32(tS, pk);
        } else if constexpr (C::EB == 2) {
          // P in chunks of PC packed columns (2 keys each), stored as soon as each
          // chunk is done, so that few registers besides the score row are live
          // (measured: 8 at d = 128, 32 at d = 64)
          constexpr int PC = D == 128 ? 8 : 32;
#pragma unroll
          for (int h = 0; h < 64 / PC; ++h) {
            uint32_t pk[PC];
            uint32_t nz2 = 0;  // COUNT: f16x2 counter of non-zero P' in this chunk
#pragma unroll
            for (int e = 0; e < PC; ++e) {
              const float2 x = ffma2(make_float2(sv[h * 2 * PC + 2 * e], sv[h * 2 * PC + 2 * e + 1]), c2, nm2);
              float p0, p1;  // S p with FP8P, p otherwise
              if ((e & 7) < kExpPoly) {
                const float2 pp = exp2_fma2(x);
                p0 = pp.x;
                p1 = pp.y;
              } else {
                p0 = ex2_approx(x.x);
                p1 = ex2_approx(x.y);
              }
              rs4[e & 3] = fadd2(rs4[e & 3], make_float2(p0, p1));
              if constexpr (FP8P) {
                uint32_t h2;
                pk[e] = e4m3_round_bf16x2(p0, p1, h2);
                if constexpr (COUNT) nz2 = count_nonzero_f16x2(h2, nz2);
              } else {
                pk[e] = pack_bf16x2(p0, p1);
              }
            }
            if constexpr (COUNT) nf_tile += f16x2_sum_u32(nz2);
            if constexpr (C::PV_SS) {
              // keys [2 PC h, 2 PC h + 2 PC) of row r in the 64-key boxes, 128-byte swizzle
              constexpr int CPB = 2 * PC / 8;  // 16-byte chunks per store group
              uint8_t* pbase = smem + C::OFF_P + i * C::P_BYTES + r * 128;
#pragma unroll
              for (int c = 0; c < CPB; ++c) {
                const int key8 = h * CPB + c;  // 8-key chunk index in the row (0..15)
                *reinterpret_cast<uint4*>(pbase + (key8 >> 3) * (C::P_BYTES / 2) + (((key8 & 7) ^ (r & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
              }
            } else if constexpr (PC == 8) {
              tmem_st8(tS + h * PC, pk);
            } else if constexpr (PC == 16) {
              tmem_st16(tS + h * PC, pk);
            } else {
              tmem_st32(tS + h * PC, *reinterpret_cast<const uint32_t(*)[32]>(pk));
            }
          }
        } else {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float p = ex2_approx(fmaf(sv[h * 32 + e], c, neg_m));
              rs4[e & 3].x += p;
              pk[e] = __float_as_uint(p);
            }
            tmem_st32(tS + h * 32, pk);
          }
        }
        if constexpr (COUNT) {
          if (row < N) {
            nf_sink += nf_part;
            nf_non += nf_tile - nf_part;
          }
        }
        // O correction after P is out (the S values are dead by now, which keeps
        // register pressure down); PV_i(j-1) is complete since S_i(j) arrived.
        if (rescale) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32(tO + ch * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 r2 = fmul2(make_float2(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])),
                                      make_float2(alpha, alpha));
              ov[e] = __float_as_uint(r2.x);
              ov[e + 1] = __float_as_uint(r2.y);
            }
            tmem_st32(tO + ch * 32, ov);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        if constexpr (C::PV_SS) fence_proxy_async_smem();  // P in shared memory, read by the tensor core
        mbar_arrive(&bar_p[i]);
        {
          const float2 t01 = fadd2(rs4[0], rs4[1]), t23 = fadd2(rs4[2], rs4[3]);
          const float2 t = fadd2(t01, t23);
          l_run += t.x + t.y;
        }
        ++cnt;
      }
      // ---- epilogue: O / l -> global, LSE -> global --------------------------
      if (ok) ok = mbar_wait_inl(&bar_o[i], 0, &abort_sh, 12 + i);
      if (ok) {
        tc_fence_after();
        // l_run is the sum of S p when P is cast (S = 1 otherwise)
        const float inv = (C::EB == 1 ? a.sv[bh_kv] : 1.0f) / l_run;
        // output: fp32 for fp32 inputs, bf16 otherwise (also for E4M3 operands)
        using OutT = typename std::conditional<C::EB == 4, float, __nv_bfloat16>::type;
        OutT* orow = reinterpret_cast<OutT*>(a.o) + (static_cast<size_t>(bh) * N + row) * D;
        if constexpr (C::EB == 2) {
          // bf16 operands: O goes through shared memory and leaves by TMA, whole
          // rows at a time (rows past N are clipped by the tensor map).  The Q
          // tile's buffer is free (every MMA that read it committed before
          // bar_o) and has the O tile's size and 128-byte-swizzled layout:
          // 16-byte chunk c of row r at r * 128 + ((c ^ r) & 7) * 16 in box c / 8.
          uint8_t* ost = smem + C::OFF_Q + i * C::TILE_BYTES + r * 128;
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32(tO + ch * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int c = ch * 4 + v4;  // 16-byte chunk of the row (8 columns)
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv);
              *reinterpret_cast<uint4*>(ost + (c >> 3) * C::BOX_BYTES + ((((c & 7) ^ r) & 7) << 4)) = w;
            }
          }
          fence_proxy_async_smem();
        }
#pragma unroll
        for (int ch = 0; ch < (C::EB == 2 ? 0 : D / 32); ++ch) {
          uint32_t ov[32];
          tmem_ld32(tO + ch * 32, ov);
          tmem_wait_ld();
          if (row < N) {
            if constexpr (C::EB != 4) {
              uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv);
                dst[v4] = w;
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(orow + ch * 32);
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4)
                dst[v4] = make_float4(__uint_as_float(ov[4 * v4 + 0]) * inv, __uint_as_float(ov[4 * v4 + 1]) * inv,
                                      __uint_as_float(ov[4 * v4 + 2]) * inv, __uint_as_float(ov[4 * v4 + 3]) * inv);
            }
          }
        }
        if (row < N)
          a.lse[static_cast<size_t>(bh) * N + row] = (m_run + log2f(l_run) - lg2S) * 0.69314718055994530942f;
      }
      if constexpr (C::EB == 2) {
        // every thread of the warpgroup arrives, also one whose wait gave up; the
        // store goes out only if no wait of the CTA gave up before the barrier
        named_bar_sync_all(2 + i, 128);  // the tile's 128 rows are in shared memory
        if (r == 0 && ok && abort_sh == 0) {
#pragma unroll
          for (int b = 0; b < C::NBOX; ++b)
            tma_store_3d(&tmO, smem + C::OFF_Q + i * C::TILE_BYTES + b * C::BOX_BYTES, b * C::BOX_COLS,
                         m0 + 128 * i, bh);
          tma_store_commit();
          tma_store_wait_all();
        }
      }
      if constexpr (COUNT) {
        // flushed = admissible keys of the row minus those whose P' stayed non-zero
        uint32_t nk = 0;
        if (row < N) nk = a.causal ? static_cast<uint32_t>(row + 1) : static_cast<uint32_t>(N);
        const uint32_t ts = min(nk, static_cast<uint32_t>(max(a.n_sink, 0)));
        const uint32_t tn = nk - ts;
        const uint32_t v0 = __reduce_add_sync(0xffffffffu, ts - nf_sink);
        const uint32_t v1 = __reduce_add_sync(0xffffffffu, ts);
        const uint32_t v2 = __reduce_add_sync(0xffffffffu, tn - nf_non);
        const uint32_t v3 = __reduce_add_sync(0xffffffffu, tn);
        if (lane == 0) {
          atomicAdd(a.stats + 0, static_cast<unsigned long long>(v0));
          atomicAdd(a.stats + 1, static_cast<unsigned long long>(v1));
          atomicAdd(a.stats + 2, static_cast<unsigned long long>(v2));
          atomicAdd(a.stats + 3, static_cast<unsigned long long>(v3));
        }
      }
    }
    // teardown of the softmax warpgroups (see the third warpgroup's)
    tc_fence_before();
    named_bar_sync_all(1, C::NTHREADS);
  }
}

}  // namespace fa
