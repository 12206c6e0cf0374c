// fwd256.cuh — exact attention forward for head dim 256 ("FlashAttention (IT)",
// "FlashAttention-2 (2023)": head dimension up to 256), same algorithm as fwd.cuh.
//
// At d = 256 the fp32 output tile of 128 query rows alone takes 256 of the 512
// tensor-memory columns, so the two-Q-tile ping-pong of fwd.cuh does not fit.
// Here a CTA owns one 128-row Q tile and walks 64-key K/V tiles; the score tile
// is double-buffered instead, so the tensor core computes S(j+1) = Q K_{j+1}^T
// while the softmax warps work on S(j):
//   TMEM: S buffers [0,64) and [64,128) (P written over them as bf16), O [256,512)
//   SMEM: Q 64 KB (resident), K and V rings of 2 x 32 KB
// MMA order: S(0), S(1), PV(0), S(2), PV(1), S(3), ...  S(j+2) reuses the
// buffer of S(j) and is issued after PV(j) (tcgen05 MMAs of one thread execute
// in order).  Because S(j+1) is issued before PV(j), "S(j+1) ready" does not
// imply "PV(j) done": a softmax thread that must rescale O (the lazy correction
// fires only when the row max grows by more than 2^8) first waits for PV(j).
// FP8P: the E4M3 P-cast of "P-Cast precision in FP8 attention" on 64-key tiles
// (the running max is exact, updated once per 64 keys, and the tiles can be
// visited in reverse order); COUNT also counts the P' that flush to zero.
// Elem = uint8_t: E4M3 operands with block scales ("flash-attention-trading-models",
// "FA3" item 3) on kind::f8f6f4 MMAs: rows of 256 bytes in two 128-byte boxes,
// 32 keys per PV step, P cast to E4M3 codes (four per tensor-memory column).
#pragma once
#include "sm100.cuh"

namespace fa {

struct Fwd256Args {
  __nv_bfloat16* o;
  float* lse;
  const float* sq;  // E4M3: [BH, nqb] scale per 128-row block of Q
  const float* sk;  // E4M3: [B*H_kv, nqb] per 128-row block of K
  const float* sv;  // E4M3: [B*H_kv] per head of V
  int nqb;          // ceil(N / 128)
  int N, BH, nblk, group;
  float scale_log2;
  int causal;
  float p_scale;     // static scale S of the E4M3 P-cast (FP8P)
  int kv_order;      // 0: key tiles 0..T-1, 1: T-1..0 (FP8P)
  unsigned long long* stats;  // COUNT: [sink flushed, sink counted, non-sink flushed, non-sink counted]
  int n_sink;
};

template <int EB>
struct Fwd256Cfg {
  static constexpr int D = 256;
  static constexpr int BM = 128, BN = 64;
  static constexpr int NB = D * EB / 128;         // 128-byte boxes across a row: 4 (bf16), 2 (E4M3)
  static constexpr int BOX_COLS = 128 / EB;
  static constexpr int Q_BOX = 128 * 128;         // 128 rows x 128 B
  static constexpr int KV_BOX = 64 * 128;         // 64 rows x 128 B
  static constexpr int Q_BYTES = NB * Q_BOX;      // 64 KB (bf16), 32 KB (E4M3)
  static constexpr int KV_BYTES = NB * KV_BOX;    // 32 KB (bf16), 16 KB (E4M3)
  static constexpr int NK_S = D * EB / 32;        // 32-byte K steps of S = Q K^T
  static constexpr int PV_KEYS = 32 / EB;         // keys per PV MMA step (8 tensor-memory columns of P)
  static constexpr int NK_PV = BN / PV_KEYS;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;   // 2 stages
  static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;
  static constexpr int SMEM_BYTES = OFF_V + 2 * KV_BYTES + 1024;
  static constexpr uint32_t COL_S = 0, COL_O = 256;  // S buffers at 0 and 64
  static constexpr int NTHREADS = 192;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <typename Elem, bool FP8P, bool COUNT = false>
__global__ void __launch_bounds__(192, 1)
    fa_fwd256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Fwd256Args a) {
  constexpr int EB = sizeof(Elem);
  static_assert(EB == 2 || (EB == 1 && FP8P), "bf16 operands, or E4M3 operands with the P-cast");
  using C = Fwd256Cfg<EB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_q, bar_kf[2], bar_ke[2], bar_vf[2], bar_ve[2], bar_s[2], bar_p[2], bar_pv, bar_o, bar_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work decode: query blocks of 8 adjacent heads together, heaviest first ----
  constexpr int kHeadGroup = 8;
  const int N = a.N;
  const int grp = blockIdx.x / (kHeadGroup * a.nblk);
  const int heads_in_group = min(kHeadGroup, a.BH - grp * kHeadGroup);
  const int r_in = blockIdx.x - grp * kHeadGroup * a.nblk;
  const int bh = grp * kHeadGroup + r_in % heads_in_group;
  int qt = r_in / heads_in_group;
  if (a.causal) qt = a.nblk - 1 - qt;
  const int m0 = qt * 128;
  const int bh_kv = bh / a.group;
  const int n_kv = (N + 63) >> 6;
  const int T = a.causal ? min(n_kv, 2 * qt + 2) : n_kv;  // key tiles this Q tile sees
  const bool rev = FP8P && a.kv_order;                       // visit them T-1 .. 0
  constexpr bool kE4M3 = EB == 1;

  if (warp == 5) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(&bar_q, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_ke[s], 1);
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
      mbar_init(&bar_s[s], 1);
      mbar_init(&bar_p[s], 128);
    }
    mbar_init(&bar_pv, 1);
    mbar_init(&bar_o, 1);
    mbar_init(&bar_done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 4) {
    // ============================ producer ===================================
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar_q, C::Q_BYTES);
      for (int b = 0; b < C::NB; ++b)
        tma_load_3d(smem + C::OFF_Q + b * C::Q_BOX, &tmQ, &bar_q, b * C::BOX_COLS, m0, bh);
      int t = 0;
      for (; t < T; ++t) {
        const int s = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        if (!mbar_wait(&bar_ke[s], ph ^ 1, &abort_sh, 80)) break;
        const int j = rev ? T - 1 - t : t;
        mbar_arrive_expect_tx(&bar_kf[s], C::KV_BYTES);
        for (int b = 0; b < C::NB; ++b)
          tma_load_3d(smem + C::OFF_K + s * C::KV_BYTES + b * C::KV_BOX, &tmK, &bar_kf[s], b * C::BOX_COLS, j * 64,
                      bh_kv);
        if (!mbar_wait(&bar_ve[s], ph ^ 1, &abort_sh, 81)) break;
        mbar_arrive_expect_tx(&bar_vf[s], C::KV_BYTES);
        for (int b = 0; b < C::NB; ++b)
          tma_load_3d(smem + C::OFF_V + s * C::KV_BYTES + b * C::KV_BOX, &tmV, &bar_vf[s], b * C::BOX_COLS, j * 64,
                      bh_kv);
      }
      mbar_wait_drain(&bar_q, 0, 100000000ull);
      for (int u = max(0, t - 2); u < t; ++u) {
        mbar_wait_drain(&bar_kf[u & 1], (u >> 1) & 1, 100000000ull);
        mbar_wait_drain(&bar_vf[u & 1], (u >> 1) & 1, 100000000ull);
      }
    }
  } else if (warp == 5) {
    // ============================ MMA issuer =================================
    if (lane == 0) {
      constexpr uint32_t fmt = kE4M3 ? kFmtE4M3 : kFmtBF16;
      constexpr uint32_t id_s = make_idesc(128, 64, fmt, 0, 0);   // S = Q K^T: N = 64 keys, K = 256
      constexpr uint32_t id_pv = make_idesc(128, 256, fmt, 0, 1); // O += P V: N = 256, K = 64 keys
      const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
      const uint32_t k_addr = smem_u32(smem + C::OFF_K), v_addr = smem_u32(smem + C::OFF_V);
      auto issue_s = [&](int t) {
        const int s = t & 1;
#pragma unroll
        for (int k = 0; k < C::NK_S; ++k) {
          const uint32_t qa = q_addr + (k >> 2) * C::Q_BOX + (k & 3) * 32;
          const uint32_t ka = k_addr + s * C::KV_BYTES + (k >> 2) * C::KV_BOX + (k & 3) * 32;
          if constexpr (kE4M3)
            mma_ss_f8(tmem + C::COL_S + 64 * s, make_sdesc_sw128(qa, 16, 1024), make_sdesc_sw128(ka, 16, 1024), id_s,
                      k > 0);
          else
            mma_ss(tmem + C::COL_S + 64 * s, make_sdesc_sw128(qa, 16, 1024), make_sdesc_sw128(ka, 16, 1024), id_s,
                   k > 0);
        }
        mma_commit(&bar_s[s]);
        mma_commit(&bar_ke[s]);
      };
      bool ok = mbar_wait(&bar_q, 0, &abort_sh, 82);
      for (int t = 0; ok && t < min(T, 2); ++t) {
        if (!(ok = mbar_wait(&bar_kf[t & 1], 0, &abort_sh, 83))) break;
        tc_fence_after();
        issue_s(t);
      }
      for (int t = 0; ok && t < T; ++t) {
        const int s = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        if (!(ok = mbar_wait(&bar_vf[s], ph, &abort_sh, 84))) break;
        if (!(ok = mbar_wait(&bar_p[s], ph, &abort_sh, 85))) break;
        tc_fence_after();
        // O += P(t) V(t): A = P from TMEM (8 columns per step: 16 bf16 or 32 E4M3
        // keys), B = V MN-major, K rows 128 B apart
#pragma unroll
        for (int k = 0; k < C::NK_PV; ++k) {
          const uint64_t bd = make_sdesc_sw128(v_addr + s * C::KV_BYTES + k * C::PV_KEYS * 128, C::KV_BOX, 1024);
          if constexpr (kE4M3)
            mma_ts_f8(tmem + C::COL_O, tmem + C::COL_S + 64 * s + k * 8, bd, id_pv, (t > 0 || k > 0) ? 1u : 0u);
          else
            mma_ts(tmem + C::COL_O, tmem + C::COL_S + 64 * s + k * 8, bd, id_pv, (t > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&bar_ve[s]);
        mma_commit(&bar_pv);
        if (t + 2 < T) {
          if (!(ok = mbar_wait(&bar_kf[s], ph ^ 1, &abort_sh, 86))) break;
          tc_fence_after();
          issue_s(t + 2);
        }
      }
      if (ok) mma_commit(&bar_o);
      mma_commit(&bar_done);
      mbar_wait_drain(&bar_done, 0, 100000000ull);
    }
  } else {
    // ============================ softmax warps ==============================
    const int r = threadIdx.x;  // row in tile == TMEM lane
    const int row = m0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    // E4M3 operands: the score factor of key tile j carries sq[query block] sk[key block]
    const float c_base = kE4M3 ? a.scale_log2 * a.sq[static_cast<size_t>(bh) * a.nqb + qt] : a.scale_log2;
    // with the P-cast the exponent carries log2(S): the exps give S p, l sums S p
    const float lg2S = FP8P ? log2f(a.p_scale) : 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    uint32_t nf_sink = 0, nf_non = 0;  // COUNT: P' that did not flush, per key class
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int s = t & 1;
      const int j = rev ? T - 1 - t : t;
      if (!(ok = mbar_wait(&bar_s[s], (t >> 1) & 1, &abort_sh, 87))) break;
      tc_fence_after();
      float sv[64];
      const uint32_t tS = tmem + lane_base + C::COL_S + 64 * s;
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      const int kbase = j * 64;
      const float c = kE4M3 ? c_base * a.sk[static_cast<size_t>(bh_kv) * a.nqb + (kbase >> 7)] : c_base;
      if (kbase + 64 > N || (a.causal && kbase + 63 > m0)) {
        const int lim = a.causal ? min(N - 1, row) : N - 1;
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (kbase + e > lim) sv[e] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = fmax3(sv[u], sv[u + 8], sv[u + 16]);
#pragma unroll
      for (int e = 24; e < 64; e += 8)
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = fmaxf(mx8[u], sv[e + u]);
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      float m_new = fmaxf(m_run, mx * c);
      // lazy correction (exps stay <= 2^8); the P-cast needs the exact running max
      if (!FP8P && m_new - m_run <= 8.0f) m_new = m_run;
      // in reverse order a row can meet tiles that lie wholly past its diagonal
      // before any admissible key: its max stays -inf, the tile adds nothing
      const bool none_yet = FP8P && m_new == -INFINITY;
      const float alpha = none_yet ? 1.f : ex2_approx(m_run - m_new);
      const bool rescale = t > 0 && __any_sync(0xffffffffu, m_new != m_run);
      l_run *= alpha;
      m_run = m_new;
      const float neg_m = lg2S - (none_yet ? 0.f : m_run);
      const float2 c2 = make_float2(c, c), nm2 = make_float2(neg_m, neg_m);
      // COUNT, tiles that hold sink keys: the P' of keys < n_sink that did not
      // flush, counted apart with the same fma, ex2 and cast as the main pass
      uint32_t nf_part = 0;
      if constexpr (COUNT) {
        if (kbase < a.n_sink && row < N) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc) {
            if (kbase + cc < a.n_sink) {
              const float qv = ex2_approx(fmaf(sv[cc], c, neg_m));
              uint16_t e8;
              asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(e8) : "f"(0.f), "f"(qv));
              nf_part += (e8 & 0xFFu) ? 1u : 0u;
            }
          }
        }
      }
      float2 rs4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t nz2 = 0;  // COUNT: f16x2 counter of non-zero P' (at most 32 per half)
      if constexpr (kE4M3) {
        // P' = E4M3(S p) as the PV MMA's A operand: four codes per column
        uint32_t pk8[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x01 = ffma2(make_float2(sv[4 * e], sv[4 * e + 1]), c2, nm2);
          const float2 x23 = ffma2(make_float2(sv[4 * e + 2], sv[4 * e + 3]), c2, nm2);
          const float2 s01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
          const float2 s23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
          rs4[e & 3] = fadd2(rs4[e & 3], fadd2(s01, s23));
          uint16_t lo, hi;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(s01.y), "f"(s01.x));
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(s23.y), "f"(s23.x));
          pk8[e] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        tmem_st16(tS, pk8);
      } else {
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 x = ffma2(make_float2(sv[2 * e], sv[2 * e + 1]), c2, nm2);
        const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);  // S p with FP8P, p otherwise
        rs4[e & 3] = fadd2(rs4[e & 3], make_float2(p0, p1));
        if constexpr (FP8P) {
          uint32_t h2;
          pk[e] = e4m3_round_bf16x2(p0, p1, h2);
          if constexpr (COUNT) nz2 = count_nonzero_f16x2(h2, nz2);
        } else {
          pk[e] = pack_bf16x2(p0, p1);
        }
      }
      tmem_st32(tS, pk);
      }
      if constexpr (COUNT) {
        if (row < N) {
          const uint32_t nf_tile = f16x2_sum_u32(nz2);
          nf_sink += nf_part;
          nf_non += nf_tile - nf_part;
        }
      }
      if (rescale) {
        // PV(t-1) may still be accumulating into O: wait for it before touching O
        if (!(ok = mbar_wait(&bar_pv, (t - 1) & 1, &abort_sh, 88))) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + C::COL_O + ch * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 r2 = fmul2(make_float2(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])),
                                    make_float2(alpha, alpha));
            ov[e] = __float_as_uint(r2.x);
            ov[e + 1] = __float_as_uint(r2.y);
          }
          tmem_st32(tmem + lane_base + C::COL_O + ch * 32, ov);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p[s]);
      const float2 t01 = fadd2(rs4[0], rs4[1]), t23 = fadd2(rs4[2], rs4[3]);
      const float2 tt = fadd2(t01, t23);
      l_run += tt.x + tt.y;
    }
    if (ok) ok = mbar_wait(&bar_o, 0, &abort_sh, 89);
    if (ok) {
      tc_fence_after();
      // l_run sums S p when P is cast; E4M3 V carries its per-head scale
      const float inv = (kE4M3 ? a.sv[bh_kv] : 1.0f) / l_run;
      __nv_bfloat16* orow = a.o + (static_cast<size_t>(bh) * N + row) * C::D;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_base + C::COL_O + ch * 32, ov);
        tmem_wait_ld();
        if (row < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pack_bf16x2(__uint_as_float(ov[8 * v4 + 0]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv),
                                 pack_bf16x2(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv),
                                 pack_bf16x2(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv),
                                 pack_bf16x2(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv));
        }
      }
      if (row < N)
        a.lse[static_cast<size_t>(bh) * N + row] = (m_run + log2f(l_run) - lg2S) * 0.69314718055994530942f;
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

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
