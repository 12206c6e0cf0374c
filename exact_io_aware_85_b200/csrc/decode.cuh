// decode.cuh — one decoding step: a single new query row per head against a
// long key/value cache, split over the key sequence.
//
// A decoding step is the last row of causal attention ("flash-attention-trading-
// models", "El algoritmo de atencion flash": the same online-softmax recurrence
// over key blocks, here for one query row).  With one row per head the work per
// byte of K/V is tiny, so the step is bound by reading the cache from HBM.  The
// key sequence is spread over many CTAs so that the whole GPU streams the cache
// (the split-KV decoding of the pages' lineage, "FlashAttention (IT)",
// "Soluzioni specializzate"), and the g query heads that share a key/value head
// ("FlashAttention for Scalable Vector Architectures", "Metodologia": GQA/MQA
// awareness) are served from one read of it.
//
//   fa_decode_split    grid (splits, B*H_kv), 256 threads, one CTA per SM: one
//                      key chunk of one key/value head.  128-key K and V tiles
//                      arrive by TMA (128-byte swizzled, rows past N
//                      zero-filled) through a 192 KB ring, so that two tiles
//                      are in flight while one is consumed.  The g query rows
//                      are the 8-wide N side of warp-level tensor-core MMAs
//                      (m16n8k16, bf16 in, fp32 accumulate):
//                        S^T = K Q^T      warp w: keys [16w, 16w + 16)
//                        O^T += V^T P^T   warp w: 16 of the d output columns
//                      At d = 256 a K or V tile is 64 KB, so the ring holds
//                      single tiles (K_i, V_i, K_i+1, ...), each refilled as
//                      soon as it is consumed: still 128-192 KB in flight.
//                      Out of a streaming kernel the tensor cores take the
//                      instruction count, not the time: on the CUDA cores the
//                      same arithmetic left the kernel issue-latency bound at
//                      a fifth of the copy rate.  Online softmax per query row
//                      in between; partial O (unnormalised), running max m and
//                      sum l -> workspace
//   fa_decode_combine  grid (B*H), d threads: merges the chunks' partials by
//                      their maxima (log-sum-exp), writes O (bf16) and LSE
#pragma once
#include "sm100.cuh"

namespace fa {

constexpr int kDecKT = 128;     // keys per tile
constexpr int kDecMaxG = 16;    // query heads per key/value head
constexpr int kDecThreads = 256;

struct DecodeArgs {
  const __nv_bfloat16* q;  // [B*H, d]
  __nv_bfloat16* o;        // [B*H, d]
  float* lse;              // [B*H]
  float* part_o;           // [nsplit, B*Hkv, g, d]
  float* part_ml;          // [nsplit, B*Hkv, g, 2]  (max in log2 units, sum)
  int N, BHkv, g, nsplit, tiles_per_split;
  float scale_log2;
};

// Shared memory: the K/V ring (tiles of 128 rows x 128 B boxes, 1024-byte
// aligned), P^T as bf16 [16 query rows][128 keys] with rows padded by 16 bytes
// (conflict-free ldmatrix), the cross-warp maxima and sums, the stage barriers.
template <int D>
struct DecodeLayout {
  static constexpr int BOX = kDecKT * 128;          // 128 rows x 128 B (64 columns)
  static constexpr int TILE = (D / 64) * BOX;       // one 128 x D tile
  static constexpr bool SPLIT_KV = D > 128;         // ring slots hold one tile (K or V), not a K+V pair
  static constexpr int STAGE = SPLIT_KV ? TILE : 2 * TILE;
  static constexpr int STAGES = 196608 / STAGE;     // 192 KB ring: 3 stages (d 128), 6 (d 64), 3 tiles (d 256)
  static constexpr int P_LD = kDecKT * 2 + 16;      // bytes per P^T row
  static constexpr int OFF_P = STAGES * STAGE;
  static constexpr int OFF_RED = OFF_P + kDecMaxG * P_LD;  // float [2][8 warps][16]
  static constexpr int OFF_BAR = OFF_RED + 2 * 8 * kDecMaxG * 4;
  static constexpr int OFF_ABORT = OFF_BAR + STAGES * 8;
  static constexpr int BYTES = OFF_ABORT + 16 + 1024;  // + alignment slack
  static_assert(BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row-major) B (16x8 bf16, column-major)
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NT: 8-wide tiles of query rows (1 for g <= 8, 2 for g <= 16).
template <int D, int NT>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const DecodeArgs a) {
  using L = DecodeLayout<D>;
  constexpr int NST = L::STAGES;
  constexpr int KSTEPS = D / 16;  // 16-deep MMA steps over the head dim
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* const pt = smem + L::OFF_P;
  float* const red_max = reinterpret_cast<float*>(smem + L::OFF_RED);  // [8][16]
  float* const red_sum = red_max + 8 * kDecMaxG;                      // [8][16]
  uint64_t* const full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  volatile int* const abort_sh = reinterpret_cast<volatile int*>(smem + L::OFF_ABORT);

  const int g = a.g;
  const int split = blockIdx.x, bhkv = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane >> 2, tq = lane & 3;  // MMA fragment coordinates
  const int t0 = split * a.tiles_per_split;
  const int ntiles_all = (a.N + kDecKT - 1) / kDecKT;
  const int nt = max(0, min(ntiles_all, t0 + a.tiles_per_split) - t0);

  if (tid == 0) {
    *abort_sh = 0;
    for (int s = 0; s < NST; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // ring loads: K+V of tile t0 + n (d <= 128), or K (n even) / V (n odd) of tile
  // t0 + n/2 (d = 256), into slot n % NST; only thread 0 issues and counts them
  const int n_loads = L::SPLIT_KV ? 2 * nt : nt;
  int issued = 0;
  auto issue = [&](int n) {
    uint8_t* st = smem + (n % NST) * L::STAGE;
    uint64_t* bar = &full[n % NST];
    mbar_arrive_expect_tx(bar, L::STAGE);
    if constexpr (L::SPLIT_KV) {
      const int key0 = (t0 + n / 2) * kDecKT;
      for (int b = 0; b < D / 64; ++b) {
        if (n & 1) tma_load_3d(st + b * L::BOX, &tmV, bar, b * 64, key0, bhkv);
        else tma_load_3d(st + b * L::BOX, &tmK, bar, b * 64, key0, bhkv);
      }
    } else {
      const int key0 = (t0 + n) * kDecKT;
      for (int b = 0; b < D / 64; ++b) {
        tma_load_3d(st + b * L::BOX, &tmK, bar, b * 64, key0, bhkv);
        tma_load_3d(st + L::TILE + b * L::BOX, &tmV, bar, b * 64, key0, bhkv);
      }
    }
    issued = n + 1;
  };
  // let every copy still in flight land before the block can exit
  auto drain_from = [&](int n0) {
    if (tid == 0)
      for (int n = n0; n < issued; ++n) mbar_wait_drain(&full[n % NST], (n / NST) & 1, 100000000ull);
  };
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int n = 0; n < NST && n < n_loads; ++n) issue(n);
  }

  // Q^T as the B operand of S^T = K Q^T: for query column n = 8j + grp and
  // head-dim step s, {q[n][16s + 2tq], q[n][16s + 2tq + 1]} and the same 8 further
  // on; rows n >= g are zero.  (Scaled after the MMA, so q stays exact in bf16.)
  uint32_t qb[NT][KSTEPS][2];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int n = 8 * j + grp;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(a.q + (static_cast<size_t>(bhkv) * g + min(n, g - 1)) * D);
#pragma unroll
    for (int s = 0; s < KSTEPS; ++s) {
      qb[j][s][0] = n < g ? qrow[8 * s + tq] : 0u;
      qb[j][s][1] = n < g ? qrow[8 * s + 4 + tq] : 0u;
    }
  }
  // per thread: query columns 8j + 2tq and 8j + 2tq + 1 (the same in the score
  // and the output fragments)
  float m_run[NT][2], l_run[NT][2];
  // output columns of this warp: MT blocks of 16 (two at d = 256), and, for
  // d = 64, its half of each tile's keys
  constexpr int MT = D > 128 ? 2 : 1;
  constexpr int WARPS_PER_D = D / (16 * MT);           // 8 (d 256, 128) or 4 (d 64)
  float oacc[NT][MT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    m_run[j][0] = m_run[j][1] = -INFINITY;
    l_run[j][0] = l_run[j][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) oacc[j][mt][0] = oacc[j][mt][1] = oacc[j][mt][2] = oacc[j][mt][3] = 0.f;
  }
  const int ocol = 16 * MT * (warp % WARPS_PER_D);
  const int khalf = warp / WARPS_PER_D;                // 0, or 0/1 for d 64
  constexpr int PV_STEPS = (kDecKT / 16) / (8 / WARPS_PER_D);
  const uint32_t pt_addr = smem_u32(pt);
  bool ok = true;

  for (int i = 0; i < nt; ++i) {
    const int nk = L::SPLIT_KV ? 2 * i : i;  // the load that holds K_i
    const uint32_t kt = smem_u32(smem + (nk % NST) * L::STAGE);
    const uint32_t vt = L::SPLIT_KV ? smem_u32(smem + ((nk + 1) % NST) * L::STAGE) : kt + L::TILE;
    const bool got = mbar_wait(&full[nk % NST], (nk / NST) & 1, abort_sh, 20);
    if (__syncthreads_or(!got)) {
      drain_from(nk);
      ok = false;
      break;
    }
    const int key0 = (t0 + i) * kDecKT;
    // ---- S^T = K Q^T for keys [16w, 16w + 16) -----------------------------------
    float sc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
    {
      const int mi = lane >> 3, r8 = lane & 7;
      const int krow = 16 * warp + r8 + 8 * (mi & 1);
#pragma unroll
      for (int s = 0; s < KSTEPS; ++s) {
        const int chunk = (s & 3) * 2 + (mi >> 1);  // 16-byte chunk in the 64-column box
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kt + (s >> 2) * L::BOX + krow * 128 + ((chunk ^ (krow & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
        for (int j = 0; j < NT; ++j) mma_16816(sc[j], a0, a1, a2, a3, qb[j][s][0], qb[j][s][1]);
      }
    }
    // scores in exp2 units; keys past N do not exist
    const int kA = key0 + 16 * warp + grp, kB = kA + 8;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      sc[j][0] = kA < a.N ? sc[j][0] * a.scale_log2 : -INFINITY;
      sc[j][1] = kA < a.N ? sc[j][1] * a.scale_log2 : -INFINITY;
      sc[j][2] = kB < a.N ? sc[j][2] * a.scale_log2 : -INFINITY;
      sc[j][3] = kB < a.N ? sc[j][3] * a.scale_log2 : -INFINITY;
    }
    // ---- tile maxima per query column: over this thread's two keys, the warp's
    // 8 key groups (lanes with equal tq), then the 8 warps -------------------------
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      float x0 = fmaxf(sc[j][0], sc[j][2]), x1 = fmaxf(sc[j][1], sc[j][3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
      }
      if (grp == 0) {
        red_max[warp * kDecMaxG + 8 * j + 2 * tq] = x0;
        red_max[warp * kDecMaxG + 8 * j + 2 * tq + 1] = x1;
      }
    }
    __syncthreads();
    if constexpr (L::SPLIT_KV) {
      // every warp is past PV(i-1) and S^T(i): the slots of V_{i-1} and K_i refill
      if (tid == 0) {
        if (i > 0 && 2 * i + 2 < n_loads) issue(2 * i + 2);
        if (2 * i + 3 < n_loads) issue(2 * i + 3);
      }
    } else {
      // the previous tile's stage is free now (every warp is past its PV)
      if (tid == 0 && i > 0 && i - 1 + NST < nt) issue(i - 1 + NST);
    }
    float alpha[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = 8 * j + 2 * tq + c;
        float mx = red_max[n];
#pragma unroll
        for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red_max[w * kDecMaxG + n]);
        const float m_new = fmaxf(m_run[j][c], mx);  // finite: every tile has a live key
        alpha[j][c] = ex2_approx(m_run[j][c] - m_new);
        m_run[j][c] = m_new;
      }
      const float p0 = ex2_approx(sc[j][0] - m_run[j][0]), p1 = ex2_approx(sc[j][1] - m_run[j][1]);
      const float p2 = ex2_approx(sc[j][2] - m_run[j][0]), p3 = ex2_approx(sc[j][3] - m_run[j][1]);
      // P^T[n][key] in bf16 for the PV MMA
      const int n0 = 8 * j + 2 * tq;
      const int kl = 16 * warp + grp;
      *reinterpret_cast<__nv_bfloat16*>(pt + n0 * L::P_LD + kl * 2) = __float2bfloat16_rn(p0);
      *reinterpret_cast<__nv_bfloat16*>(pt + (n0 + 1) * L::P_LD + kl * 2) = __float2bfloat16_rn(p1);
      *reinterpret_cast<__nv_bfloat16*>(pt + n0 * L::P_LD + (kl + 8) * 2) = __float2bfloat16_rn(p2);
      *reinterpret_cast<__nv_bfloat16*>(pt + (n0 + 1) * L::P_LD + (kl + 8) * 2) = __float2bfloat16_rn(p3);
      float s0 = p0 + p2, s1 = p1 + p3;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, off);
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      }
      if (grp == 0) {
        red_sum[warp * kDecMaxG + n0] = s0;
        red_sum[warp * kDecMaxG + n0 + 1] = s1;
      }
    }
    if constexpr (L::SPLIT_KV) {
      // V_i has its own slot and barrier
      const bool got_v = mbar_wait(&full[(nk + 1) % NST], ((nk + 1) / NST) & 1, abort_sh, 21);
      if (__syncthreads_or(!got_v)) {
        drain_from(nk + 1);
        ok = false;
        break;
      }
    } else {
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = 8 * j + 2 * tq + c;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += red_sum[w * kDecMaxG + n];
        l_run[j][c] = l_run[j][c] * alpha[j][c] + sum;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        oacc[j][mt][0] *= alpha[j][0];
        oacc[j][mt][1] *= alpha[j][1];
        oacc[j][mt][2] *= alpha[j][0];
        oacc[j][mt][3] *= alpha[j][1];
      }
    }
    // ---- O^T += V^T P^T for output columns [ocol, ocol + 16 MT) -----------------
    {
      const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
      for (int s = 0; s < PV_STEPS; ++s) {
        const int kk = khalf * PV_STEPS + s;           // 16-key step
        const int vrow = 16 * kk + r8 + 8 * (mi >> 1);
        uint32_t av[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int col = ocol + 16 * mt;
          const int cbase = (col % 64) / 8 + (mi & 1);  // 16-byte chunk of the 8 columns
          ldsm_x4_t(vt + (col / 64) * L::BOX + vrow * 128 + ((cbase ^ (vrow & 7)) << 4), av[mt][0], av[mt][1],
                    av[mt][2], av[mt][3]);
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          uint32_t b0, b1;
          ldsm_x2(pt_addr + (8 * j + r8) * L::P_LD + (16 * kk + 8 * (mi & 1)) * 2, b0, b1);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) mma_16816(oacc[j][mt], av[mt][0], av[mt][1], av[mt][2], av[mt][3], b0, b1);
        }
      }
    }
  }
  if (!ok) return;
  __syncthreads();  // every warp is done with the ring
  // ---- partials: O^T fragment (column ocol + grp (+8), query 8j + 2tq (+1)) ------
  const size_t slot = static_cast<size_t>(split) * a.BHkv + bhkv;
  float* po = a.part_o + slot * g * D;
  if constexpr (WARPS_PER_D == 8) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int n0 = 8 * j + 2 * tq;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int col = ocol + 16 * mt + grp;
        if (n0 < g) {
          po[n0 * D + col] = oacc[j][mt][0];
          po[n0 * D + col + 8] = oacc[j][mt][2];
        }
        if (n0 + 1 < g) {
          po[(n0 + 1) * D + col] = oacc[j][mt][1];
          po[(n0 + 1) * D + col + 8] = oacc[j][mt][3];
        }
      }
    }
  } else {
    // d = 64: the two key halves' partial O meet in the idle ring
    float* red = reinterpret_cast<float*>(smem);  // [2][16][D]
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int n0 = 8 * j + 2 * tq;
      red[(khalf * kDecMaxG + n0) * D + ocol + grp] = oacc[j][0][0];
      red[(khalf * kDecMaxG + n0 + 1) * D + ocol + grp] = oacc[j][0][1];
      red[(khalf * kDecMaxG + n0) * D + ocol + grp + 8] = oacc[j][0][2];
      red[(khalf * kDecMaxG + n0 + 1) * D + ocol + grp + 8] = oacc[j][0][3];
    }
    __syncthreads();
    for (int idx = tid; idx < g * D; idx += kDecThreads) po[idx] = red[idx] + red[kDecMaxG * D + idx];
  }
  if (warp == 0 && grp == 0) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = 8 * j + 2 * tq + c;
        if (n < g) {
          a.part_ml[(slot * g + n) * 2 + 0] = m_run[j][c];
          a.part_ml[(slot * g + n) * 2 + 1] = l_run[j][c];
        }
      }
  }
}

template <int D>
__global__ void __launch_bounds__(D) fa_decode_combine_kernel(const DecodeArgs a) {
  const int bh = blockIdx.x;  // query head (b*H + h)
  const int bhkv = bh / a.g, r = bh % a.g;
  const int c = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, a.part_ml[((static_cast<size_t>(s) * a.BHkv + bhkv) * a.g + r) * 2]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < a.nsplit; ++s) {
    const size_t slot = (static_cast<size_t>(s) * a.BHkv + bhkv) * a.g + r;
    const float w = ex2_approx(a.part_ml[slot * 2] - M);
    L = fmaf(a.part_ml[slot * 2 + 1], w, L);
    acc = fmaf(a.part_o[slot * D + c], w, acc);
  }
  a.o[static_cast<size_t>(bh) * D + c] = __float2bfloat16_rn(acc / L);
  if (c == 0) a.lse[bh] = (M + log2f(L)) * 0.69314718055994530942f;
}

}  // namespace fa
