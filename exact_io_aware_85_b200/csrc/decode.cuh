// decode.cuh — one decoding step: a single new query row per head against a
// long key/value cache, split over the key sequence.
//
// A decoding step is the last row of causal attention ("flash-attention-trading-
// models", "El algoritmo de atencion flash": the same online-softmax recurrence
// over key blocks, here for one query row).  With one row per head the work per
// byte of K/V is tiny, so the step is bound by reading the cache from HBM; the
// tensor cores' 128-row tiles would sit almost empty.  The kernel therefore runs
// on the CUDA cores and spreads the key sequence over many CTAs so that the
// whole GPU streams the cache (the split-KV decoding of the pages' lineage,
// "FlashAttention (IT)", "Soluzioni specializzate"), and the g query heads that
// share a key/value head ("FlashAttention for Scalable Vector Architectures",
// "Metodologia": GQA/MQA awareness) are served from one read of it.
//
//   fa_decode_split    grid (splits, B*H_kv), 256 threads: one key chunk of one
//                      key/value head; 64-key tiles double-buffered with cp.async;
//                      scores for the g query rows, online softmax, partial
//                      O (unnormalised), running max m and sum l -> workspace
//   fa_decode_combine  grid (B*H), d threads: merges the chunks' partials by
//                      their maxima (log-sum-exp), writes O (bf16) and LSE
#pragma once
#include "sm100.cuh"

namespace fa {

constexpr int kDecKT = 64;      // keys per tile
constexpr int kDecMaxG = 16;    // query heads per key/value head
constexpr int kDecThreads = 256;

struct DecodeArgs {
  const __nv_bfloat16* q;  // [B*H, d]
  const __nv_bfloat16* k;  // [B*Hkv, N, d]
  const __nv_bfloat16* v;
  __nv_bfloat16* o;        // [B*H, d]
  float* lse;              // [B*H]
  float* part_o;           // [nsplit, B*Hkv, g, d]
  float* part_ml;          // [nsplit, B*Hkv, g, 2]  (max in log2 units, sum)
  int N, BHkv, g, nsplit, tiles_per_split;
  float scale_log2;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <int D>
struct DecodeSmem {
  static constexpr int KROW = D + 8;  // padded K rows: 16 lanes' 16-byte reads land in distinct bank groups
  float q[kDecMaxG][D];
  __nv_bfloat16 k[2][kDecKT][KROW];
  __nv_bfloat16 v[2][kDecKT][D];
  float s[kDecMaxG][kDecKT];
  float m[kDecMaxG], l[kDecMaxG], alpha[kDecMaxG];
};

template <int D>
__global__ void __launch_bounds__(kDecThreads) fa_decode_split_kernel(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  DecodeSmem<D>& sm = *reinterpret_cast<DecodeSmem<D>*>(smem_raw);
  const int split = blockIdx.x, bhkv = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = a.g;
  const int t0 = split * a.tiles_per_split;
  const int ntiles_all = (a.N + kDecKT - 1) / kDecKT;
  const int t1 = min(ntiles_all, t0 + a.tiles_per_split);
  const __nv_bfloat16* kbase = a.k + static_cast<size_t>(bhkv) * a.N * D;
  const __nv_bfloat16* vbase = a.v + static_cast<size_t>(bhkv) * a.N * D;

  // query rows of the group, pre-scaled so that exp2 of a score is the weight
  for (int idx = tid; idx < g * D; idx += kDecThreads) {
    const int r = idx / D, c = idx % D;
    sm.q[r][c] = __bfloat162float(a.q[(static_cast<size_t>(bhkv) * g + r) * D + c]) * a.scale_log2;
  }
  if (tid < kDecMaxG) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.f;
  }
  auto load_tile = [&](int t, int buf) {
    constexpr int CH = D / 8;  // 16-byte chunks per row
    for (int idx = tid; idx < kDecKT * CH; idx += kDecThreads) {
      const int row = idx / CH, ch = idx % CH;
      const int key = t * kDecKT + row;
      const bool ok = key < a.N;
      const size_t off = static_cast<size_t>(ok ? key : 0) * D + ch * 8;
      cp_async16(&sm.k[buf][row][ch * 8], kbase + off, ok);
      cp_async16(&sm.v[buf][row][ch * 8], vbase + off, ok);
    }
    cp_async_commit();
  };
  if (t0 < t1) load_tile(t0, 0);

  // PV ownership: pairs (query row, 4 columns); at most 2 per thread
  constexpr int C4 = D / 4;
  float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};

  for (int t = t0; t < t1; ++t) {
    const int buf = (t - t0) & 1;
    if (t + 1 < t1) {
      load_tile(t + 1, buf ^ 1);
      cp_async_wait_one();
    } else {
      cp_async_wait_all();
    }
    __syncthreads();
    // ---- scores: thread = (key, query group); rows r = qg, qg + 4, ... -------------
    {
      const int key = tid % kDecKT, qg = tid / kDecKT;
      const bool live = t * kDecKT + key < a.N;
      float dot[kDecMaxG / 4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint4 w = *reinterpret_cast<const uint4*>(&sm.k[buf][key][ch * 8]);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int u = 0; u < kDecMaxG / 4; ++u) {
          const int r = qg + 4 * u;
          if (r < g) {
            const float4 q0 = *reinterpret_cast<const float4*>(&sm.q[r][ch * 8]);
            const float4 q1 = *reinterpret_cast<const float4*>(&sm.q[r][ch * 8 + 4]);
            dot[u] = fmaf(q0.x, kf[0], dot[u]);
            dot[u] = fmaf(q0.y, kf[1], dot[u]);
            dot[u] = fmaf(q0.z, kf[2], dot[u]);
            dot[u] = fmaf(q0.w, kf[3], dot[u]);
            dot[u] = fmaf(q1.x, kf[4], dot[u]);
            dot[u] = fmaf(q1.y, kf[5], dot[u]);
            dot[u] = fmaf(q1.z, kf[6], dot[u]);
            dot[u] = fmaf(q1.w, kf[7], dot[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kDecMaxG / 4; ++u) {
        const int r = qg + 4 * u;
        if (r < g) sm.s[r][key] = live ? dot[u] : -INFINITY;
      }
    }
    __syncthreads();
    // ---- online softmax: warp w takes rows w and w + 8 ------------------------------
    for (int r = warp; r < g; r += kDecThreads / 32) {
      const float s0 = sm.s[r][lane], s1 = sm.s[r][lane + 32];
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = sm.m[r];
      const float m_new = fmaxf(m_old, mx);  // finite: every tile has a live key
      const float p0 = ex2_approx(s0 - m_new), p1 = ex2_approx(s1 - m_new);
      sm.s[r][lane] = p0;
      sm.s[r][lane + 32] = p1;
      float sum = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) {
        const float al = ex2_approx(m_old - m_new);
        sm.alpha[r] = al;
        sm.l[r] = sm.l[r] * al + sum;
        sm.m[r] = m_new;
      }
    }
    __syncthreads();
    // ---- O += P V --------------------------------------------------------------------
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int pair = tid + u * kDecThreads;
      if (pair < g * C4) {
        const int r = pair / C4, c = (pair % C4) * 4;
        const float al = sm.alpha[r];
        float4 o4 = make_float4(acc[u].x * al, acc[u].y * al, acc[u].z * al, acc[u].w * al);
#pragma unroll 8
        for (int kk = 0; kk < kDecKT; ++kk) {
          const float p = sm.s[r][kk];
          const uint2 w = *reinterpret_cast<const uint2*>(&sm.v[buf][kk][c]);
          const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
          const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
          o4.x = fmaf(p, v01.x, o4.x);
          o4.y = fmaf(p, v01.y, o4.y);
          o4.z = fmaf(p, v23.x, o4.z);
          o4.w = fmaf(p, v23.y, o4.w);
        }
        acc[u] = o4;
      }
    }
    __syncthreads();  // the next iteration's copies overwrite this tile's buffer
  }
  // ---- partials -------------------------------------------------------------------------
  const size_t slot = static_cast<size_t>(split) * a.BHkv + bhkv;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int pair = tid + u * kDecThreads;
    if (pair < g * C4) {
      const int r = pair / C4, c = (pair % C4) * 4;
      *reinterpret_cast<float4*>(a.part_o + (slot * g + r) * D + c) = acc[u];
    }
  }
  if (tid < g) {
    a.part_ml[(slot * g + tid) * 2 + 0] = sm.m[tid];
    a.part_ml[(slot * g + tid) * 2 + 1] = sm.l[tid];
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
