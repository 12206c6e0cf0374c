// fp8.cuh — FP8 (E4M3) operands for the attention forward.
//
// "flash-attention-trading-models", section "FA3", item 3: FP8 attention with
// incoherent processing -- the rows of Q and K are multiplied by a random
// orthogonal matrix before block quantisation, which spreads an outlier's
// magnitude over the whole row; (Q M)(K M)^T = Q K^T, so the scores are
// unchanged in exact arithmetic.  M = diag(signs) H / sqrt(d) with H the
// Sylvester Walsh-Hadamard matrix; the signs are the caller's random draw.
//
// Quantisation: Q and K get one scale per 128-row block (the attention kernel's
// tile), V one scale per head; scale = amax / 448 (1 for an all-zero block) and
// the code is E4M3(x / scale), rounded to nearest even and saturated.
//
// Launches (caller's stream), in this order:
//   fa_fp8_v_clear    sv = 0
//   fa_fp8_qk_quant   grid (blocks, B*H, 3): z = 0 Q codes and scales, z = 1 K,
//                     z = 2 the V block maxima (atomicMax into sv)
//   fa_fp8_v_quant    V codes with the per-head scale (sv holds the maximum)
//   fa_fp8_v_scale    sv: per-head maximum -> scale
#pragma once
#include "sm100.cuh"

namespace fa {

// In-register fast Walsh-Hadamard transform of one row of D values (unnormalised).
template <int D>
__device__ __forceinline__ void fwht_row(float (&x)[D]) {
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
#pragma unroll
    for (int i = 0; i < D; ++i) {
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
    }
  }
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Block reduction of a non-negative float over the 128 threads of the CTA.
__device__ __forceinline__ float block_max_128(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return m;
}

struct Fp8QuantArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* signs;  // [D] +-1, or nullptr (no rotation)
  uint8_t* q8;
  uint8_t* k8;
  uint8_t* v8;
  float* sq;           // [BH, nblk]
  float* sk;           // [BH_kv, nblk]
  float* sv;           // [BH_kv]: first the per-head amax (as ordered bits), then the scale
  int N, nblk;
  int BH, BH_kv;       // query heads, key/value heads (B*H, B*H_kv)
};

// One CTA = one 128-row block of one (b,h); thread = row.
template <int D>
__global__ void __launch_bounds__(128) fa_fp8_qk_quant_kernel(const Fp8QuantArgs a) {
  __shared__ float red[4];
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;  // 0 Q, 1 K, 2 V maxima
  // grid.y covers the larger head count; the whole CTA leaves before any barrier
  if (bh >= (which == 0 ? a.BH : a.BH_kv)) return;
  const int row = blk * 128 + threadIdx.x;
  const bool live = row < a.N;
  const __nv_bfloat16* src = which == 0 ? a.q : (which == 1 ? a.k : a.v);
  float x[D];
  if (live) {
    const uint4* p = reinterpret_cast<const uint4*>(src + (static_cast<size_t>(bh) * a.N + row) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 w = p[c];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        x[8 * c + 2 * e] = f.x;
        x[8 * c + 2 * e + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < D; ++c) x[c] = 0.f;
  }
  if (which < 2 && a.signs != nullptr) {
#pragma unroll
    for (int c = 0; c < D; ++c) x[c] *= a.signs[c];
    fwht_row<D>(x);
    const float norm = rsqrtf(static_cast<float>(D));
#pragma unroll
    for (int c = 0; c < D; ++c) x[c] *= norm;
  }
  float am = 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) am = fmaxf(am, fabsf(x[c]));
  const float amax = block_max_128(am, red);
  if (which == 2) {
    // V: contribute the block maximum to the per-head maximum (non-negative floats
    // order like their bit patterns)
    if (threadIdx.x == 0) atomicMax(reinterpret_cast<int*>(a.sv) + bh, __float_as_int(amax));
    return;
  }
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  if (threadIdx.x == 0) (which == 0 ? a.sq : a.sk)[static_cast<size_t>(bh) * a.nblk + blk] = scale;
  if (!live) return;
  uint8_t* dst = (which == 0 ? a.q8 : a.k8) + (static_cast<size_t>(bh) * a.N + row) * D;
#pragma unroll
  for (int c = 0; c < D / 16; ++c) {
    uint4 w;
    w.x = e4m3x4(__fdiv_rn(x[16 * c + 0], scale), __fdiv_rn(x[16 * c + 1], scale), __fdiv_rn(x[16 * c + 2], scale),
                 __fdiv_rn(x[16 * c + 3], scale));
    w.y = e4m3x4(__fdiv_rn(x[16 * c + 4], scale), __fdiv_rn(x[16 * c + 5], scale), __fdiv_rn(x[16 * c + 6], scale),
                 __fdiv_rn(x[16 * c + 7], scale));
    w.z = e4m3x4(__fdiv_rn(x[16 * c + 8], scale), __fdiv_rn(x[16 * c + 9], scale),
                 __fdiv_rn(x[16 * c + 10], scale), __fdiv_rn(x[16 * c + 11], scale));
    w.w = e4m3x4(__fdiv_rn(x[16 * c + 12], scale), __fdiv_rn(x[16 * c + 13], scale),
                 __fdiv_rn(x[16 * c + 14], scale), __fdiv_rn(x[16 * c + 15], scale));
    reinterpret_cast<uint4*>(dst)[c] = w;
  }
}

// d = 256: two lanes per row (lanes l and l ^ 16 of a warp hold columns
// [0, 128) and [128, 256)), so that no thread keeps a whole row in registers.
// The Hadamard transform's stages h = 1 .. 64 stay inside each half; its last
// stage pairs column i with i + 128, the two lanes of the row: a shuffle
// butterfly.  Otherwise as fa_fp8_qk_quant_kernel (one CTA = 128 rows).
__global__ void __launch_bounds__(256) fa_fp8_qk_quant256_kernel(const Fp8QuantArgs a) {
  constexpr int D = 256, HD = 128;
  __shared__ float red[8];
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;  // 0 Q, 1 K, 2 V maxima
  // grid.y covers the larger head count; the whole CTA leaves before any barrier
  if (bh >= (which == 0 ? a.BH : a.BH_kv)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int row = blk * 128 + warp * 16 + (lane & 15);
  const bool live = row < a.N;
  const __nv_bfloat16* src = which == 0 ? a.q : (which == 1 ? a.k : a.v);
  float x[HD];
  if (live) {
    const uint4* p = reinterpret_cast<const uint4*>(src + (static_cast<size_t>(bh) * a.N + row) * D + half * HD);
#pragma unroll
    for (int c = 0; c < HD / 8; ++c) {
      const uint4 w = p[c];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        x[8 * c + 2 * e] = f.x;
        x[8 * c + 2 * e + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < HD; ++c) x[c] = 0.f;
  }
  if (which < 2 && a.signs != nullptr) {
#pragma unroll
    for (int c = 0; c < HD; ++c) x[c] *= a.signs[half * HD + c];
    fwht_row<HD>(x);
#pragma unroll
    for (int c = 0; c < HD; ++c) {
      const float o = __shfl_xor_sync(0xffffffffu, x[c], 16);
      x[c] = half ? o - x[c] : x[c] + o;  // (a + b, a - b) over the lanes (lo, hi)
    }
    const float norm = rsqrtf(static_cast<float>(D));
#pragma unroll
    for (int c = 0; c < HD; ++c) x[c] *= norm;
  }
  float am = 0.f;
#pragma unroll
  for (int c = 0; c < HD; ++c) am = fmaxf(am, fabsf(x[c]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
  if (lane == 0) red[warp] = am;
  __syncthreads();
  float amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  if (which == 2) {
    if (threadIdx.x == 0) atomicMax(reinterpret_cast<int*>(a.sv) + bh, __float_as_int(amax));
    return;
  }
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  if (threadIdx.x == 0) (which == 0 ? a.sq : a.sk)[static_cast<size_t>(bh) * a.nblk + blk] = scale;
  if (!live) return;
  uint8_t* dst = (which == 0 ? a.q8 : a.k8) + (static_cast<size_t>(bh) * a.N + row) * D + half * HD;
#pragma unroll
  for (int c = 0; c < HD / 16; ++c) {
    uint4 w;
    w.x = e4m3x4(__fdiv_rn(x[16 * c + 0], scale), __fdiv_rn(x[16 * c + 1], scale), __fdiv_rn(x[16 * c + 2], scale),
                 __fdiv_rn(x[16 * c + 3], scale));
    w.y = e4m3x4(__fdiv_rn(x[16 * c + 4], scale), __fdiv_rn(x[16 * c + 5], scale), __fdiv_rn(x[16 * c + 6], scale),
                 __fdiv_rn(x[16 * c + 7], scale));
    w.z = e4m3x4(__fdiv_rn(x[16 * c + 8], scale), __fdiv_rn(x[16 * c + 9], scale),
                 __fdiv_rn(x[16 * c + 10], scale), __fdiv_rn(x[16 * c + 11], scale));
    w.w = e4m3x4(__fdiv_rn(x[16 * c + 12], scale), __fdiv_rn(x[16 * c + 13], scale),
                 __fdiv_rn(x[16 * c + 14], scale), __fdiv_rn(x[16 * c + 15], scale));
    reinterpret_cast<uint4*>(dst)[c] = w;
  }
}

// Clears the per-head V maxima before fa_fp8_qk_quant_kernel accumulates them.
__global__ void fa_fp8_v_clear_kernel(float* sv, int BH) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < BH) sv[i] = 0.f;
}

// V codes with the per-head scale; thread = 8 consecutive values.
template <int D>
__global__ void __launch_bounds__(256) fa_fp8_v_quant_kernel(const Fp8QuantArgs a, long long nvec) {
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= nvec) return;
  const long long bh = g / (static_cast<long long>(a.N) * (D / 8));
  const float amax = a.sv[bh];
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  const uint4 w = reinterpret_cast<const uint4*>(a.v)[g];
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
  float f[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(h[e]);
    f[2 * e] = __fdiv_rn(t.x, scale);
    f[2 * e + 1] = __fdiv_rn(t.y, scale);
  }
  uint2 o;
  o.x = e4m3x4(f[0], f[1], f[2], f[3]);
  o.y = e4m3x4(f[4], f[5], f[6], f[7]);
  reinterpret_cast<uint2*>(a.v8)[g] = o;
}

// Per-head maximum -> dequantisation scale.
__global__ void fa_fp8_v_scale_kernel(float* sv, int BH) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < BH) {
    const float amax = sv[i];
    sv[i] = amax > 0.f ? amax / 448.f : 1.f;
  }
}

}  // namespace fa
