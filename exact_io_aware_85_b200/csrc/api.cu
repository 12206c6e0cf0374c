// api.cu — host side of libfa.so: argument validation, TMA descriptor encoding,
// launch configuration and the extern "C" entry points declared in include/fa.h.
//
// The whole library is one translation unit (this file includes the kernel
// headers), so the device status word and the kernels live together.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "sm100.cuh"
#include "fwd.cuh"
#include "bwd.cuh"
#include "fp8.cuh"
#include "decode.cuh"
#include "fwd256.cuh"
#include "bwd256.cuh"

namespace fa {
// Self-test of the failure path: waits on an mbarrier that nothing will ever
// signal, with the given bound; the wait gives up, records FA_ERR_TIMEOUT in the
// status word and the kernel returns normally, leaving the context usable.
__global__ void fa_watchdog_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_try_wait(smem_u32(&bar), 0)) mbar_wait_slow(smem_u32(&bar), 0, &abort_flag, 77, limit_ns);
  }
  __syncthreads();
}
// Self-test of the FMA-pipe exponential: y_fma = exp2_fma2(x), y_mufu = ex2.approx(x).
__global__ void fa_exp2_selftest_kernel(const float* x, float* y_fma, float* y_mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 p = exp2_fma2(make_float2(x[i], x[i + 1]));
    y_fma[i] = p.x;
    y_fma[i + 1] = p.y;
    y_mufu[i] = ex2_approx(x[i]);
    y_mufu[i + 1] = ex2_approx(x[i + 1]);
  } else if (i < n) {
    y_fma[i] = exp2_fma2(make_float2(x[i], 0.f)).x;
    y_mufu[i] = ex2_approx(x[i]);
  }
}
}  // namespace fa

namespace {

thread_local int t_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [B*H, N, d] row-major tensor seen as a 3-D TMA tensor (d, N, B*H); box of
// 128 bytes x 128 rows with the 128-byte swizzle.  Rows beyond N read as zero.
int encode_qkv_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int N, int BH,
                   CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B, int box_rows = 128, int box_cols = 0) {
  auto fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem_bytes,
                           static_cast<cuuint64_t>(d) * static_cast<cuuint64_t>(N) * elem_bytes};
  // boxes of 128-byte rows unless given (64-byte rows with the 64-byte swizzle)
  if (box_cols <= 0) box_cols = 128 / elem_bytes;
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FA_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Size limits, set by what the launches can express rather than by memory:
// N <= 2^30 (row indices and 256-row block offsets stay int), B*H < 2^31 and
// fewer than 2^31 CTAs in the largest grid (B*H x 128-row blocks, gridDim.x),
// and B*H*N*d < 2^40 elements (the one-thread-per-8-elements grids of the
// backward's pre and post passes).  Element offsets are 64-bit everywhere.
bool sizes_fit(int B, int H, int N, int d) {
  if (N > (1 << 30)) return false;
  const long long BH = static_cast<long long>(B) * H;
  if (BH >= (1ll << 31)) return false;
  if (BH * ((static_cast<long long>(N) + 127) / 128) >= (1ll << 31)) return false;
  return BH * N * d < (1ll << 40);
}

int check_common(const void* q, const void* k, const void* v, const void* o, const void* lse, int B, int H, int N,
                 int d, float scale, bool allow256 = false) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && !(allow256 && d == 256)) return FA_ERR_UNSUPPORTED;
  if (!sizes_fit(B, H, N, d)) return FA_ERR_UNSUPPORTED;
  // lse is written one fp32 scalar at a time
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return FA_ERR_ALIGNMENT;
  return FA_OK;
}

template <typename T, int D, bool FP8P, bool COUNT = false>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int causal,
               float scale, float S, int kv_order, unsigned long long* stats, int n_sink, cudaStream_t stream,
               const float* sq = nullptr, const float* sk = nullptr, const float* sv = nullptr, int Hkv = 0) {
  if (Hkv <= 0) Hkv = H;
  using C = fa::FwdCfg<T, D, FP8P>;
  constexpr CUtensorMapDataType dt = sizeof(T) == 2   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                     : sizeof(T) == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const int BH = B * H;
  CUtensorMap mq, mk, mv;
  int st;
  // E4M3 rows at d = 64 are 64 bytes: whole-row boxes with the 64-byte swizzle
  const CUtensorMapSwizzle swz = C::SW64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  if ((st = encode_qkv_map(&mq, q, dt, sizeof(T), D, N, BH, swz, 128, C::BOX_COLS)) != FA_OK) return st;
  if ((st = encode_qkv_map(&mk, k, dt, sizeof(T), D, N, B * Hkv, swz, 128, C::BOX_COLS)) != FA_OK) return st;
  // fp32 V feeds the tf32 MMA as an MN-major operand, which needs the 32-byte-atom swizzle
  if ((st = encode_qkv_map(&mv, v, dt, sizeof(T), D, N, B * Hkv,
                           sizeof(T) == 4 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : swz, 128, C::BOX_COLS)) != FA_OK)
    return st;
  // O leaves by TMA store when the operands are bf16 (the map is unused otherwise)
  CUtensorMap mo = mq;
  if (sizeof(T) == 2 && (st = encode_qkv_map(&mo, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, N, BH)) != FA_OK)
    return st;
  fa::FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.N = N;
  a.BH = BH;
  a.nblk = (N + 255) / 256;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.p_scale = S;
  a.causal = causal ? 1 : 0;
  a.kv_order = kv_order;
  a.stats = stats;
  a.n_sink = n_sink;
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.nqb = (N + 127) / 128;
  a.group = H / Hkv;
  auto kern = fa::fa_fwd_kernel<T, D, FP8P, COUNT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e);
  // the softmax warpgroups raise their budget out of the block's launch
  // allocation (setmaxnreg); with fewer registers at launch the raise would
  // wait forever, so such a build is refused here
  cudaFuncAttributes fattr;
  e = cudaFuncGetAttributes(&fattr, kern);
  if (e != cudaSuccess) return cuda_fail(e);
  if (fattr.numRegs < C::LAUNCH_REGS) return FA_ERR_UNSUPPORTED;
  const long long grid = static_cast<long long>(a.nblk) * BH;
  kern<<<static_cast<unsigned>(grid), C::NTHREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
               void* dk, void* dv, int B, int H, int N, int causal, float scale, void* workspace,
               cudaStream_t stream, int Hkv = 0) {
  if (Hkv <= 0) Hkv = H;
  const int BH = B * H;
  const int BHkv = B * Hkv;
  const int n_tiles = (N + 127) / 128;
  // d = 256 runs two CTAs per key tile
  if (D == 256 && 2ll * n_tiles * BHkv >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  const int npad = n_tiles * 128;
  float* lse2 = static_cast<float*>(workspace);
  float* dvec = lse2 + static_cast<size_t>(BH) * npad;
  float* dq_acc = dvec + static_cast<size_t>(BH) * npad;
  CUtensorMap mq, mk, mv, mdo;
  int st;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if ((st = encode_qkv_map(&mq, q, dt, 2, D, N, BH)) != FA_OK) return st;
  if ((st = encode_qkv_map(&mk, k, dt, 2, D, N, BHkv)) != FA_OK) return st;
  if ((st = encode_qkv_map(&mv, v, dt, 2, D, N, BHkv)) != FA_OK) return st;
  if ((st = encode_qkv_map(&mdo, dO, dt, 2, D, N, BH)) != FA_OK) return st;
  // 1. D, LSE*log2(e), zeroed dQ accumulator
  const long long rows = static_cast<long long>(BH) * npad;
  const long long pre_threads = rows * (D / 8);
  fa::fa_bwd_pre_kernel<D><<<static_cast<unsigned>((pre_threads + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, lse2, dvec, dq_acc, N, npad,
      rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  // 2. main pass over (key tile, batch*head)
  fa::BwdArgs a;
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.lse2 = lse2;
  a.dvec = dvec;
  a.dq_acc = dq_acc;
  a.N = N;
  a.Npad = npad;
  a.BH = BH;
  a.n_tiles = n_tiles;
  a.group = H / Hkv;
  a.BHkv = BHkv;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.causal = causal ? 1 : 0;
  if constexpr (D == 128) {
    // 128-query steps (Q and dO tiles of 128 rows)
    using CQ = fa::BwdQ128Cfg;
    auto kern = fa::fa_bwd_main_q128_kernel;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CQ::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    // the gradient warpgroups raise their budget out of the launch allocation
    // (setmaxnreg): refuse a build whose launch register count is too small
    cudaFuncAttributes fattr;
    e = cudaFuncGetAttributes(&fattr, kern);
    if (e != cudaSuccess) return cuda_fail(e);
    if (fattr.numRegs < CQ::LAUNCH_REGS) return FA_ERR_UNSUPPORTED;
    kern<<<static_cast<unsigned>(static_cast<long long>(n_tiles) * BHkv), CQ::NTHREADS, CQ::SMEM_BYTES, stream>>>(
        mq, mk, mv, mdo, a);
  } else if constexpr (D == 256) {
    // CTA pairs (clusters of 2) per key tile: rank 0 scores, dK and dQ[:, :128];
    // rank 1 dP, dV and dQ[:, 128:]; P^T and dS^T exchanged in shared memory
    CUtensorMap mq64, mdo64;
    if ((st = encode_qkv_map(&mq64, q, dt, 2, D, N, BH, CU_TENSOR_MAP_SWIZZLE_128B, 64)) != FA_OK) return st;
    if ((st = encode_qkv_map(&mdo64, dO, dt, 2, D, N, BH, CU_TENSOR_MAP_SWIZZLE_128B, 64)) != FA_OK) return st;
    using CP = fa::BwdPairCfg;
    auto kern = fa::fa_bwd_main_pair256_kernel;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CP::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    kern<<<static_cast<unsigned>(2ll * n_tiles * BHkv), CP::NTHREADS, CP::SMEM_BYTES, stream>>>(mq64, mk, mv, mdo64,
                                                                                              a);
  } else {
    using C = fa::BwdCfg<D>;
    auto kern = fa::fa_bwd_main_kernel<D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    kern<<<static_cast<unsigned>(static_cast<long long>(n_tiles) * BHkv), C::NTHREADS, C::SMEM_BYTES, stream>>>(
        mq, mk, mv, mdo, a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  // 3. dQ accumulator -> bf16
  const long long vecs = static_cast<long long>(BH) * N * (D / 8);
  // the 128-query pass at d = 128 accumulates dS / scale (its dK epilogue and this
  // pass apply the scale); the others accumulate dS
  fa::fa_bwd_post_kernel<D><<<static_cast<unsigned>((vecs + 255) / 256), 256, 0, stream>>>(
      dq_acc, static_cast<__nv_bfloat16*>(dq), N, npad, vecs, D == 128 ? scale : 1.0f);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

int launch_bwd_d(int d, const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int N, int causal, float scale, void* workspace,
                 cudaStream_t s, int Hkv = 0) {
  if (d == 64) return launch_bwd<64>(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, causal, scale, workspace, s, Hkv);
  if (d == 256) return launch_bwd<256>(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, causal, scale, workspace, s, Hkv);
  return launch_bwd<128>(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, causal, scale, workspace, s, Hkv);
}

// ---------------------------------------------------------------------------
// Allocation-free backward: the workspace lives in a fixed device array that
// the library defines itself.  Host code must not hand the array's name to a
// kernel (on the host it only stands for the symbol); each device's address of
// it is looked up once with cudaGetSymbolAddress and cached.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = FA_BWD_NOALLOC_MAX_BYTES;  // 32 MiB, held by every GPU that loads the library
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
// per device: the address of the array and the id of the CUDA context it was
// looked up in (a reset device gets a new context, whose id is new for the life
// of the process, and the address is looked up again)
void* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};

using PFN_ctx_get_current = CUresult (*)(CUcontext*);
using PFN_ctx_get_id = CUresult (*)(CUcontext, unsigned long long*);

// Id of the context current on this thread, 0 if there is none yet (the
// runtime makes one current at its first call that needs it) or the driver
// cannot tell; with 0 the address is looked up again on every call.
unsigned long long current_context_id() {
  static PFN_ctx_get_current get_cur = nullptr;
  static PFN_ctx_get_id get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_ctx_get_current>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_ctx_get_id>(p);
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace

static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];
static_assert(sizeof(g_bwd_scratch) == FA_BWD_NOALLOC_MAX_BYTES, "scratch array size is the header's limit");

namespace {
// The device address of the scratch array in the current context.  On the host
// the array's name only stands for the symbol; the address is looked up with
// cudaGetSymbolAddress once per device and context, with that device current.
int noalloc_scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}
// Head dim 256: one 128-row Q tile per CTA, 64-key K/V tiles (fwd256.cuh);
// T = uint8_t takes E4M3 codes with their block scales.
template <typename T, bool FP8P, bool COUNT = false>
int launch_fwd256(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv, int N,
                  int causal, float scale, cudaStream_t stream, float S = 1.f, int kv_order = 0,
                  unsigned long long* stats = nullptr, int n_sink = 0, const float* sq = nullptr,
                  const float* sk = nullptr, const float* sv = nullptr) {
  using C = fa::Fwd256Cfg<sizeof(T)>;
  const auto dt = sizeof(T) == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap mq, mk, mv;
  int st;
  if ((st = encode_qkv_map(&mq, q, dt, sizeof(T), 256, N, B * H, CU_TENSOR_MAP_SWIZZLE_128B, 128)) != FA_OK) return st;
  if ((st = encode_qkv_map(&mk, k, dt, sizeof(T), 256, N, B * Hkv, CU_TENSOR_MAP_SWIZZLE_128B, 64)) != FA_OK)
    return st;
  if ((st = encode_qkv_map(&mv, v, dt, sizeof(T), 256, N, B * Hkv, CU_TENSOR_MAP_SWIZZLE_128B, 64)) != FA_OK)
    return st;
  fa::Fwd256Args a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.nqb = (N + 127) / 128;
  a.N = N;
  a.BH = B * H;
  a.nblk = (N + 127) / 128;
  a.group = H / Hkv;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.causal = causal ? 1 : 0;
  a.p_scale = S;
  a.kv_order = kv_order;
  a.stats = stats;
  a.n_sink = n_sink;
  auto kern = fa::fa_fwd256_kernel<T, FP8P, COUNT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e);
  kern<<<static_cast<unsigned>(static_cast<long long>(a.nblk) * a.BH), C::NTHREADS, C::SMEM_BYTES, stream>>>(mq, mk,
                                                                                                          mv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

// Decode split plan: enough key chunks that B * H_kv * chunks is about sixteen
// CTAs per SM (148 SMs; two are resident at a time), so the last wave is a small
// fraction of the work; chunks of whole 64-key tiles.  A pure function of the
// sizes, so the workspace size is known before any launch.
template <int D, int NT>
cudaError_t launch_decode_split(dim3 grid, cudaStream_t s, const CUtensorMap& mk, const CUtensorMap& mv,
                                const fa::DecodeArgs& a) {
  constexpr int smem = fa::DecodeLayout<D>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(fa::fa_decode_split_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  fa::fa_decode_split_kernel<D, NT><<<grid, fa::kDecThreads, smem, s>>>(mk, mv, a);
  return cudaSuccess;
}

// Key chunks per key/value head: one wave of split CTAs (one per SM), so that
// the pipeline of each CTA fills once and streams a long chunk.
void decode_plan(int B, int Hkv, int N, int* nsplit, int* tiles_per_split) {
  const int tiles = (N + fa::kDecKT - 1) / fa::kDecKT;
  const int bhkv = B * Hkv;
  const int target = std::max(1, 148 / bhkv);
  const int ns = std::min(tiles, target);
  *tiles_per_split = (tiles + ns - 1) / ns;
  *nsplit = (tiles + *tiles_per_split - 1) / *tiles_per_split;
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d, int causal,
           float scale, void* stream) {
  int st = check_common(q, k, v, o, lse, B, H, N, d, scale, true);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256) return launch_fwd256<__nv_bfloat16, false>(q, k, v, o, lse, B, H, H, N, causal, scale, s);
  if (d == 64) return launch_fwd<__nv_bfloat16, 64, false>(q, k, v, o, lse, B, H, N, causal, scale, 1.f, 0, nullptr, 0, s);
  return launch_fwd<__nv_bfloat16, 128, false>(q, k, v, o, lse, B, H, N, causal, scale, 1.f, 0, nullptr, 0, s);
}

int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N, int d,
               int causal, float scale, void* stream) {
  int st = check_common(q, k, v, o, lse, B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (d != 64) return FA_ERR_UNSUPPORTED;  // fp32 tiles of 128 x 128 do not fit the shared-memory ring
  return launch_fwd<float, 64, false>(q, k, v, o, lse, B, H, N, causal, scale, 1.f, 0, nullptr, 0,
                                      static_cast<cudaStream_t>(stream));
}

int fa_fwd_fp8p(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                int causal, float scale, float S, int kv_order, unsigned long long* stats, int n_sink,
                void* stream) {
  int st = check_common(q, k, v, o, lse, B, H, N, d, scale, true);
  if (st != FA_OK) return st;
  if (!(std::isfinite(S) && S > 0.f)) return FA_ERR_INVALID_ARG;
  if (kv_order != 0 && kv_order != 1) return FA_ERR_INVALID_ARG;
  if (n_sink < 0) return FA_ERR_INVALID_ARG;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)) return FA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256)  // 64-key tiles: the running max of the P-cast moves once per 64 keys
    return stats ? launch_fwd256<__nv_bfloat16, true, true>(q, k, v, o, lse, B, H, H, N, causal, scale, s, S,
                                                            kv_order, stats, n_sink)
                 : launch_fwd256<__nv_bfloat16, true>(q, k, v, o, lse, B, H, H, N, causal, scale, s, S, kv_order,
                                                      nullptr, n_sink);
  // the flush counting is a separate instantiation: without stats the kernel carries none of it
  if (d == 64)
    return stats ? launch_fwd<__nv_bfloat16, 64, true, true>(q, k, v, o, lse, B, H, N, causal, scale, S, kv_order,
                                                             stats, n_sink, s)
                 : launch_fwd<__nv_bfloat16, 64, true>(q, k, v, o, lse, B, H, N, causal, scale, S, kv_order, nullptr,
                                                       n_sink, s);
  return stats ? launch_fwd<__nv_bfloat16, 128, true, true>(q, k, v, o, lse, B, H, N, causal, scale, S, kv_order,
                                                            stats, n_sink, s)
               : launch_fwd<__nv_bfloat16, 128, true>(q, k, v, o, lse, B, H, N, causal, scale, S, kv_order, nullptr,
                                                      n_sink, s);
}

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N, int d,
               int causal, float scale, void* stream) {
  int st = check_common(q, k, v, o, lse, B, H, N, d, scale, true);
  if (st != FA_OK) return st;
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256) return launch_fwd256<__nv_bfloat16, false>(q, k, v, o, lse, B, H, H_kv, N, causal, scale, s);
  if (d == 64)
    return launch_fwd<__nv_bfloat16, 64, false>(q, k, v, o, lse, B, H, N, causal, scale, 1.f, 0, nullptr, 0, s,
                                                nullptr, nullptr, nullptr, H_kv);
  return launch_fwd<__nv_bfloat16, 128, false>(q, k, v, o, lse, B, H, N, causal, scale, 1.f, 0, nullptr, 0, s,
                                               nullptr, nullptr, nullptr, H_kv);
}

int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
               void* dk, void* dv, int B, int H, int H_kv, int N, int d, int causal, float scale, void* workspace,
               size_t workspace_bytes, void* stream) {
  int st = check_common(q, k, v, o, lse, B, H, N, d, scale, true);
  if (st != FA_OK) return st;
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID_ARG;
  if (!dO || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return FA_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_ALIGNMENT;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_bwd_d(d, q, k, v, o, dO, lse, dq, dk, dv, B, H, N, causal, scale, workspace, s, H_kv);
}

size_t fa_decode_workspace_bytes(int B, int H, int H_kv, int N, int d) {
  if (B < 1 || H < 1 || H_kv < 1 || N < 1 || H % H_kv != 0 || (d != 64 && d != 128 && d != 256)) return 0;
  int ns, tps;
  decode_plan(B, H_kv, N, &ns, &tps);
  const size_t bytes = static_cast<size_t>(ns) * B * H * (static_cast<size_t>(d) + 2) * sizeof(float);
  return (bytes + 255) / 256 * 256;
}

int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N, int d,
              float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || H_kv < 1 || N < 1 || H % H_kv != 0) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const int g = H / H_kv;
  if (g > fa::kDecMaxG) return FA_ERR_UNSUPPORTED;
  if (!sizes_fit(B, H, N, d)) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H_kv > 65535) return FA_ERR_UNSUPPORTED;  // key/value heads are gridDim.y
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return FA_ERR_ALIGNMENT;
  if (workspace_bytes < fa_decode_workspace_bytes(B, H, H_kv, N, d)) return FA_ERR_INVALID_ARG;
  fa::DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.N = N;
  a.BHkv = B * H_kv;
  a.g = g;
  decode_plan(B, H_kv, N, &a.nsplit, &a.tiles_per_split);
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = a.part_o + static_cast<size_t>(a.nsplit) * B * H * d;
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // K and V as [B*H_kv, N, d] in 128-key x 64-column boxes, 128-byte swizzled
  CUtensorMap mk, mv;
  int st;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if ((st = encode_qkv_map(&mk, k, dt, 2, d, N, B * H_kv, CU_TENSOR_MAP_SWIZZLE_128B, fa::kDecKT)) != FA_OK) return st;
  if ((st = encode_qkv_map(&mv, v, dt, 2, d, N, B * H_kv, CU_TENSOR_MAP_SWIZZLE_128B, fa::kDecKT)) != FA_OK) return st;
  const dim3 grid(a.nsplit, a.BHkv);
  cudaError_t e;
  if (d == 64) {
    e = g <= 8 ? launch_decode_split<64, 1>(grid, s, mk, mv, a) : launch_decode_split<64, 2>(grid, s, mk, mv, a);
    if (e != cudaSuccess) return cuda_fail(e);
    fa::fa_decode_combine_kernel<64><<<B * H, 64, 0, s>>>(a);
  } else if (d == 128) {
    e = g <= 8 ? launch_decode_split<128, 1>(grid, s, mk, mv, a) : launch_decode_split<128, 2>(grid, s, mk, mv, a);
    if (e != cudaSuccess) return cuda_fail(e);
    fa::fa_decode_combine_kernel<128><<<B * H, 128, 0, s>>>(a);
  } else {
    e = g <= 8 ? launch_decode_split<256, 1>(grid, s, mk, mv, a) : launch_decode_split<256, 2>(grid, s, mk, mv, a);
    if (e != cudaSuccess) return cuda_fail(e);
    fa::fa_decode_combine_kernel<256><<<B * H, 256, 0, s>>>(a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

int fa_fp8_quantize_gqa(const void* q, const void* k, const void* v, const float* signs, void* q8, void* k8,
                        void* v8, float* sq, float* sk, float* sv, int B, int H, int H_kv, int N, int d,
                        void* stream) {
  if (!q || !k || !v || !q8 || !k8 || !v8 || !sq || !sk || !sv) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!sizes_fit(B, H, N, d)) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return FA_ERR_UNSUPPORTED;  // heads are gridDim.y of the Q/K pass
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q8) || !aligned16(k8) || !aligned16(v8))
    return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(sq) | reinterpret_cast<uintptr_t>(sk) | reinterpret_cast<uintptr_t>(sv) |
       reinterpret_cast<uintptr_t>(signs)) & 3u)
    return FA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = B * H, BHkv = B * H_kv;
  fa::Fp8QuantArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.signs = signs;
  a.q8 = static_cast<uint8_t*>(q8);
  a.k8 = static_cast<uint8_t*>(k8);
  a.v8 = static_cast<uint8_t*>(v8);
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.N = N;
  a.nblk = (N + 127) / 128;
  a.BH = BH;
  a.BH_kv = BHkv;
  fa::fa_fp8_v_clear_kernel<<<(BHkv + 255) / 256, 256, 0, s>>>(sv, BHkv);
  const dim3 grid(a.nblk, BH, 3);  // BH >= BH_kv
  const long long nvec = static_cast<long long>(BHkv) * N * (d / 8);
  if (d == 64) {
    fa::fa_fp8_qk_quant_kernel<64><<<grid, 128, 0, s>>>(a);
    fa::fa_fp8_v_quant_kernel<64><<<static_cast<unsigned>((nvec + 255) / 256), 256, 0, s>>>(a, nvec);
  } else if (d == 256) {
    fa::fa_fp8_qk_quant256_kernel<<<grid, 256, 0, s>>>(a);
    fa::fa_fp8_v_quant_kernel<256><<<static_cast<unsigned>((nvec + 255) / 256), 256, 0, s>>>(a, nvec);
  } else {
    fa::fa_fp8_qk_quant_kernel<128><<<grid, 128, 0, s>>>(a);
    fa::fa_fp8_v_quant_kernel<128><<<static_cast<unsigned>((nvec + 255) / 256), 256, 0, s>>>(a, nvec);
  }
  fa::fa_fp8_v_scale_kernel<<<(BHkv + 255) / 256, 256, 0, s>>>(sv, BHkv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

int fa_fp8_quantize(const void* q, const void* k, const void* v, const float* signs, void* q8, void* k8, void* v8,
                    float* sq, float* sk, float* sv, int B, int H, int N, int d, void* stream) {
  return fa_fp8_quantize_gqa(q, k, v, signs, q8, k8, v8, sq, sk, sv, B, H, H, N, d, stream);
}

int fa_fwd_fp8_gqa(const void* q8, const void* k8, const void* v8, const float* sq, const float* sk,
                   const float* sv, void* o, float* lse, int B, int H, int H_kv, int N, int d, int causal, float scale,
                   float S, int kv_order, void* stream) {
  int st = check_common(q8, k8, v8, o, lse, B, H, N, d, scale, true);
  if (st != FA_OK) return st;
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID_ARG;
  if (!sq || !sk || !sv) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(S) && S > 0.f)) return FA_ERR_INVALID_ARG;
  if (kv_order != 0 && kv_order != 1) return FA_ERR_INVALID_ARG;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256)
    return launch_fwd256<uint8_t, true>(q8, k8, v8, o, lse, B, H, H_kv, N, causal, scale, s, S, kv_order, nullptr, 0,
                                        sq, sk, sv);
  if (d == 64)
    return launch_fwd<uint8_t, 64, true>(q8, k8, v8, o, lse, B, H, N, causal, scale, S, kv_order, nullptr, 0, s, sq,
                                         sk, sv, H_kv);
  return launch_fwd<uint8_t, 128, true>(q8, k8, v8, o, lse, B, H, N, causal, scale, S, kv_order, nullptr, 0, s, sq, sk,
                                        sv, H_kv);
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq, const float* sk, const float* sv,
               void* o, float* lse, int B, int H, int N, int d, int causal, float scale, float S, int kv_order,
               void* stream) {
  return fa_fwd_fp8_gqa(q8, k8, v8, sq, sk, sv, o, lse, B, H, H, N, d, causal, scale, S, kv_order, stream);
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128 && d != 256)) return 0;
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  const size_t bytes = static_cast<size_t>(B) * H * npad * (2 + static_cast<size_t>(d)) * sizeof(float);
  return (bytes + 255) / 256 * 256;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
           void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* workspace,
           size_t workspace_bytes, void* stream) {
  int st = check_common(q, k, v, o, lse, B, H, N, d, scale, true);
  if (st != FA_OK) return st;
  if (!dO || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return FA_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_ALIGNMENT;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_bwd_d(d, q, k, v, o, dO, lse, dq, dk, dv, B, H, N, causal, scale, workspace, s);
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                   void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* stream) {
  int st = check_common(q, k, v, o, lse, B, H, N, d, scale, true);
  if (st != FA_OK) return st;
  if (!dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return FA_ERR_ALIGNMENT;
  if (fa_bwd_workspace_bytes(B, H, N, d) > kNoAllocScratchBytes) return FA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if ((st = noalloc_scratch_for_current_device(&ws)) != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_bwd_d(d, q, k, v, o, dO, lse, dq, dk, dv, B, H, N, causal, scale, ws, s);
}

int fa_exp2_selftest(const float* x, float* y_fma, float* y_mufu, int n, void* stream) {
  if (!x || !y_fma || !y_mufu || n < 1) return FA_ERR_INVALID_ARG;
  if (!aligned4(x) || !aligned4(y_fma) || !aligned4(y_mufu)) return FA_ERR_ALIGNMENT;
  const int pairs = (n + 1) / 2;
  fa::fa_exp2_selftest_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_fma, y_mufu,
                                                                                                  n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

int fa_watchdog_selftest(unsigned int limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 10000000u) return FA_ERR_INVALID_ARG;
  fa::fa_watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

const char* fa_status_string(int status) {
  switch (status & 0xFF) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_CHECK: return "FA_ERR_CHECK";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

int fa_check_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, fa::g_fa_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (v != 0) {
    static const int zero = 0;
    e = cudaMemcpyToSymbolAsync(fa::g_fa_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return v & 0xFF;
}

}  // extern "C"
