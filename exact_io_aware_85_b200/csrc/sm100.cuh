// sm100.cuh — thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// attention kernels use: mbarriers, TMA tiled bulk copies, tcgen05 tensor-memory
// allocation, tcgen05.mma (kind::f16) with shared-memory descriptors, tcgen05.ld/st,
// and the fences that order them.  Every wrapper is hand-written from the public
// PTX ISA description of the instruction; nothing here is generated.
//
// Every wait in this library is bounded: a wait that runs past FA_WAIT_LIMIT_NS
// records FA_ERR_TIMEOUT in the device status word, raises the CTA-local abort
// flag and returns false, so a broken pipeline ends the kernel instead of hanging
// the GPU.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda.h>

#ifndef FA_WAIT_LIMIT_NS
#define FA_WAIT_LIMIT_NS 2000000000ull   // 2 s: far above any legitimate wait
#endif

namespace fa {

// ----------------------------------------------------------------------------
// generic helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}


// Status word shared by all kernels of the library.  Codes match fa_status in
// include/fa.h; bits [8,16) carry the id of the wait that gave up.  The library
// is compiled as a single translation unit, so the definition lives here.
__device__ int g_fa_status = 0;

// Debug builds (-DFA_DEBUG) check the arguments of every TMA copy, tensor-memory
// load/store and MMA before issuing it; a failed check records FA_ERR_CHECK (6)
// with the check's site in bits 8-15 of the status word (the first failure
// wins) and the operation is skipped, so a bad index is reported instead of
// reaching the hardware.  Release builds compile the checks away.
#ifdef FA_DEBUG
__device__ __forceinline__ bool fa_check(bool ok, int site) {
  if (!ok) atomicCAS(&g_fa_status, 0, 6 | (site << 8));
  return ok;
}
#define FA_CHECK(cond, site) fa::fa_check((cond), (site))
#else
#define FA_CHECK(cond, site) true
#endif
// N of an instruction descriptor (bits 17-22 hold N / 8)
__host__ __device__ constexpr uint32_t idesc_n(uint32_t idesc) { return ((idesc >> 17) & 63u) << 3; }
// tensor memory: the columns [col, col + n) exist (512 allocated) and, for loads
// and stores, the lanes are the calling warp's quarter (warp w reaches lanes
// 32 (w % 4) .. 32 (w % 4) + 31)
__device__ __forceinline__ bool tmem_cols_ok(uint32_t taddr, uint32_t n) { return (taddr & 0xFFFFu) + n <= 512u; }
__device__ __forceinline__ bool tmem_quarter_ok(uint32_t taddr) {
  return (taddr >> 21) == ((threadIdx.x >> 5) & 3u) && ((taddr >> 16) & 31u) == 0u;
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  `abort_flag`
// is a CTA-shared word; once any thread of the CTA gave up, the others stop
// waiting too.  Returns false on timeout/abort.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag, int site,
                                            uint64_t limit_ns = FA_WAIT_LIMIT_NS) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicCAS(&g_fa_status, 0, 5 /*FA_ERR_TIMEOUT*/ | (site << 8));
        *abort_flag = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  return mbar_wait_slow(a, parity, abort_flag, site);
}
// The same bounded wait with the slow path inlined, for warps whose register
// budget was raised with setmaxnreg: ptxas cannot call an out-of-line function
// from code that runs with more registers than the kernel was launched with.
__device__ __forceinline__ bool mbar_wait_inl(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int site) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > FA_WAIT_LIMIT_NS) {
        atomicCAS(&g_fa_status, 0, 5 /*FA_ERR_TIMEOUT*/ | (site << 8));
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// TMA (tiled bulk tensor copies), global -> shared, completion on an mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  // boxes land 128-byte aligned; x must start on a 16-byte boundary (every box
  // here starts at a multiple of 8 elements of at most 2 bytes, or 32 fp32)
  if (!FA_CHECK((smem_u32(smem_dst) & 127u) == 0 && x >= 0 && (x & 7) == 0 && z >= 0, 200)) return;
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
// shared -> global tiled bulk store (rows past the tensor's extent are not
// written); completion is tracked with the bulk-async group of the thread
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int x, int y, int z) {
  if (!FA_CHECK((smem_u32(smem_src) & 127u) == 0 && x >= 0 && (x & 7) == 0 && y >= 0 && z >= 0, 201)) return;
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk store of this thread has completed
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// make generic-proxy shared-memory writes visible to the async proxy (TMA, tcgen05.mma)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier that threads may reach from different code paths, also with
// their warp diverged (the non-.aligned form counts arriving threads, wherever
// and however they arrive).
__device__ __forceinline__ void named_bar_sync_all(int id, int nthreads) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ----------------------------------------------------------------------------
// Thread-block clusters: two CTAs of one cluster exchange operand tiles through
// distributed shared memory.  The copies are plain shared-to-shared bulk copies
// into the peer CTA (no multicast loads); their completion is counted in bytes
// on an mbarrier of the receiving CTA, like a TMA load's.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// every thread of every CTA of the cluster; release/acquire at cluster scope
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the shared::cluster address of the same shared-memory object in CTA `rank`
__device__ __forceinline__ uint32_t peer_smem(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// one arrival on a barrier of the peer CTA that also raises its expected bytes
__device__ __forceinline__ void mbar_arrive_expect_tx_peer(uint32_t peer_bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(peer_bar),
               "r"(bytes)
               : "memory");
}
// `bytes` (multiple of 16, both addresses 16-byte aligned) from this CTA's shared
// memory into the peer's, completed on the peer's barrier `peer_bar`
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t peer_dst, const void* src, uint32_t bytes,
                                                  uint32_t peer_bar) {
  if (!FA_CHECK(((peer_dst | smem_u32(src) | bytes) & 15u) == 0, 206)) return;
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   peer_dst),
               "r"(smem_u32(src)), "r"(bytes), "r"(peer_bar)
               : "memory");
}
// Bounded wait as mbar_wait, acquiring at cluster scope: for barriers that the
// peer CTA arrives on.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  int site) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(a, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > FA_WAIT_LIMIT_NS) {
        atomicCAS(&g_fa_status, 0, 5 /*FA_ERR_TIMEOUT*/ | (site << 8));
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Per-warpgroup register budgets (all four warps of a warpgroup execute the same
// instruction).  `dec` returns registers to the block's pool, `inc` waits until
// the pool holds enough; the pool is the block's launch allocation (threads x
// registers per thread at launch), so the budgets must add up to no more.
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
// from the launch budget FROM to TO, in whichever direction that is
template <uint32_t FROM, uint32_t TO>
__device__ __forceinline__ void setmaxnreg_to() {
  if constexpr (TO > FROM)
    setmaxnreg_inc<TO>();
  else if constexpr (TO < FROM)
    setmaxnreg_dec<TO>();
}

// ----------------------------------------------------------------------------
// tcgen05: tensor memory
// ----------------------------------------------------------------------------
// One full warp allocates `ncols` (power of two >= 32) TMEM columns; the base
// address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ----------------------------------------------------------------------------
// tcgen05.mma  (single CTA, kind::f16 / kind::tf32, fp32 accumulate in TMEM)
// ----------------------------------------------------------------------------
// Instruction descriptor (32 bit): D format at [4,6) (1 = f32), A format [7,10),
// B format [10,13) (f16 = 0, bf16 = 1, tf32 = 2), A major [15], B major [16]
// (0 = K-major, 1 = MN-major), N>>3 at [17,23), M>>4 at [24,29).
enum : uint32_t { kFmtF16 = 0, kFmtBF16 = 1, kFmtTF32 = 2, kFmtE4M3 = 0 /* kind::f8f6f4 */ };
__host__ __device__ constexpr uint32_t make_idesc(uint32_t M, uint32_t N, uint32_t ab_fmt, uint32_t a_mn_major,
                                                  uint32_t b_mn_major) {
  return (1u << 4) | (ab_fmt << 7) | (ab_fmt << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Shared-memory matrix descriptor (64 bit) for a 128-byte-swizzled operand:
// start address>>4 at [0,14), leading byte offset>>4 at [16,30), stride byte
// offset>>4 at [32,46), version 1 at [46,48), layout type 2 (SWIZZLE_128B) at
// [61,64).  K-major: SBO = distance between 8-row groups (1024 B for dense rows
// of 128 B); LBO unused.  MN-major: LBO = distance between 64-element column
// blocks, SBO = distance between 8-row groups along K.
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// The same for the 64-byte swizzle (layout type 4): rows of 64 bytes, the
// pattern repeats every 8 rows (512 bytes).  Used for E4M3 tiles at d = 64.
__device__ __forceinline__ uint64_t make_sdesc_sw64(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 4ull << 61;
  return d;
}

// The descriptor of the same operand `bytes` further on: the start address is
// the low 14-bit field (address >> 4), so the offset adds there directly as long
// as address + bytes stays below 2^18 (all of shared memory does).  Building one
// base descriptor per operand and adding constant offsets keeps the issuing
// thread's work between MMAs to one add.
__device__ __forceinline__ uint64_t sdesc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// Same, for the 128-byte swizzle with 32-byte atoms (layout type 1), the only
// MN-major layout the tf32 MMA accepts; 4-row (512 B) swizzle period along K.
__device__ __forceinline__ uint64_t make_sdesc_sw128_32b(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 1ull << 61;
  return d;
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  if (!FA_CHECK((d_tmem >> 16) == 0u && tmem_cols_ok(d_tmem, idesc_n(idesc)), 205)) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ss_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  if (!FA_CHECK((d_tmem >> 16) == 0u && tmem_cols_ok(d_tmem, idesc_n(idesc)), 205)) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// A operand from tensor memory (K-major, packed 2 x 16-bit per 32-bit column)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  if (!FA_CHECK((d_tmem >> 16) == 0u && tmem_cols_ok(d_tmem, idesc_n(idesc)) && (a_tmem >> 16) == 0u &&
                    tmem_cols_ok(a_tmem, 8), 205)) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  if (!FA_CHECK((d_tmem >> 16) == 0u && tmem_cols_ok(d_tmem, idesc_n(idesc)) && (a_tmem >> 16) == 0u &&
                    tmem_cols_ok(a_tmem, 8), 205)) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// kind::f8f6f4 (E4M3 operands, K = 32 per instruction), A from shared memory or TMEM
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  if (!FA_CHECK((d_tmem >> 16) == 0u && tmem_cols_ok(d_tmem, idesc_n(idesc)), 205)) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  if (!FA_CHECK((d_tmem >> 16) == 0u && tmem_cols_ok(d_tmem, idesc_n(idesc)) && (a_tmem >> 16) == 0u &&
                    tmem_cols_ok(a_tmem, 8), 205)) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 op issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// The same arrival on the barrier at `bar`'s offset in each CTA of the cluster
// named by `cta_mask` (bit r = cluster rank r); a signal only, no data moves.
__device__ __forceinline__ void mma_commit_cluster(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05.ld / tcgen05.st, shape 32x32b: thread t of warp w (w%4 = q) touches
// TMEM lane 32q+t; .xN moves N consecutive 32-bit columns.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  if (!FA_CHECK(tmem_quarter_ok(taddr) && tmem_cols_ok(taddr, 32), 203)) return;
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  if (!FA_CHECK(tmem_quarter_ok(taddr) && tmem_cols_ok(taddr, 32), 204)) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
      "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  if (!FA_CHECK(tmem_quarter_ok(taddr) && tmem_cols_ok(taddr, 8), 204)) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
      "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  if (!FA_CHECK(tmem_quarter_ok(taddr) && tmem_cols_ok(taddr, 16), 204)) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// ----------------------------------------------------------------------------
// arithmetic helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Blackwell packed fp32x2 arithmetic: two lanes of work per issue slot.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, C, D;\n\t"
      "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\tmov.b64 C, {%6, %7};\n\t"
      "fma.rn.f32x2 D, A, B, C;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, D;\n\t"
      "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "add.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, D;\n\t"
      "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mul.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, D;\n\t"
      "mov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "sub.rn.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 2^x of two values on the FMA and integer pipes, so that part of a softmax
// tile's exponentials run beside the MUFU ex2 instead of queueing for it.
// x is clamped to >= -126 (exponent field >= 1 after the shift below), split as
// x = j + f with j = round-to-nearest(x) (adding 1.5 * 2^23 leaves j in the low
// mantissa bits; subtracting it again gives j exactly, and x - j is exact) and
// |f| <= 1/2; 2^f comes from a degree-3 polynomial and j is added to the
// exponent field as an integer.  The polynomial is the minimax approximation of
// 2^f on [-1/2, 1/2] in relative error, found with the Remez exchange algorithm
// (equioscillation at five points); with these float32 coefficients its largest
// relative error is 7.5e-5, below the 2^-9 half-ulp of the bf16 P it feeds.
// Inputs are <= 127 (the softmax arguments here are <= 8).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float c0 = 0.99992805719375610f, c1 = 0.69326096773147583f, c2 = 0.24261112511157990f,
                  c3 = 0.05517166852951050f;
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 kRound = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
  const float2 t = fadd2(x, kRound);
  const float2 f = fsub2(x, fsub2(t, kRound));
  float2 p = ffma2(make_float2(c3, c3), f, make_float2(c2, c2));
  p = ffma2(p, f, make_float2(c1, c1));
  p = ffma2(p, f, make_float2(c0, c0));
  // t's bits are 0x4B400000 + j: shifted left by 23 only j remains, in the exponent field
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// three-input maximum (one instruction)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// pack two fp32 into bf16x2 (round to nearest even); `lo` lands in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// E4M3 cast of two fp32 values (round to nearest even, saturating at +-448),
// returned as the bf16x2 pair of the same values, and `h2` = the same pair as
// f16x2.  E4M3 -> f16x2 is exact and every non-zero E4M3 value (2^-9 .. 448) is
// an f16 normal whose 7 lowest mantissa bits are zero, so h2 >> 3 holds each
// value's sign, exponent field and top 7 mantissa bits in bf16 position; read as
// bf16 that is the value times 2^(15-127), and one exact bf16x2 multiply by 2^112
// restores it (zero stays zero).  Inputs must be >= 0.
__device__ __forceinline__ uint32_t e4m3_round_bf16x2(float lo, float hi, uint32_t& h2) {
  uint16_t e;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(e) : "f"(hi), "f"(lo));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(e));
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(h2 >> 3), "r"(0x77807780u));
  return r;
}
// Non-zero flags of an f16x2 pair of E4M3 values, added into an f16x2 counter:
// a non-zero value is >= 2^-9, so 2^10 times it saturates to 1.0; zero stays 0.
// Each half counts exactly up to 2048.
__device__ __forceinline__ uint32_t count_nonzero_f16x2(uint32_t h2, uint32_t acc) {
  uint32_t f, r;
  asm("mul.rn.sat.f16x2 %0, %1, %2;" : "=r"(f) : "r"(h2), "r"(0x64006400u));
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(f), "r"(acc));
  return r;
}
__device__ __forceinline__ uint32_t f16x2_sum_u32(uint32_t h2) {
  const __half2 v = *reinterpret_cast<const __half2*>(&h2);
  return static_cast<uint32_t>(__low2float(v) + __high2float(v));
}

// Wait used only on teardown paths: bounded by time, ignores the abort flag.
// Inlined: an out-of-line copy cannot be shared by warps whose register
// budgets differ (setmaxnreg).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

}  // namespace fa
