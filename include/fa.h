/*
 * fa.h -- C ABI of libfa.so: exact IO-aware tiled attention on NVIDIA B200 (sm_100a).
 *
 * The operation is O = softmax(scale * Q K^T) V, computed tile by tile with the
 * online-softmax recurrence so that the N x N score matrix never reaches device
 * memory ("flash-attention-trading-models", sections "El algoritmo de atencion
 * flash" and "La recurrencia de softmax en linea"; "FlashAttention (IT)",
 * sections "Tiling" and "Calcolo online del Softmax").  Alongside O every entry
 * point writes the per-row logsumexp, the O(N) statistic that the backward pass
 * needs ("flash-attention-trading-models", section "Pase hacia atras").
 *
 * Conventions shared by every entry point
 *  - Layout: q, k, v, o, dO, dq, dk, dv are contiguous row-major [B, H, N, d]
 *    device arrays (the (batch, heads, seq, head_dim) layout of the pages'
 *    framework example); lse is a contiguous [B, H, N] float32 device array.
 *    LSE is the natural-log logsumexp of the scaled scores of each query row.
 *  - Sizes: B >= 1, H >= 1, N >= 1, d in {64, 128}; every entry point but
 *    fa_fwd_f32 (d = 64 only) also takes d = 256 ("FlashAttention (IT)",
 *    "FlashAttention-2 (2023)").  Limits of the launches: N <= 2^30,
 *    B*H < 2^31, B*H*ceil(N/128) < 2^31 (twice that for the d = 256 backward,
 *    which runs two CTAs per key tile) and B*H*N*d < 2^40; element offsets
 *    are 64-bit, so any size that fits in device memory within these is taken.
 *  - scale: the softmax scale (usually 1/sqrt(d)); finite and > 0.
 *  - causal != 0: query i attends to keys j <= i (square, top-left aligned);
 *    tiles that lie entirely in the future are skipped, never loaded.
 *  - Alignment: every device pointer 16-byte aligned, except lse (4-byte:
 *    the kernels write it one fp32 scalar at a time).
 *  - Ownership: the caller allocates and owns every buffer.  The library never
 *    allocates, frees or synchronises (fa_check_status synchronises the stream
 *    it is given); all work is enqueued on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).
 *  - Errors: invalid arguments are rejected before anything is launched and
 *    return a non-zero fa_status; there is no fallback path.  A failed launch
 *    returns FA_ERR_CUDA (fa_last_cuda_error() gives the cudaError_t).  Device
 *    pipelines that stall past a bound record FA_ERR_TIMEOUT in a device status
 *    word that fa_check_status() reads after the caller's work has finished.
 *  - Thread safety: entry points may be called concurrently from host threads,
 *    with these shared parts: fa_last_cuda_error() is per host thread; the
 *    timeout status word is per device and shared by every caller in the
 *    process, so fa_check_status() reports (and clears) a timeout raised by any
 *    thread's kernels on the current device; fa_bwd_noalloc calls share one
 *    scratch array per device and must not overlap on the GPU.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad scale/S/kv_order */
  FA_ERR_UNSUPPORTED = 2, /* a head dim the entry point does not take (64 and 128
                             everywhere but fa_fwd_f32, which takes 64; 256 where
                             the entry point's comment says so), sizes over the
                             limits above, B*H_kv > 65535 (fa_decode) or
                             B*H > 65535 (fa_fp8_quantize), more than 16 query heads
                             per key/value head (fa_decode), or a workspace larger
                             than FA_BWD_NOALLOC_MAX_BYTES (fa_bwd_noalloc) */
  FA_ERR_ALIGNMENT = 3,   /* a pointer without the alignment the conventions require */
  FA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  FA_ERR_TIMEOUT = 5,     /* a device-side wait gave up (reported by fa_check_status) */
  FA_ERR_CHECK = 6        /* debug builds only (compiled with FA_DEBUG): a device-side
                             argument check of a TMA copy, tensor-memory access or MMA
                             failed and the operation was skipped (reported by
                             fa_check_status; bits 8-15 of the raw word name the check) */
} fa_status;

/* Forward, bf16 in/out, fp32 accumulation on the tensor cores.
 * q, k, v: bf16 [B,H,N,d]; o: bf16 [B,H,N,d] (written); lse: fp32 [B,H,N] (written). */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d, int causal,
           float scale, void* stream);

/* Forward, fp32 in/out: the same algorithm on the tf32 tensor-core path.  Q and
 * K are rounded to tf32 (round to nearest even) in shared memory before S = Q K^T,
 * so the scores carry no truncation bias; V and P enter P V as the tensor core
 * reads them (their low 13 mantissa bits are ignored).  fp32 accumulation and
 * fp32 softmax.  d = 64 only.  q, k, v, o: fp32 [B,H,N,d]; lse: fp32 [B,H,N]. */
int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N, int d,
               int causal, float scale, void* stream);

/* Bytes of device workspace fa_bwd needs for these sizes (fp32 row term D and
 * the fp32 dQ accumulator), rounded up to 256 bytes. */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/* Backward of fa_fwd: recomputes the scores tile by tile from q, k and the saved
 * lse, and writes dq, dk, dv (bf16 [B,H,N,d]) for the upstream gradient dO
 * ("flash-attention-trading-models", section "Pase hacia atras").
 * o and lse must be the outputs of fa_fwd on the same q, k, v, causal, scale.
 * workspace: caller-owned device buffer of at least fa_bwd_workspace_bytes()
 * bytes, 256-byte aligned; its contents on entry do not matter. */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
           void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* workspace,
           size_t workspace_bytes, void* stream);

/* Backward for callers that cannot allocate device memory: some embedders run
 * under an allocator they do not own (a framework's caching pool, a process
 * whose memory budget is fixed up front) or in code paths where a cudaMalloc
 * would synchronise the device or is forbidden outright, so they cannot supply
 * fa_bwd's workspace.  This variant takes the same arguments as fa_bwd minus the
 * workspace and uses a scratch array that the library itself defines in device
 * memory: FA_BWD_NOALLOC_MAX_BYTES (32 MiB), reserved on every GPU that loads the
 * library for as long as it stays loaded.  It calls no allocation routine.
 *  - Sizes whose workspace (fa_bwd_workspace_bytes) exceeds that maximum are
 *    rejected with FA_ERR_UNSUPPORTED before anything is launched.
 *  - The first call on a device looks up that device's address of the array
 *    (cudaGetSymbolAddress, with the device current) and caches it with the id
 *    of the CUDA context; a call in another context (after a device reset, for
 *    one) looks it up again.  Make the first call on a device before any stream
 *    capture.
 *  - All calls on a device share the one array and it keeps the previous call's
 *    contents; each call rewrites every part it reads (the first of its kernels
 *    rewrites the row statistics and zeroes the dQ accumulator).  Calls whose
 *    work overlaps on the GPU (different streams, or different host threads)
 *    race on the array: serialise them.
 * The pages have no counterpart to this entry point; results are those of
 * fa_bwd on the same inputs. */
#define FA_BWD_NOALLOC_MAX_BYTES (32u << 20)
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                   void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale, void* stream);

/* Forward with the probability tile P cast to FP8 E4M3 before the P.V product
 * ("P-Cast precision in FP8 attention", sections 1-2): P' = E4M3(S * p) with
 * round-to-nearest-even and saturation at 448, accumulated against V, and the
 * epilogue divides by S * l, where the running sum l is taken from the
 * unquantised p.  The running max used for p includes the current tile.
 *   S        static scale, finite and > 0 (the page recommends 256);
 *   kv_order 0 visits key tiles 0 -> N, 1 visits them N -> 0;
 *   stats    NULL, or a device array of 4 uint64 that the kernel ADDS to:
 *            [0] sink P' that flushed to zero, [1] sink P counted,
 *            [2] non-sink P' that flushed to zero, [3] non-sink P counted,
 *            where a key is a sink when its index is < n_sink (n_sink >= 0).
 * Key tiles are 128 keys at d = 64 and 128 and 64 keys at d = 256: the running
 * max moves once per tile, so the tile size is part of the result.
 * q, k, v, o: bf16 [B,H,N,d]; lse: fp32 [B,H,N]; d in {64, 128, 256}. */
int fa_fwd_fp8p(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                int causal, float scale, float S, int kv_order, unsigned long long* stats, int n_sink, void* stream);

/* Grouped-query / multi-query attention ("FlashAttention for Scalable Vector
 * Architectures", "Metodologia": a key/value head shared by several query heads;
 * "FlashAttention (IT)", "FlashAttention-2 (2023)": Multi-Query Attention).
 * q, o: [B,H,N,d]; k, v: [B,H_kv,N,d] with H a multiple of H_kv; query head h
 * uses key/value head h / (H / H_kv).  H_kv = 1 is multi-query attention,
 * H_kv = H is fa_fwd.  lse: [B,H,N].  Other conventions as fa_fwd. */
int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N, int d,
               int causal, float scale, void* stream);

/* Backward of fa_fwd_gqa: dq [B,H,N,d]; dk, dv [B,H_kv,N,d] are the sums of the
 * gradients over the query heads of each group (accumulated inside the kernel,
 * no extra pass).  workspace: fa_bwd_workspace_bytes(B, H, N, d).  Other
 * conventions as fa_bwd. */
int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
               void* dk, void* dv, int B, int H, int H_kv, int N, int d, int causal, float scale, void* workspace,
               size_t workspace_bytes, void* stream);

/* One decoding step: for each query head a single new query row attends to all
 * N cached keys of its key/value head (the last row of causal attention,
 * "flash-attention-trading-models", "El algoritmo de atencion flash").  Bound by
 * reading the cache once: split over the key sequence with a log-sum-exp merge
 * of the chunks, K/V streamed by TMA, the per-chunk arithmetic on warp-level
 * tensor-core MMAs; the g = H / H_kv query heads of a key/value head are served
 * from one read of it (g <= 16).  Two launches on `stream` (split, combine).
 * q, o: bf16 [B,H,d]; k, v: bf16 [B,H_kv,N,d]; lse: fp32 [B,H]; d in {64, 128, 256}.
 * workspace: caller-owned, >= fa_decode_workspace_bytes(), 16-byte aligned. */
size_t fa_decode_workspace_bytes(int B, int H, int H_kv, int N, int d);
int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N, int d,
              float scale, void* workspace, size_t workspace_bytes, void* stream);

/* FP8 operands for fa_fwd_fp8 ("flash-attention-trading-models", section "FA3",
 * item 3: FP8 with incoherent processing).  Quantises bf16 q, k, v [B,H,N,d]
 * to E4M3 codes (round to nearest even, saturating):
 *  - q and k, one scale per block of 128 rows of each (b,h), after the optional
 *    rotation x -> x diag(signs) H / sqrt(d) (H the Sylvester Walsh-Hadamard
 *    matrix; signs = NULL skips it): the caller draws the d random signs (+-1,
 *    fp32 device array).  The rotation leaves q k^T unchanged and spreads
 *    outliers, which is what lowers the quantisation error;
 *  - v, one scale per head, never rotated.
 * Outputs (caller-owned device memory): q8, k8, v8 uint8 [B,H,N,d] E4M3 codes;
 * sq, sk fp32 [B,H,ceil(N/128)] and sv fp32 [B,H] dequantisation scales
 * (block amax / 448, 1 for an all-zero block).  d in {64, 128, 256}. */
int fa_fp8_quantize(const void* q, const void* k, const void* v, const float* signs, void* q8, void* k8, void* v8,
                    float* sq, float* sk, float* sv, int B, int H, int N, int d, void* stream);

/* Forward on E4M3 operands from fa_fp8_quantize: S = (q8 k8^T)(sq sk) scale on
 * the kind::f8f6f4 tensor cores, the online softmax in fp32, P' = E4M3(S_p p)
 * (static scale S_p, key-tile order kv_order as in fa_fwd_fp8p), O += P' v8 on
 * the tensor cores, and O = acc * sv / (S_p * l) -> bf16 [B,H,N,d]; lse fp32
 * [B,H,N] of the quantised scores.  d in {64, 128, 256} (64-byte E4M3 rows at
 * d = 64 are staged with the 64-byte swizzle; at d = 256 the key tiles are 64
 * keys, so the running max of the P-cast moves once per 64 keys). */
int fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq, const float* sk, const float* sv,
               void* o, float* lse, int B, int H, int N, int d, int causal, float scale, float S, int kv_order,
               void* stream);

/* Grouped-query FP8 ("FlashAttention (IT)", "FlashAttention-2 (2023)": Multi-Query
 * Attention, with the FP8 operands of "flash-attention-trading-models", "FA3"):
 * k, v, k8, v8 [B,H_kv,N,d], sk [B,H_kv,ceil(N/128)], sv [B,H_kv]; q, q8, o
 * [B,H,N,d], sq [B,H,ceil(N/128)], lse [B,H,N]; H a multiple of H_kv, query
 * head h reads key/value head h / (H / H_kv).  Each key/value head is
 * quantised once, so the codes and scales equal those fa_fp8_quantize gives
 * for k, v repeated over the group.  Other conventions as fa_fp8_quantize and
 * fa_fwd_fp8 (which are these calls with H_kv = H). */
int fa_fp8_quantize_gqa(const void* q, const void* k, const void* v, const float* signs, void* q8, void* k8,
                        void* v8, float* sq, float* sk, float* sv, int B, int H, int H_kv, int N, int d, void* stream);
int fa_fwd_fp8_gqa(const void* q8, const void* k8, const void* v8, const float* sq, const float* sk,
                   const float* sv, void* o, float* lse, int B, int H, int H_kv, int N, int d, int causal, float scale,
                   float S, int kv_order, void* stream);

/* Human-readable name of an fa_status code. */
const char* fa_status_string(int status);

/* The cudaError_t of the last FA_ERR_CUDA returned on this host thread. */
int fa_last_cuda_error(void);

/* Reads the device status word after the work on `stream` has finished (a copy
 * enqueued on `stream`, then cudaStreamSynchronize(stream); NULL = the legacy
 * default stream, which also waits for the other blocking streams), and clears
 * it: FA_OK, or FA_ERR_TIMEOUT if a bounded wait in a kernel of this library gave
 * up on the current device since the last call (FA_ERR_CUDA if a copy or the
 * synchronisation failed).  The word is per device, not per stream: a timeout
 * raised by work on another stream is reported too, once that work is done. */
int fa_check_status(void* stream);

/* Self-test of the exponential that part of the d = 64 softmax computes on the
 * FMA pipe instead of the MUFU (range reduction x = j + f, |f| <= 1/2, then a
 * degree-3 minimax polynomial for 2^f fitted by the Remez exchange algorithm):
 * y_fma[i] = that exponential of x[i], y_mufu[i] = ex2.approx.ftz(x[i]), for
 * n float32 values in device memory (4-byte aligned), x[i] <= 127.  Enqueued on
 * `stream`.  Lets a test bound the polynomial's error against the hardware. */
int fa_exp2_selftest(const float* x, float* y_fma, float* y_mufu, int n, void* stream);

/* Failure-path self-test: launches a one-block kernel whose bounded wait on a
 * barrier that nothing signals gives up after limit_us microseconds (1 .. 10^7),
 * records FA_ERR_TIMEOUT in the device status word and returns; the CUDA context
 * stays usable.  fa_check_status() then reports FA_ERR_TIMEOUT.  Every wait in
 * the attention kernels is bounded the same way (at 2 s). */
int fa_watchdog_selftest(unsigned int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
