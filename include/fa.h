/*
 * fa.h -- C ABI of libfa: exact attention (forward and backward) on B200 (sm_100a).
 *
 * The operation ("第17讲 Tensor Core、HBM、SRAM 与 FlashAttention", §8.1 scaled
 * dot-product attention; §8.2 the tiled flow; §8.3 online softmax):
 *
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 *
 * evaluated tile by tile with an online softmax, so the N x N score and
 * probability matrices never reach device memory.  The forward also writes
 * the per-row log-sum-exp lse_i = ln sum_j exp(scale q_i.k_j) (natural log,
 * over the visible keys), from which the backward recomputes the
 * probabilities instead of storing them ("CS336 Lecture 5 · GPUs, TPUs"
 * notes, section "FlashAttention 解析", item ② on recomputation).
 *
 * Conventions shared by the attention entry points (fa_fwd, fa_fwd_fp8,
 * fa_bwd, fa_bwd_deterministic, fa_bwd_noalloc; fa_decode and fa_gemm state
 * their own shapes):
 *   - Tensors Q, K, V, O, dO, dQ, dK, dV are dense row-major [B, H, N, d]
 *     (d contiguous, then N, then H, then B), bf16 unless stated.  lse and
 *     the backward's D are [B, H, N] fp32.  Queries and keys share length N.
 *   - causal != 0 means query i sees keys j <= i (top-left aligned).
 *   - d must be 64 or 128.  N >= 1, B >= 1, H >= 1, B*H*N*d < 2^31.
 *   - scale must be finite and >= 0 (1/sqrt(d) is the usual choice).
 *   - Device pointers must be 16-byte aligned (lse and workspace: 16 bytes
 *     too).  The caller owns every buffer: the library allocates, frees and
 *     synchronises nothing; all work is enqueued on `stream` (0 = legacy
 *     default stream) of the current device.
 *   - Arguments are validated before anything is launched; on error nothing
 *     is enqueued and a negative fa_status is returned.  No exception ever
 *     crosses the ABI.
 *   - Calls are thread-safe.  Two calls that run concurrently on the GPU must
 *     not share output or workspace buffers.
 *   - Results are deterministic for the forward, dK and dV.  fa_bwd sums
 *     the per-block dQ contributions with fp32 reduce-add copies whose order
 *     varies, so its dQ may differ in the last bits between runs (the pages
 *     note that tiled attention is not bit-identical to the untiled
 *     computation, §8.4 of the first page); fa_bwd_deterministic gives a
 *     run-to-run identical dQ at some cost in speed.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fa_stream_t; /* same type as cudaStream_t */

typedef enum {
  FA_OK = 0,
  FA_ERR_NULL = -1,           /* a required pointer is NULL */
  FA_ERR_SHAPE = -2,          /* B, H or N < 1, a tensor too large, or a decode
                                 shape out of range (Nq, Nk, ld_kv, B*H) */
  FA_ERR_UNSUPPORTED_D = -3,  /* d not in {64, 128} */
  FA_ERR_ALIGN = -4,          /* a pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = -5,      /* workspace smaller than its *_workspace_size */
  FA_ERR_LAUNCH = -6,         /* the CUDA runtime rejected a launch or query */
  FA_ERR_TIMEOUT = -7,        /* a device-side wait gave up (reported later) */
  FA_ERR_DEVICE_ASSERT = -8,  /* a device-side consistency check failed */
  FA_ERR_ARCH = -9,           /* the current device is not sm_100 */
  FA_ERR_ARG = -10,           /* scale negative or not finite; bad grad_dtype */
  FA_ERR_NOALLOC_LIMIT = -11  /* fa_bwd_noalloc: scratch need above its fixed maximum */
} fa_status;

/*
 * Forward.
 *   q, k, v : inputs, bf16 [B,H,N,d], device memory, read only.
 *   o       : output, bf16 [B,H,N,d], device memory, written.
 *   lse     : output, fp32 [B,H,N], device memory, written (natural log).
 * Returns FA_OK once the kernel is enqueued.  Kernel-side failures (a bounded
 * wait that timed out) are latched in a per-device status word that
 * fa_check_device_errors() reads.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int H, int N, int d, float scale, int causal,
           fa_stream_t stream);

/*
 * Forward with FP8 operands: O = softmax(scale * Q K^T [+ causal]) V where
 * Q, K and V are given as E4M3 values with one fp32 dequantisation factor per
 * (b, h) each (the real value is e4m3 * descale).  The low-precision trick
 * of "第17讲 Tensor Core、HBM、SRAM 与 FlashAttention" §4.4 (FP8 on the tensor
 * cores, twice the BF16 rate) applied to both GEMMs: S = Q K^T from E4M3
 * operands with fp32 accumulation, and O += P V with P rounded to E4M3.  O
 * is normalised by the sum of the rounded P, so each output row is a convex
 * combination of V rows; lse uses the unrounded P.  Accuracy is set by the
 * E4M3 rounding of P (relative 2^-4); see the library's design notes.
 *   q, k, v     : E4M3 [B,H,N,d], device, read only; d must be 128.
 *   descale_q,
 *   descale_k,
 *   descale_v   : fp32 [B*H], device, read only (4-byte aligned).
 *   o           : bf16 [B,H,N,d], device, written.
 *   lse         : fp32 [B,H,N], device, written (natural log).
 * Other arguments and errors as fa_fwd; d != 128 gives FA_ERR_UNSUPPORTED_D.
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, const float *descale_q,
               const float *descale_k, const float *descale_v, void *o, float *lse,
               int B, int H, int N, int d, float scale, int causal, fa_stream_t stream);

/*
 * Backward: gradients of L = sum(O * dO) for the forward above.  The
 * formulas are not on the pages (they only say the backward recomputes the
 * probabilities tile by tile); the library computes the exact gradient:
 *     P_ij  = exp(scale q_i.k_j - lse_i)        (0 where masked)
 *     D_i   = sum_c dO_ic O_ic
 *     dV_j  = sum_i P_ij dO_i
 *     dS_ij = P_ij (dO_i.v_j - D_i)
 *     dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
 *   q, k, v, o, dO : bf16 [B,H,N,d], device, read only (o and lse from fa_fwd
 *                    with the same q, k, v, scale and causal).
 *   lse            : fp32 [B,H,N], device, read only.
 *   dq, dk, dv     : outputs [B,H,N,d], device, written; bf16 when
 *                    grad_dtype == 0, fp32 when grad_dtype == 1.
 *   workspace      : device scratch of at least fa_bwd_workspace_size(B,H,N,d)
 *                    bytes, 16-byte aligned, owned by the caller; its contents
 *                    on entry do not matter and on exit are unspecified.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o,
           const void *dO, const float *lse, void *dq, void *dk, void *dv,
           int B, int H, int N, int d, float scale, int causal,
           void *workspace, size_t workspace_bytes, int grad_dtype,
           fa_stream_t stream);

/* Bytes of scratch fa_bwd (and fa_bwd_deterministic) needs: an fp32 dQ
 * accumulator [B,H,N,d], then lse * log2(e) and D = rowsum(dO * O) as fp32
 * [B,H,Npad] with Npad = N rounded up to 128, each rounded up to 256 bytes,
 * then 256 bytes for the work-unit counter of the dynamic scheduler.
 * 0 on invalid shapes. */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Deterministic backward: the same gradients, arguments, layouts, workspace
 * and errors as fa_bwd, but every output bit is reproducible from run to run.
 * fa_bwd sums the per-block dQ contributions with fp32 reduce-add copies in
 * an order that varies; here dK and dV come from the same key-block-major
 * kernel without its dQ part, and a second, query-block-major kernel
 * recomputes P and dS tile by tile in a fixed key order and writes each dQ
 * row once.  It does three more tile multiplications per tile pair than
 * fa_bwd (S and dP are formed twice) but sends no dQ traffic through L2
 * reductions.  Not on the pages, whose only statement on the subject is that
 * tiled attention is not bit-identical to the untiled computation (§8.4 of
 * the first page).
 */
int fa_bwd_deterministic(const void *q, const void *k, const void *v, const void *o,
                         const void *dO, const float *lse, void *dq, void *dk, void *dv,
                         int B, int H, int N, int d, float scale, int causal,
                         void *workspace, size_t workspace_bytes, int grad_dtype,
                         fa_stream_t stream);

/* Human-readable text for an fa_status value (static storage). */
const char *fa_strerror(int status);

/* Synchronises `stream`, then reads and clears the current device's status
 * word that kernels set when a bounded wait gives up or a consistency check
 * fails.  Returns FA_OK, FA_ERR_TIMEOUT, FA_ERR_DEVICE_ASSERT or
 * FA_ERR_LAUNCH (a CUDA error is pending on the device). */
int fa_check_device_errors(fa_stream_t stream);

/* Failure-detection self-test (no counterpart on the pages: a test hook).
 * Enqueues a one-thread kernel whose wait on an mbarrier can never complete;
 * the wait gives up after limit_ms (1..2000) milliseconds exactly as the
 * library's kernels' bounded waits do, latches the timeout bit in the status
 * word and returns, so the next fa_check_device_errors() reports
 * FA_ERR_TIMEOUT and the CUDA context stays usable.  Nothing hangs or
 * faults.  Returns FA_OK once enqueued, FA_ERR_ARG for a limit out of range. */
int fa_selftest_wait_timeout(int limit_ms, fa_stream_t stream);

/* Number of persistent CTAs fa_fwd / fa_bwd launch for a problem on the
 * current device (pass = 0 forward, 1 backward), and the number of work
 * units they share (forward: scheduling items, each one Q tile pair, or
 * for causal problems with an even number >= 8 of tile pairs per head
 * mostly two complementary pairs of one head; backward: K/V blocks);
 * for the harness and its wave-quantization checks.
 * Returns FA_OK or an error status (no launch happens). */
int fa_launch_shape(int pass, int B, int H, int N, int d, int causal,
                    int *ctas, int *work_units);

/* Work-unit schedule of fa_fwd / fa_fwd_fp8 on a device with `sms` SMs (host
 * arithmetic, no device needed).  A head of N queries has P = ceil(N/256)
 * Q tile pairs; a causal pair t costs about 4t + 3 key tiles, so pairs t and
 * P-1-t cost the same together for every t.  When the problem is causal and
 * P is even and >= 8, the first *merged_heads heads are dealt as items of
 * two such complementary pairs (head-major, so running CTAs share a few
 * heads' K and V in L2) and the last R = (P/2) << *tail_shift heads as single
 * pairs, longest first, with *tail_shift the smallest shift giving R * P >=
 * 2 * sms (two rounds of the persistent grid).  Otherwise, and when
 * B*H <= R, every item is one pair (*merged_heads = 0, *tail_shift = 0).  *items = merged_heads * P/2 + (B*H - merged_heads) * P
 * items are dealt to min(*items, sms) CTAs.  B, H, N, sms >= 1 and
 * B*H*P < 2^31, else FA_ERR_SHAPE; FA_ERR_NULL for a NULL output. */
int fa_fwd_schedule(int B, int H, int N, int causal, int sms, int *items,
                    int *merged_heads, int *tail_shift);

/*
 * Decode: attention of Nq new queries per head against a key/value cache
 * ("第17讲 Tensor Core、HBM、SRAM 与 FlashAttention", §9.2 prefill and decode,
 * §9.3 what the KV cache holds; the attention is the §8.1 formula).  The
 * cache of each head is read once, split into chunks of keys handled by
 * separate CTAs; the chunks' partial softmax states (m, l, o) are merged
 * with the online-softmax rescaling of §8.3 by the last CTA of each head.
 *   q           : bf16 [B,H,Nq,d], device, read only; 1 <= Nq <= 8.
 *   k_cache,
 *   v_cache     : bf16 [B,H,ld_kv,d], device, read only; rows 0 .. len_b-1 of
 *                 each head are the cached keys / values of batch b.
 *   o           : bf16 [B,H,Nq,d], device, written.
 *   lse         : fp32 [B,H,Nq], device, written (natural log; -inf for a
 *                 query that sees no key, whose o row is then 0).
 *   cache_lens  : int32 [B], device, read only: len_b, the valid rows of
 *                 batch b (values are clamped to [0, Nk]); NULL means every
 *                 batch has Nk valid rows.
 *   Nk          : the longest valid length, 1 <= Nk <= ld_kv (sets the split).
 *   causal      : the Nq queries are the newest positions: query i sees keys
 *                 j <= len_b - Nq + i.  Without it every valid key is seen.
 *   num_splits  : chunks per head; 0 lets the library choose (wave-quantized
 *                 to the SM count); otherwise it is rounded to whole 64-key
 *                 tiles and capped by the chunk-size limit.
 *   workspace   : device scratch of fa_decode_workspace_size(...) bytes with
 *                 the same B, H, Nq, Nk, d and num_splits, 16-byte aligned,
 *                 owned by the caller (NULL allowed when that size is 0).  Its
 *                 first B*H 32-bit words are per-head counters that must be
 *                 zero before the first call (cudaMemset once); each call
 *                 leaves them zero again.  After FA_ERR_TIMEOUT, zero them
 *                 again.  Calls sharing a workspace must not overlap on the GPU.
 * The result is deterministic: the merge order is fixed.  B*H <= 65535.
 */
size_t fa_decode_workspace_size(int B, int H, int Nq, int Nk, int d, int num_splits);
int fa_decode(const void *q, const void *k_cache, const void *v_cache, void *o,
              float *lse, const int *cache_lens, int B, int H, int Nq, int Nk,
              int ld_kv, int d, float scale, int causal, int num_splits,
              void *workspace, size_t workspace_bytes, fa_stream_t stream);

/* The split fa_decode uses for B*H heads on a device with `sms` SMs that
 * hold `ctas_per_sm` decode CTAs each: *splits chunks of *chunk_keys keys
 * per head (host arithmetic only, no device access).  Among chunk sizes of
 * whole 64-key tiles up to the kernel's limit it picks the one with the
 * fewest waves x (tiles per chunk + 1), ties going to longer chunks. */
int fa_decode_plan(int BH, int Nq, int Nk, int d, int num_splits, int sms,
                   int ctas_per_sm, int *splits, int *chunk_keys);

/*
 * Matrix multiply C = A B: bf16 A [M,K] and B [K,N] (row-major with row
 * strides lda, ldb), fp32 accumulation, bf16 C [M,N] (row stride ldc).  The
 * matrix multiply of the throughput-versus-size curve that "CS336 Lecture 5 ·
 * GPUs, TPUs" opens with (notes, opening goal and the "矩阵谜题" section):
 * 256 x 128 or 256 x 256 output tiles (fa_gemm_tiles), one persistent CTA per
 * SM, so the tile count over the SM count sets the number of rounds (wave
 * quantization).  An operand
 * whose rows are not 16-byte aligned (leading dimension not a multiple of 8
 * elements, or an unaligned base) is first copied into the workspace with an
 * aligned leading dimension, because the tensor-memory copies need aligned
 * rows; that copy is the cost of such sizes.
 *   workspace : device scratch of fa_gemm_workspace_size(A, B, M, N, K, lda,
 *               ldb) bytes (0 when both operands are aligned; NULL allowed
 *               then), 16-byte aligned, owned by the caller.
 * Pointers need only 2-byte alignment.  M, N, K >= 1, lda >= K, ldb >= N,
 * ldc >= N.
 */
size_t fa_gemm_workspace_size(const void *A, const void *B, int M, int N, int K, int lda,
                              int ldb);
int fa_gemm(const void *A, const void *B, void *C, int M, int N, int K, int lda, int ldb,
            int ldc, void *workspace, size_t workspace_bytes, fa_stream_t stream);

/* Output tiling of fa_gemm on a device with `sms` SMs (host arithmetic):
 * tiles are 256 x *tile_n, *tile_n = 256 when ceil(M/256) x ceil(N/256) >= sms
 * (every SM still gets a tile), else 128; *tiles_m x *tiles_n of them. */
int fa_gemm_tiles(int M, int N, int sms, int *tile_n, int *tiles_m, int *tiles_n);

/*
 * Opt-in per-kernel timing with CUDA events (a tracing aid; off by default).
 * After fa_trace_start(), every kernel the library enqueues, on any stream of
 * any device, is bracketed by two CUDA events recorded on its launch stream,
 * until fa_trace_stop().  fa_trace_stop() waits for those events and fills,
 * for each kernel id k < n_kernels, launches[k] and total_ms[k] (summed event
 * durations).  Kernel ids: 0 forward, 1 backward preprocess, 2 backward main,
 * 3 dQ conversion, 4 dQ pass of the deterministic backward, 5 decode,
 * 6 GEMM, 7 GEMM operand packing (fa_trace_kernel_name gives the kernel's
 * name).  The
 * library creates the events on first use and reuses them afterwards; event
 * records add a few microseconds per launch.  fa_trace_start() discards a
 * previous unfinished record.  Launches enqueued on a stream that is being
 * captured into a CUDA graph are bracketed by external event nodes
 * (cudaEventRecordExternal): the graph's replay stamps them, and
 * fa_trace_stop() (called after the replay) reads the last replay's times.
 */
int fa_trace_start(void);
int fa_trace_stop(int n_kernels, int *launches, double *total_ms);
/* The same trace restricted to the kernels whose bit is set in kernel_mask
 * (bit k: kernel id k); the others are launched without events, so a timed
 * region can measure its dominant kernel while adding as few stream
 * commands as possible.  fa_trace_start() is fa_trace_start_mask(~0u). */
int fa_trace_start_mask(unsigned kernel_mask);
const char *fa_trace_kernel_name(int kernel);

/*
 * Backward for callers that cannot allocate device memory.  (No counterpart
 * on the pages: this is a packaging variant of fa_bwd.)  Some callers cannot
 * call cudaMalloc: a plugin inside a host framework that owns every byte of
 * device memory and gives its plugins none, or a latency-critical path where
 * cudaMalloc's implicit device synchronisation is not allowed.  This entry
 * point runs exactly the fa_bwd computation, with the same arguments minus
 * the workspace, but takes its scratch from a fixed array inside the
 * library's device image instead of from the caller.
 *   - Maximum: fa_bwd_workspace_size(B,H,N,d) must not exceed
 *     FA_BWD_NOALLOC_MAX_SCRATCH (32 MiB, e.g. B*H = 64 heads of N = 1024 at
 *     d = 64); larger problems return FA_ERR_NOALLOC_LIMIT before anything is
 *     enqueued.
 *   - The array exists on every GPU that loads the library and is held until
 *     the process exits.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The function allocates and frees nothing.
 *   - All calls on a device share the one array: calls that overlap on the
 *     GPU (different streams, no ordering between them) race and corrupt each
 *     other's results.  Order them on one stream or with events.
 *   - The array keeps the previous call's contents; every part that must
 *     start at zero is cleared by the call itself.
 * Returns FA_OK once the kernels are enqueued, or an fa_status error.
 */
#define FA_BWD_NOALLOC_MAX_SCRATCH ((size_t)32 << 20)
int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                   const void *dO, const float *lse, void *dq, void *dk, void *dv,
                   int B, int H, int N, int d, float scale, int causal,
                   int grad_dtype, fa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
