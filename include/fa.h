/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa_sm100.so).
 *
 * The library computes exact scaled-dot-product attention and its gradient
 * without ever writing the N x N score or probability matrices to device
 * memory:
 *
 *   forward   O = softmax(scale * Q K^T [+ causal mask]) V,
 *             LSE_i = m_i + ln(l_i)   (m: row max of the scaled scores,
 *                                      l: row sum of exp(score - m))
 *   backward  dV = P^T dO, dP = dO V^T, dS = P o (dP - rowsum(dO o O)),
 *             dQ = scale dS K, dK = scale dS^T Q, with P recomputed from Q, K
 *             and the saved LSE.
 *
 * Passages that define the operations (web pages on FlashAttention):
 *   - "FlashAttention-2: Faster Attention with Better Parallelism and Work
 *     Partitioning" review page: core-algorithm answer, section 1 (S = QK^T,
 *     P = softmax(S), O = PV), section 2 (1) tiling with B_r x B_c blocks,
 *     (2) forward pass with a running max m and running sum l, (3) backward
 *     pass recomputing softmax from the saved (m, l) and forming dQ, dK, dV;
 *     the FLOP answer (forward 4 N^2 d, backward 2.5x forward; O(N) extra
 *     memory for the softmax statistics).
 *   - "IO-4 FlashAttention (Memory IO optimisation based attention
 *     acceleration)" note: the scaled form softmax(QK^T / sqrt(d_k)) V;
 *     section 4 online softmax; section 5 O(n) memory.
 *   - "[LLM] Flash Attention" blog post: "Recomputation" (S, P recomputed
 *     in the backward instead of stored).
 * Readings where the pages are silent or garbled: the causal mask hides key
 * j from query i when j > i; the saved statistic is the single natural-log
 * LSE; the page's dS formula is read as the row-wise softmax Jacobian and
 * the scale is applied to dQ and dK (chain rule through S = scale Q K^T).
 *
 * Conventions for every entry point
 *   Layout     q, k, v, o, dO, dq, dk, dv: contiguous [B, H, N, d] row-major
 *              (d fastest); lse: contiguous [B, H, N] fp32, natural log.
 *   Pointers   device pointers, each 16-byte aligned; the caller owns all
 *              memory.  The library never allocates device memory.  It keeps
 *              one 4-byte device status word per process (a file-scope
 *              device variable) and the fixed scratch array of
 *              fa_backward_noalloc (FA_NOALLOC_SCRATCH_BYTES, also
 *              file-scope), nothing else.
 *   Streams    `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *              default stream).  Every call is asynchronous on that stream;
 *              no call synchronises the host except fa_device_status.
 *   Errors     argument errors are reported before anything is launched and
 *              no output is touched; launch errors map to FA_ERR_CUDA.
 *              Kernels never trap: a device-side wait that runs past its time
 *              limit records the fact in the status word, the kernel returns,
 *              and fa_device_status reports FA_ERR_DEVICE_TIMEOUT.
 *   Outputs    are overwritten, never accumulated into.
 *   Devices    sm_100a (B200) only; any other device gives FA_ERR_UNSUPPORTED.
 */
#ifndef FA_SM100_H_
#define FA_SM100_H_

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1,     /* null pointer, B/H/N < 1, non-finite or non-positive scale */
  FA_ERR_UNSUPPORTED = -2,     /* head dim or dtype not built, or not an sm_100 device */
  FA_ERR_MISALIGNED = -3,      /* a pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = -4,       /* workspace null, too small or not 256-byte aligned */
  FA_ERR_CUDA = -5,            /* a CUDA runtime/driver call failed (see fa_last_cuda_error) */
  FA_ERR_DEVICE_TIMEOUT = -6   /* a kernel's bounded wait ran out (reported by fa_device_status) */
} fa_status;

typedef enum {
  FA_BF16 = 0,   /* bf16 storage, fp32 accumulation on the tensor cores */
  FA_FP32 = 1    /* fp32 storage and fp32 FMA arithmetic (small-case path) */
} fa_dtype;

/*
 * fa_forward -- bf16 forward.
 *   q, k, v  [B, H, N, d] bf16 inputs.
 *   o        [B, H, N, d] bf16 output (the normalised attention output).
 *   lse      [B, H, N] fp32 output, LSE_i = ln sum_j exp(scale q_i.k_j) over
 *            the keys query i sees.
 *   d        head dimension: 64, 80 or 128.
 *   N        sequence length, any N >= 1 (ragged tails are masked).
 *   scale    score multiplier (1/sqrt(d) for standard attention), > 0.
 *   causal   0: every query sees every key; 1: query i sees keys j <= i.
 */
FA_API fa_status fa_forward(const void* q, const void* k, const void* v, void* o,
                     float* lse, int B, int H, int N, int d, float scale,
                     int causal, void* stream);

/*
 * fa_forward_ex -- as fa_forward with an explicit storage dtype.
 *   FA_BF16: identical to fa_forward.
 *   FA_FP32: q, k, v, o are fp32; any d in [1, 128]; fp32 arithmetic
 *            throughout (no tensor-core rounding), for accuracy checks.
 */
FA_API fa_status fa_forward_ex(const void* q, const void* k, const void* v, void* o,
                        float* lse, int B, int H, int N, int d, float scale,
                        int causal, fa_dtype dtype, void* stream);

/*
 * fa_backward_workspace_size -- bytes of device scratch fa_backward needs:
 * two fp32 row vectors per head padded to a multiple of 128 rows
 * (D = rowsum(dO o O) and the base-2 LSE), each rounded up to 256 bytes:
 * 2 * round256(4 * B * H * ceil(N / 128) * 128).  Linear in N (no N x N
 * buffer); independent of d.  Returns 0 for arguments that fa_backward would
 * reject.
 */
FA_API size_t fa_backward_workspace_size(int B, int H, int N, int d);

/*
 * fa_backward -- bf16 backward.
 *   q, k, v, o, dO  [B, H, N, d] bf16 inputs (o is the forward output).
 *   lse             [B, H, N] fp32, the forward's LSE.
 *   dq, dk, dv      [B, H, N, d] bf16 outputs.
 *   workspace       device scratch of at least
 *                   fa_backward_workspace_size(B, H, N, d) bytes, 256-byte
 *                   aligned, owned by the caller; its contents on entry do
 *                   not matter and are clobbered.  Two calls that overlap on
 *                   the GPU must not share one workspace.
 *   Other arguments as in fa_forward (same scale and causal as the forward).
 * Launches two kernels in stream order: the dQ kernel (which also writes the
 * row statistics D = rowsum(dO o O) and the base-2 LSE into the workspace)
 * and the dK/dV kernel.  dQ is computed by its own kernel (it recomputes S
 * and dP per query tile), so no atomics are used and the result is bitwise
 * reproducible.
 */
FA_API fa_status fa_backward(const void* q, const void* k, const void* v,
                      const void* o, const void* dO, const float* lse,
                      void* dq, void* dk, void* dv,
                      int B, int H, int N, int d, float scale, int causal,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_backward_ex -- as fa_backward with an explicit storage dtype.
 *   FA_FP32: all tensors fp32, any d in [1, 128], fp32 arithmetic.
 */
FA_API fa_status fa_backward_ex(const void* q, const void* k, const void* v,
                         const void* o, const void* dO, const float* lse,
                         void* dq, void* dk, void* dv,
                         int B, int H, int N, int d, float scale, int causal,
                         void* workspace, size_t workspace_bytes,
                         fa_dtype dtype, void* stream);

/*
 * fa_forward_blocksparse -- bf16 forward of block-sparse attention: the
 * combination of FlashAttention-2 with a block sparsity pattern described in
 * "FlashAttention-2: Faster Attention with Better Parallelism and Work
 * Partitioning" (review page), answer on combining it with sparse / hybrid
 * attention, section 3 (1) "Sparse FlashAttention" (a pattern defined on
 * blocks matched to the kernel's tiles; only the important blocks are
 * processed), and the limitations answer, section 2 (3) (dense global plus
 * sparse local attention).
 *   block_mask  device pointer, uint8 [mask_heads, nt, nt] with
 *               nt = ceil(N / 128): byte (h, I, J) != 0 lets query rows
 *               128 I .. 128 I + 127 see keys 128 J .. 128 J + 127 of head h.
 *               Key tiles a query tile may not see are never loaded.
 *   mask_heads  1 (one mask for every head) or H (head h of every batch
 *               entry uses mask h).
 *   causal      applied on top of the mask (query i sees keys j <= i).
 * A query row that sees no key at all gets O = 0 and LSE = -inf.  The mask
 * must stay unchanged until the call's kernels have run.  Other arguments and
 * errors as fa_forward; a null block_mask or mask_heads not in {1, H} is
 * FA_ERR_INVALID_ARG.
 */
FA_API fa_status fa_forward_blocksparse(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int H, int N, int d, float scale,
                                        int causal, const unsigned char* block_mask,
                                        int mask_heads, void* stream);

/*
 * fa_backward_blocksparse -- bf16 backward of fa_forward_blocksparse: the
 * gradients of the masked softmax attention (hidden entries have P = 0, so
 * they pass no gradient).  Key tiles no query may see get dK = dV = 0; query
 * rows that see no key get dQ = 0.  Arguments as fa_backward plus the same
 * block_mask / mask_heads as the forward; the workspace is sized by
 * fa_backward_workspace_size.
 */
FA_API fa_status fa_backward_blocksparse(const void* q, const void* k, const void* v,
                                         const void* o, const void* dO, const float* lse,
                                         void* dq, void* dk, void* dv, int B, int H, int N,
                                         int d, float scale, int causal,
                                         const unsigned char* block_mask, int mask_heads,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_forward_splitkv -- bf16 forward for decoding: N_q new queries against a
 * cache of N_k >= 1 keys/values, the key range split across CTAs.  Each
 * (head, query tile pair, key split) computes a partial O and LSE over its
 * keys with the online softmax; a second kernel merges the partials by the
 * same running-max / running-sum rule ("FlashAttention-2: Faster Attention
 * with Better Parallelism and Work Partitioning" review: core-algorithm
 * answer, (2) forward pass step 2, and its answer on FlashAttention's Split-K
 * scheme, where K and V are split across workers whose partial results are
 * combined).  Splitting the keys gives a few-query problem enough parallel
 * work to keep every SM reading K and V.
 *   q, o        [B, H, N_q, d] bf16;  lse [B, H, N_q] fp32 (natural log).
 *   k, v        [B, H, N_k, d] bf16.
 *   causal      0: every query sees every key; 1: the queries are the last
 *               N_q positions: query i sees keys j <= i + (N_k - N_q).  Rows
 *               that see no key (only when N_q > N_k) get O = 0, LSE = -inf.
 *   num_splits  >= 1 key ranges per (head, query tile pair); clamped to the
 *               number of 128-key tiles.  fa_splitkv_default_splits picks one.
 *   workspace   device scratch of fa_splitkv_workspace_size(...) bytes,
 *               256-byte aligned (fp32 partials), owned by the caller;
 *               concurrent calls must not share it.
 * d in {64, 80, 128}.  Errors as fa_forward; FA_ERR_WORKSPACE for a missing,
 * small or misaligned workspace.  Two kernels in stream order.
 */
FA_API fa_status fa_forward_splitkv(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int B, int H, int Nq, int Nk, int d,
                                    float scale, int causal, int num_splits, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Key splits for fa_forward_splitkv that give every SM of the current device
 * about one work item (floor(SMs / items), clamped to 1 .. ceil(N_k / 128));
 * 0 for invalid sizes. */
FA_API int fa_splitkv_default_splits(int B, int H, int Nq, int Nk);

/* Workspace bytes fa_forward_splitkv needs for these sizes and num_splits:
 * fp32 partial O and LSE for every split, each rounded up to 256 bytes;
 * 0 for invalid arguments. */
FA_API size_t fa_splitkv_workspace_size(int B, int H, int Nq, int Nk, int d, int num_splits);

/*
 * fa_backward_noalloc -- the bf16 backward of fa_backward, for callers that
 * cannot allocate device memory or hand over a workspace: code whose device
 * memory is entirely owned by another allocator, plugins and callbacks that
 * receive tensors but cannot reserve scratch, and latency-bound loops that
 * must not call cudaMalloc (it can synchronise the device).  The FlashAttention
 * pages have no counterpart to this entry point; it is a convenience of this
 * library.
 *
 * The scratch comes from a fixed device array of FA_NOALLOC_SCRATCH_BYTES
 * built into the library (held on every GPU that loads it, until the process
 * exits).  Problems whose workspace, fa_backward_workspace_size(B, H, N, d),
 * exceeds that size are rejected with FA_ERR_WORKSPACE before anything runs.
 * All calls on a GPU share the array: each call re-initialises what it needs,
 * but calls whose kernels overlap on the GPU (e.g. on two streams) race.  The
 * first call on each device looks up the array's device address (once, with
 * that device current); make that first call before any stream capture.
 * No device memory is allocated.  Arguments and results are those of
 * fa_backward (bf16, d in {64, 80, 128}).
 */
#define FA_NOALLOC_SCRATCH_BYTES (64u << 20)
FA_API fa_status fa_backward_noalloc(const void* q, const void* k, const void* v,
                              const void* o, const void* dO, const float* lse,
                              void* dq, void* dk, void* dv,
                              int B, int H, int N, int d, float scale, int causal,
                              void* stream);

/*
 * fa_forward_fp8 -- FP8 forward: the attention of fa_forward computed with
 * E4M3 inputs and E4M3 tensor-core matmuls, the extension the
 * "FlashAttention-2: Faster Attention with Better Parallelism and Work
 * Partitioning" review page lists under future work, (5) "FP8 and latest
 * hardware" (FP8 in the matmuls and the softmax), mixed with wider types
 * where accuracy needs them (its auto-tuning answer, section 1 (2)).
 *   q, k, v     E4M3 codes (1 byte each: sign, 4 exponent bits with bias 7,
 *               3 mantissa bits; 0x7F / 0xFF are NaN), [B, H, N, d]
 *               contiguous, 16-byte aligned.
 *   q_descale, k_descale, v_descale
 *               device pointers to one fp32 dequantisation factor each
 *               (element = value(code) * descale); NULL means 1.  Read by
 *               the kernel, so they may be produced on the device (e.g. by
 *               fa_quantize_fp8) without a host synchronisation.
 *   o           bf16 [B, H, N, d]; lse fp32 [B, H, N] (natural log).
 * Both products Q K^T and P V run as E4M3 x E4M3 with fp32 accumulation; the
 * softmax statistics are fp32 and the probabilities are rounded to E4M3
 * before P V (error at most max(2^-4 p, 2^-10) for a probability p taken
 * against the reference max: relative 2^-4 in E4M3's normal range, at most
 * 2^-10 absolute among its subnormals, and values below 2^-10 flush to 0).  The result approximates the
 * exact attention of the dequantised inputs; the rounding of P bounds the
 * difference per element.  d in {64, 80, 128}; scale, causal, stream and
 * errors as fa_forward.
 */
FA_API fa_status fa_forward_fp8(const void* q, const void* k, const void* v,
                                const float* q_descale, const float* k_descale,
                                const float* v_descale, void* o, float* lse,
                                int B, int H, int N, int d, float scale, int causal,
                                void* stream);

/*
 * fa_quantize_fp8 -- per-tensor E4M3 quantisation for fa_forward_fp8's
 * inputs (the pages fix no FP8 scaling; this is the plain per-tensor
 * reading): amax = max |x| over the n elements, codes[e] =
 * RN(x[e] * (448 / amax)) with saturation to +-448, *descale = amax / 448
 * (each quotient and product one fp32 operation rounded to nearest).  When
 * 448 / amax has no finite fp32 value (amax = 0, or amax below about
 * 1.3e-36) the factor and *descale are 1: the codes are x rounded to E4M3 as
 * it is (all such values round to signed zeros).
 *   x        device pointer, n elements of dtype FA_BF16 or FA_FP32,
 *            16-byte aligned.
 *   codes    device pointer, n bytes, 16-byte aligned.
 *   descale  device pointer to one fp32 (4-byte aligned); written on the
 *            stream, so a following fa_forward_fp8 on the same stream can
 *            read it.
 * Non-finite inputs give unspecified codes.  n = 0 or a null pointer is
 * FA_ERR_INVALID_ARG.
 */
FA_API fa_status fa_quantize_fp8(const void* x, fa_dtype dtype, size_t n, void* codes,
                                 float* descale, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
FA_API const char* fa_status_string(fa_status s);

/* The cudaError_t value of the last call that returned FA_ERR_CUDA on this
 * host thread (0 if none). */
FA_API int fa_last_cuda_error(void);

/*
 * fa_device_status -- synchronise the current device, then report whether a
 * kernel of this library recorded a wait timeout since the last reset.
 * Returns FA_OK or FA_ERR_DEVICE_TIMEOUT; *site (if non-NULL) receives the
 * recorded wait-site code (0 when none).  reset != 0 clears the word.
 */
FA_API fa_status fa_device_status(int reset, int* site);

/*
 * fa_set_wait_timeout_ns -- time limit of every device-side wait in kernels
 * launched after this call (default 2e9 ns).  0 restores the default.
 */
FA_API void fa_set_wait_timeout_ns(unsigned long long ns);

/*
 * Key-tile size of the dense bf16 forward (fa_forward, fa_forward_ex with
 * FA_BF16).  The block sizes B_r x B_c of the tiled algorithm are left to be
 * tuned per GPU ("FlashAttention-2: Faster Attention with Better Parallelism
 * and Work Partitioning" review page, implementation-cost answer, section
 * (2), and auto-tuning answer, section 1 (1), which lists candidate sizes).
 * The library has two forward kernels with 128-row query tiles: one with
 * 128-key tiles and one with 64-key tiles and two score buffers per query
 * tile, and a built-in table that picks one from (d, N, causal).
 *
 * fa_set_forward_key_tile(keys): 0 restores the table; 64 or 128 forces that
 * kernel for every later call (a process-wide setting, e.g. for measuring
 * both); anything else is FA_ERR_INVALID_ARG.  Block-sparse and split-KV
 * forwards always use 128-key tiles.
 * fa_forward_key_tile(d, N, causal): the key-tile size the next dense bf16
 * forward of that shape would use (64 or 128), 0 for an unsupported shape.
 */
FA_API fa_status fa_set_forward_key_tile(int keys);
FA_API int fa_forward_key_tile(int d, int N, int causal);

/*
 * fa_selftest_wait_timeout -- failure-detection self test: launches one
 * 32-thread block that waits on a barrier nothing ever completes, under the
 * current time limit; the wait gives up, records its site code (0x7e57) in
 * the status word and the kernel returns.  The caller then reads
 * fa_device_status.  Nothing faults, traps or hangs.
 */
FA_API fa_status fa_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif  /* FA_SM100_H_ */
