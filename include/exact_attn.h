/*
 * exact_attn.h -- C ABI of the B200 (sm_100a) exact-attention library.
 *
 * The library computes exact scaled-dot-product attention the IO-aware way:
 *   O = softmax(scale * Q K^T [+ causal mask]) V,   LSE_i = ln sum_j exp(scale * q_i . k_j)
 * with Q/K/V tiles staged on chip and the score and probability matrices never
 * written to device memory, as described in "Describe Flash Attention at a
 * high level" (mantramindai), section "The two ideas" (tiling and online
 * softmax), and "How FlashAttention Speeds Up the Attention Layer"
 * (hassanahmed.net), the tiling and online-softmax paragraphs. The result is
 * the same as the plain definition up to floating-point rounding
 * (mantramindai, "Follow-up questions to expect", first question).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library
 *     never allocates, frees or keeps them past the call.
 *   - Tensors are dense and row-major: Q, O are [B, H, Nq, d]; K, V are
 *     [B, H, Nkv, d]; LSE is [B, H, Nq]. Q, K, V, O are bfloat16 (passed as
 *     void*) except where an entry point says otherwise (attn_fwd_fp8 reads
 *     e4m3 Q, K, V); LSE, split partials and workspaces are fp32.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL means the legacy default stream). It returns after enqueueing.
 *   - Argument errors are reported synchronously, before anything is launched:
 *     ATTN_ERR_INVALID_ARG (null pointer, non-positive size, size overflow),
 *     ATTN_ERR_UNSUPPORTED (head dim other than 64 or 128), ATTN_ERR_ALIGNMENT
 *     (a bf16 tensor not 16-byte aligned, an fp32 tensor not 4-byte aligned).
 *     No silent fallback exists: an input the kernels do not handle is refused.
 *   - Errors seen while launching return ATTN_ERR_CUDA. Errors inside a kernel
 *     (a pipeline wait that gave up after its time limit) are recorded in a
 *     device status word and reported by attn_status().
 *   - Causal masking is bottom-right aligned: key j is visible to query i iff
 *     j <= i + (Nkv - Nq). A query row with no visible key gets O = 0 and
 *     LSE = -inf.
 *   - LSE is the natural logarithm of the sum of exp over the visible scaled
 *     scores.
 */
#ifndef EXACT_ATTN_B200_H
#define EXACT_ATTN_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,
    ATTN_ERR_UNSUPPORTED = 2,
    ATTN_ERR_ALIGNMENT = 3,
    ATTN_ERR_CUDA = 4,
    ATTN_ERR_TIMEOUT = 5,
    ATTN_ERR_SCRATCH_LIMIT = 6,
    ATTN_ERR_BAD_INDEX = 7,
    ATTN_ERR_INDEX_CHECK = 8
} attn_status_t;

/* Version of this ABI (bumped on any incompatible change). */
int attn_abi_version(void);

/*
 * Prefill forward: O and LSE for Nq query rows against Nkv keys per (b, h).
 *
 * Defines: the fused attention kernel of "flashattention-memory-bound"
 * (appliedaiprep), "A strong answer" (QK^T, softmax and .V fused in one kernel,
 * tiles kept on chip), with the online-softmax recurrence of mantramindai
 * "The two ideas" (running max m and sum l; earlier partial output rescaled by
 * exp(m_old - m_new)). The per-row LSE is emitted so that a later merge or a
 * backward pass can use it.
 *
 *   q   bf16 [B, H, Nq, d]      (read)
 *   k   bf16 [B, H, Nkv, d]     (read)
 *   v   bf16 [B, H, Nkv, d]     (read)
 *   o   bf16 [B, H, Nq, d]      (written; rounded to nearest even)
 *   lse fp32 [B, H, Nq]         (written)
 *   d in {64, 128}; B, H, Nq, Nkv >= 1; causal 0 or 1; scale finite (usually
 *   1/sqrt(d)). Any Nq, Nkv is accepted; tails of a 128-row tile are masked.
 *
 *   Work is dealt to one persistent CTA per SM. When the K and V of all heads
 *   exceed 192 MB, the CTAs take their work units from a counter in device
 *   memory owned by the library (one of 64 entries, chosen round robin per
 *   call and returned to zero by the launch itself), in an order that keeps a
 *   few heads' K/V in L2. Two launches that run at the same time use
 *   different entries unless 64 further launches start while the first still
 *   runs; such launches would share an entry and give wrong results. The
 *   environment variable EXACT_ATTN_FWD_SCHEDULE=static|dynamic, read at
 *   every call, forces one deal or the other; the result is bit-identical.
 */
attn_status_t attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int H, int Nq, int Nkv, int d, int causal, float scale,
                       void *stream);

/*
 * Prefill forward on 8-bit inputs: the same O and LSE as attn_fwd for the
 * values x = descale * code, with Q, K and V given as e4m3 codes (OCP FP8
 * E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
 * 0x7F/0xFF NaN) and one fp32 descale factor per (b, h) for each of them.
 *
 * Defines: the FP8 path the pages name for FlashAttention-3 ("Describe Flash
 * Attention at a high level" (mantramindai), section "Versions";
 * "How FlashAttention Speeds Up the Attention Layer" (hassanahmed.net), the
 * FlashAttention-3 paragraph). The pages give no format or scaling; this
 * library reads them as e4m3 inputs with per-head descale factors, both
 * products on the 8-bit tensor-core path (kind::f8f6f4), and P rounded to e4m3
 * for the P V product (O is accumulated in fp32 and returned as bf16).
 *
 *   q                 e4m3 [B, H, Nq, d]      (read; one byte per element)
 *   k, v              e4m3 [B, H, Nkv, d]     (read)
 *   q/k/v_descale     fp32 [B, H]             (read; device memory; finite)
 *   o                 bf16 [B, H, Nq, d]      (written)
 *   lse               fp32 [B, H, Nq]         (written; natural log, as attn_fwd)
 *   d in {64, 128} (ATTN_ERR_UNSUPPORTED otherwise); causal, scale and the
 *   size limits and the work deal (K/V measured in bytes) as attn_fwd; q, k, v,
 *   o 16-byte aligned, the rest 4-byte.
 */
attn_status_t attn_fwd_fp8(const void *q, const void *k, const void *v, const float *q_descale,
                           const float *k_descale, const float *v_descale, void *o, float *lse,
                           int B, int H, int Nq, int Nkv, int d, int causal, float scale,
                           void *stream);

/*
 * Split-KV decode, step 1: per-chunk partials for one query row per (b, h).
 *
 * Defines: the decode method of "Describe Flash Attention at a high level"
 * (mantramindai), "Follow-up questions to expect", last question: with one
 * query row, parallelism comes from splitting the KV sequence across thread
 * blocks. The keys are cut into num_splits chunks of L = ceil(Nkv / num_splits)
 * consecutive keys (the last chunk shorter; trailing chunks may be empty).
 * Chunk c yields the exact attention of the row restricted to its keys,
 * normalised within the chunk, and that chunk's LSE.
 *
 *   q        bf16 [B, H, 1, d]        (read)
 *   k, v     bf16 [B, H, Nkv, d]      (read)
 *   o_part   fp32 [B, H, num_splits, d]   (written; an empty chunk gives 0)
 *   lse_part fp32 [B, H, num_splits]      (written; an empty chunk gives -inf)
 *   d in {64, 128}; 1 <= num_splits <= 65535. No mask (decode sees every key).
 */
attn_status_t attn_decode_partials(const void *q, const void *k, const void *v,
                                   float *o_part, float *lse_part, int B, int H, int Nkv,
                                   int d, float scale, int num_splits, void *stream);

/*
 * Split-KV decode, step 2: merge per-chunk partials with the max-and-sum trick
 * (mantramindai, "Follow-up questions to expect", last question):
 *   M = max_c lse_c;  W = sum_c exp(lse_c - M);  LSE = M + ln W;
 *   O = sum_c exp(lse_c - M) / W * O_c     (all chunks empty: O = 0, LSE = -inf)
 *
 *   o_part   fp32 [B, H, S, d]   (read)
 *   lse_part fp32 [B, H, S]      (read)
 *   o        bf16 [B, H, 1, d]   (written)
 *   lse      fp32 [B, H, 1]      (written)
 *   d in {64, 128}; 1 <= S <= 65535.
 */
attn_status_t attn_lse_merge(const float *o_part, const float *lse_part, void *o, float *lse,
                             int B, int H, int S, int d, void *stream);

/*
 * Split-KV decode across GPUs, step 2: the same merge over partials gathered
 * from R ranks, each of which computed S chunks of its own slice of the KV
 * sequence (the decode split of mantramindai, "Follow-up questions to expect",
 * last question, carried from thread blocks to GPUs: every rank holds a
 * contiguous shard of the keys, runs attn_decode_partials on it, and the
 * ranks' partials are all-gathered, rank after rank, into one buffer).
 *
 *   o_part   fp32 [R, B, H, S, d]   (read; rank r's attn_decode_partials output
 *                                    at offset r * B * H * S * d)
 *   lse_part fp32 [R, B, H, S]      (read)
 *   o        bf16 [B, H, 1, d], lse fp32 [B, H, 1]   (written)
 *   d in {64, 128}; 1 <= S, R <= 65535; S * R <= 2^24. The result does not
 *   depend on how the keys were split (up to rounding); empty chunks (lse =
 *   -inf) have weight 0. With R = 1 this is attn_lse_merge.
 */
attn_status_t attn_lse_merge_gathered(const float *o_part, const float *lse_part, void *o,
                                      float *lse, int R, int B, int H, int S, int d,
                                      void *stream);

/*
 * Bytes of caller-provided workspace attn_decode_splitkv needs for the
 * partials: B*H*num_splits*(d + 1)*4, rounded up to 256. Returns 0 for
 * invalid sizes.
 */
size_t attn_decode_workspace_bytes(int B, int H, int d, int num_splits);

/*
 * Split-KV decode, both steps: attn_decode_partials into `workspace`, then
 * attn_lse_merge into o and lse, enqueued in that order on `stream`.
 *
 *   workspace  device memory of at least attn_decode_workspace_bytes(...)
 *              bytes, 256-byte aligned, owned by the caller; its contents on
 *              entry do not matter and on return are unspecified. Two calls
 *              that run at the same time must not share one workspace.
 *   Other arguments as for attn_decode_partials and attn_lse_merge.
 */
attn_status_t attn_decode_splitkv(const void *q, const void *k, const void *v, void *o,
                                  float *lse, int B, int H, int Nkv, int d, float scale,
                                  int num_splits, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * Paged-KV split-KV decode, step 1: per-chunk partials over a paged KV cache.
 *
 * Defines: the "paged variants for decode" the serving systems use
 * (mantramindai, "Versions", last paragraph; PagedAttention in appliedaiprep,
 * "What interviewers probe next"). The pages give no layout; this library's:
 * the cache holds num_pages physical pages of page_size tokens for every head,
 *   k_cache, v_cache  bf16 [num_pages, H, page_size, d]   (read)
 * token j of sequence b is in physical page block_table[b][j / page_size],
 * slot j % page_size;
 *   block_table  int32 [B, max_pages_per_seq]           (read)
 *   seq_lens     int32 [B], tokens cached per sequence   (read)
 *   q            bf16 [B, H, 1, d]                       (read)
 *   o_part, lse_part as for attn_decode_partials, with chunks of
 *   ceil(seq_lens[b] / num_splits) tokens per sequence.
 * page_size is a power of two in [16, 1024]. A sequence of length 0 yields
 * empty chunks (O = 0, LSE = -inf after the merge). Table entries outside
 * [0, num_pages) and lengths outside [0, max_pages_per_seq * page_size] are
 * never dereferenced: the keys concerned are skipped and attn_status()
 * reports ATTN_ERR_BAD_INDEX.
 */
attn_status_t attn_decode_paged_partials(const void *q, const void *k_cache, const void *v_cache,
                                         const int *block_table, const int *seq_lens,
                                         float *o_part, float *lse_part, int B, int H, int d,
                                         int page_size, int max_pages_per_seq, int num_pages,
                                         float scale, int num_splits, void *stream);

/*
 * Paged-KV split-KV decode, both steps: attn_decode_paged_partials into
 * `workspace` (attn_decode_workspace_bytes(B, H, d, num_splits) bytes, 256-byte
 * aligned, caller-owned), then attn_lse_merge into o [B, H, 1, d] (bf16) and
 * lse [B, H, 1] (fp32).
 */
attn_status_t attn_decode_paged(const void *q, const void *k_cache, const void *v_cache,
                                const int *block_table, const int *seq_lens, void *o, float *lse,
                                int B, int H, int d, int page_size, int max_pages_per_seq,
                                int num_pages, float scale, int num_splits, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Split-KV decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point; it exists for library
 * users. It computes exactly what attn_decode_splitkv computes, with the same
 * arguments except the workspace: the partials go to a fixed 32 MiB array
 * owned by this library (one per GPU that loads it, held until the process
 * exits). It is meant for callers that may not call cudaMalloc or cannot hand
 * over a device buffer, e.g. code inside an allocator's callbacks or a plugin
 * whose host framework owns all device memory.
 *
 *   Every argument is checked before anything is launched, with the codes
 *   attn_decode_splitkv returns (null q, k, v, o or lse, B * H > 65535 or
 *   num_splits > 65535: ATTN_ERR_INVALID_ARG; misaligned pointers:
 *   ATTN_ERR_ALIGNMENT). Returns ATTN_ERR_SCRATCH_LIMIT, also without
 *   launching, when the partials (attn_decode_workspace_bytes(B, H, d,
 *   num_splits) bytes) exceed 32 MiB.
 *   All calls on a device share the array: calls that overlap on the GPU race
 *   and must be serialised by the caller. The array keeps the last call's
 *   contents; none of it needs to start at zero.
 *   The first call in each CUDA context looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   The address is cached with the context's unique id, so a context that is
 *   destroyed and created again (e.g. after cudaDeviceReset) is looked up
 *   afresh.
 */
attn_status_t attn_decode_splitkv_noalloc(const void *q, const void *k, const void *v, void *o,
                                          float *lse, int B, int H, int Nkv, int d, float scale,
                                          int num_splits, void *stream);

/*
 * Backward pass: bytes of device workspace attn_bwd needs, or 0 if the
 * arguments are invalid. Layout (owned by the caller, 256-byte aligned), with
 * NqPad = Nq rounded up to a multiple of 64: fp32 D [B, H, NqPad] and fp32
 * LSE * log2(e) [B, H, NqPad], each padded to 256 bytes, 256 bytes for the
 * three maxima that set attn_bwd_deterministic's accumulator scale, then the
 * dQ accumulator: fp32 [B, H, Nq, d] for attn_bwd, int64 fixed point for
 * attn_bwd_deterministic (the size covers the int64 form). Nothing in it
 * needs initialising.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int Nq, int d);

/*
 * Backward pass: dQ, dK, dV of L = sum(dO * O) for the attention attn_fwd
 * computes, recomputing the score and probability tiles from Q, K and the
 * forward pass's LSE instead of storing P.
 *
 * Defines: "Describe Flash Attention at a high level" (mantramindai), "The two
 * ideas", item 3 (recompute score tiles in the backward pass instead of storing
 * P) and "How FlashAttention Speeds Up the Attention Layer" (hassanahmed.net),
 * the training paragraph after the online softmax; the gradients are those of
 * standard attention (mantramindai, "Follow-up questions to expect", first
 * question). With P = exp(scale * Q K^T - LSE) (masked entries 0):
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P o (dP - D),
 *   dQ = scale * dS K,  dK = scale * dS^T Q.
 *
 *   q, o, dout  bf16 [B, H, Nq, d]    (read; o is the forward output)
 *   k, v        bf16 [B, H, Nkv, d]   (read)
 *   lse         fp32 [B, H, Nq]       (read; the forward pass's LSE)
 *   dq          bf16 [B, H, Nq, d]    (written)
 *   dk, dv      bf16 [B, H, Nkv, d]   (written)
 *   workspace   device, >= attn_bwd_workspace_bytes(B, H, Nq, d) bytes,
 *               256-byte aligned; overwritten.
 *   d in {64, 128}; causal 0 or 1 (bottom-right, as attn_fwd); B * H <= 65535.
 *   A query row whose LSE is -inf (it sees no key) contributes nothing.
 *   Three kernels run on `stream` in order: D, LSE * log2(e) and zeroing of
 *   the accumulator; the main kernel (one CTA per 128-key block and head,
 *   64-row query blocks); and the dQ conversion. dQ is summed with fp32 atomic
 *   adds, so its last bits may vary from run to run; dK and dV do not
 *   (attn_bwd_deterministic gives bit-identical dQ too).
 */
attn_status_t attn_bwd(const void *q, const void *k, const void *v, const void *o,
                       const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                       int H, int Nq, int Nkv, int d, int causal, float scale, void *workspace,
                       size_t workspace_bytes, void *stream);

/*
 * attn_bwd whose dQ, like dK and dV, is the same bits on every run: same
 * arguments, workspace and errors. dQ is summed in a fixed-point int64
 * accumulator (multiples of 2^-F) with integer atomic adds, which are exact in
 * any order; F is chosen per call so that no partial sum can overflow, from
 * the bound |sum_j dS_ij K_jc| <= 2 max|K| max_i ||dO_i|| max_j ||V_j|| (times
 * 2 for bf16 rounding), computed by an extra kernel over K and V and by the
 * first kernel over dO (a 12-byte memset of the workspace comes first).
 * Inputs must be finite. The integer atomics cost more than fp32 ones (about
 * 1.5x the backward's time at 8K).
 */
attn_status_t attn_bwd_deterministic(const void *q, const void *k, const void *v, const void *o,
                                     const void *dout, const float *lse, void *dq, void *dk,
                                     void *dv, int B, int H, int Nq, int Nkv, int d, int causal,
                                     float scale, void *workspace, size_t workspace_bytes,
                                     void *stream);

/*
 * Synchronises `stream`, then returns and clears the device status word:
 * ATTN_ERR_TIMEOUT if a kernel's pipeline wait gave up since the last call
 * (its outputs are then invalid), ATTN_ERR_BAD_INDEX if a paged decode met an
 * out-of-range block-table entry or length (those keys were skipped),
 * ATTN_ERR_INDEX_CHECK if, in the debug build of the library (compiled with
 * -DATTN_DEBUG), a kernel computed a global-memory index outside its tensor
 * (the access was skipped; the normal build does not check),
 * ATTN_ERR_CUDA if the stream reported an error, ATTN_OK otherwise.
 */
attn_status_t attn_status(void *stream);

/*
 * Diagnostic for the failure-detection path: enqueues a one-block kernel that
 * waits on a barrier nothing ever completes, through the same bounded wait the
 * pipeline kernels use, with a limit of `limit_us` microseconds
 * (1 <= limit_us <= 1000000). The kernel gives up, records a timeout and
 * exits; the next attn_status() on the stream returns ATTN_ERR_TIMEOUT, and the
 * CUDA context stays usable. No counterpart on the pages (library testing aid).
 */
attn_status_t attn_selftest_wait_timeout(unsigned limit_us, void *stream);

/* A static, human-readable description of a status code. */
const char *attn_strerror(attn_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTN_B200_H */
