/*
 * libattn.h -- C ABI of a B200 (sm_100a) fused exact attention library.
 *
 * The operation is exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T + mask) V
 *
 * as stated by the standard_attention listing of "4.5 注意力优化实战：从PyTorch到
 * CUDA的完整流程" (第一步 §1): Q, K, V of shape (batch, heads, seq_len, head_dim),
 * scores scaled once, masked entries set to -inf, a row softmax, then a product
 * with V.  It is computed as one fused, tiled pass with the running-max /
 * running-sum ("online softmax") recurrence of the same page (第三步 §1) and of the
 * codechina FlashAttention article (§3.2), so the [N, N] score matrix never
 * reaches device memory.  The forward pass also saves, per query row, the
 * natural-log logsumexp of the masked scaled scores; the backward pass uses it to
 * recompute the probabilities ("4.5 注意力优化实战" 第四步 §2: the backward needs the
 * softmax normaliser kept from the forward).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Element types: q, k, v, o, dout, dq, dk, dv are bf16 (2 bytes, IEEE-style
 *   bfloat16); lse is fp32.  Accumulation is fp32.
 * - head_dim d must be 64 or 128 (anything else returns ATTN_ERR_UNSUPPORTED).
 * - scale must be finite and > 0 (typically 1/sqrt(d)).
 * - Dense layout (cu_seqlens == NULL): tensors are contiguous [B, H, N, d];
 *   lse is [B, H, N]; key_keep is [B, N].  N >= 1 is arbitrary.
 * - Packed variable-length layout (cu_seqlens != NULL): B is the number of
 *   sequences, N is an upper bound on every sequence length, cu_seqlens is a
 *   DEVICE int32 array of B+1 non-decreasing offsets starting at 0; tensors are
 *   token-major [total, H, d] with total = cu_seqlens[B]; lse is [total, H];
 *   key_keep is [total].  Causal indices are local to each sequence.
 *   The tile loader needs the token count on the host: the *_varlen entry
 *   points take it as `total_tokens`; attn_fwd / attn_fwd_masked / attn_bwd
 *   called with a non-NULL cu_seqlens assume total_tokens = B*N, i.e. the packed
 *   buffers must then be allocated for B*N token rows (rows past
 *   cu_seqlens[B] are read as padding but never written).
 * - Causal masking: key j is visible to query i iff j <= i (lower triangle,
 *   equal query/key lengths; "Profiling in PyTorch (part 3)", math backend
 *   section, tril mask).
 * - key_keep (nullable, DEVICE uint8): 1 = the key may be attended, 0 = masked
 *   for every query.  A query row that sees no key at all gets O = 0 and
 *   lse = -inf (never NaN), as the _safe_softmax discussion of the same page
 *   asks; its gradients are 0 and it contributes nothing to dK/dV.
 * - Ownership: every pointer is caller-owned DEVICE memory (except where noted);
 *   the library allocates nothing per call, so calls on different streams are
 *   independent.  (The kernels that claim their work units at run time -- tile
 *   masks, packed sequences, very large backward problems -- take one of 1,024
 *   library-owned counter pairs per launch, round-robin, and return it to zero when
 *   they finish; a device runs at most 128 kernels at once.)  Base pointers must
 *   be 16-byte aligned.
 * - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   Every compute call is asynchronous on that stream.
 * - Errors: a non-OK code returned from a call means nothing was launched
 *   (argument errors) or a launch failed (ATTN_ERR_CUDA).  Faults detected on the
 *   device (a bounded wait that expired) are reported by attn_status().  After a
 *   non-OK status the outputs are unspecified.
 */
#ifndef LIBATTN_H
#define LIBATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad scale       */
    ATTN_ERR_UNSUPPORTED = 2, /* head_dim not 64/128, or device is not sm_100      */
    ATTN_ERR_MISALIGNED = 3,  /* a base pointer is not 16-byte aligned             */
    ATTN_ERR_WORKSPACE = 4,   /* backward workspace missing or too small           */
    ATTN_ERR_CUDA = 5,        /* a CUDA runtime/driver call or launch failed       */
    ATTN_ERR_TIMEOUT = 6,     /* a device-side bounded wait expired (attn_status)  */
    ATTN_ERR_DEBUG_CHECK = 7  /* a consistency check of the debug library failed   */
} attn_status_t;

/*
 * Forward pass without a key mask.
 *   q, k, v : inputs (bf16), layout per the conventions above.
 *   o       : output (bf16), same layout as q.
 *   lse     : output (fp32), natural-log logsumexp per query row; -inf for rows
 *             that see no key.
 *   B, H, N, d, scale, is_causal, cu_seqlens : as above (cu_seqlens nullable).
 * Returns an attn_status_t code.
 */
ATTN_API int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int H, int N, int d, float scale, int is_causal,
             const int32_t *cu_seqlens, void *stream);

/* Forward pass with an optional per-key padding mask (key_keep, nullable). */
ATTN_API int attn_fwd_masked(const void *q, const void *k, const void *v, void *o, float *lse,
                    int B, int H, int N, int d, float scale, int is_causal,
                    const int32_t *cu_seqlens, const uint8_t *key_keep, void *stream);

/*
 * Bytes of device workspace attn_bwd needs for these sizes (for packed inputs,
 * pass the same B and N as to attn_bwd; the bound B*N >= total is used): two
 * fp32 terms per query row and head, plus the fp32 dQ accumulator (d per query
 * row and head).  Returns 0 for invalid sizes.
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass.  Recomputes the probabilities from q, k and the forward's lse,
 * and writes the input gradients:
 *   dV = P^T dO,  dS = P o (dO V^T - rowsum(dO o O)),  dQ = scale dS K,
 *   dK = scale dS^T Q.
 *   o, lse     : the forward's outputs for the same inputs and masking.
 *   dout       : upstream gradient dL/dO (bf16, layout of o).
 *   dq, dk, dv : outputs (bf16, layout of q).
 *   workspace  : caller-owned device memory of at least
 *                attn_bwd_workspace_bytes(B, H, N, d) bytes, 256-byte aligned;
 *                its contents are scratch and need no initialisation.
 * One pass per 128-key tile computes every product of the method once; the
 * contributions of the key tiles to dQ are summed in an fp32 accumulator in the
 * workspace (fp32 accumulation, "4.5 注意力优化实战" 第四步 §2 backward).  Their
 * order of arrival depends on scheduling, so dq may differ between calls in its
 * last bits; attn_bwd_deterministic gives bit-identical results.
 * Returns an attn_status_t code.
 */
ATTN_API int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
             const void *dout, void *dq, void *dk, void *dv,
             int B, int H, int N, int d, float scale, int is_causal,
             const int32_t *cu_seqlens, const uint8_t *key_keep,
             void *workspace, size_t workspace_bytes, void *stream);

/*
 * The same backward computed in an order that does not depend on scheduling, so
 * that repeated calls on the same inputs give bit-identical dq, dk and dv: dK/dV
 * in one pass per 128-key tile, dQ in a separate pass per 128-row query tile
 * ("4.5 注意力优化实战：从PyTorch到CUDA的完整流程", 第四步 §2: dQ sweeps all key/value
 * blocks), with no atomics.  Arguments as attn_bwd; the workspace needs at least
 * attn_bwd_deterministic_workspace_bytes(B, H, N, d) bytes (two fp32 terms per
 * query row and head; attn_bwd_workspace_bytes is always enough).
 */
ATTN_API size_t attn_bwd_deterministic_workspace_bytes(int B, int H, int N, int d);
ATTN_API int attn_bwd_deterministic(const void *q, const void *k, const void *v, const void *o,
                                    const float *lse, const void *dout, void *dq, void *dk, void *dv,
                                    int B, int H, int N, int d, float scale, int is_causal,
                                    const int32_t *cu_seqlens, const uint8_t *key_keep,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Packed variable-length forward with an exact token count.
 *   num_seqs     : number of sequences (cu_seqlens has num_seqs+1 entries)
 *   total_tokens : rows of the packed tensors (== cu_seqlens[num_seqs]); the
 *                  tile loader never reads past this row
 *   max_seqlen   : upper bound on every sequence length (grid sizing)
 *   key_keep     : nullable, [total_tokens] uint8
 * Other arguments as for attn_fwd_masked.
 */
ATTN_API int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                    int num_seqs, int total_tokens, int max_seqlen, int H, int d, float scale,
                    int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep,
                    void *stream);

/* Workspace bytes for attn_bwd_varlen. Returns 0 for invalid sizes. */
ATTN_API size_t attn_bwd_varlen_workspace_bytes(int total_tokens, int H, int d);

/* Packed variable-length backward with an exact token count (see attn_fwd_varlen). */
ATTN_API int attn_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const float *lse,
                    const void *dout, void *dq, void *dk, void *dv,
                    int num_seqs, int total_tokens, int max_seqlen, int H, int d, float scale,
                    int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * One kernel of one of the two backward algorithms; lets a caller time or schedule
 * them separately, and gives the packed layout its deterministic backward.
 * Deterministic backward (attn_bwd_deterministic launches phases 0, 1, 2 in order):
 *   phase 0 : per-row terms D_i = rowsum(dO o O) and lse2 = lse*log2(e), in
 *             `workspace`
 *   phase 1 : dK and dV (one pass per 128-key tile over the query tiles)
 *   phase 2 : dQ (one pass per 128-row query tile over the key tiles)
 *   Phases 1 and 2 both read only the inputs and phase 0's terms, so after phase 0
 *   they may run in either order (or concurrently on two streams).  The workspace
 *   needs at least attn_bwd_deterministic_workspace_bytes bytes (for the packed
 *   layout with B = 1, N = total_tokens).
 * Single-pass backward (attn_bwd / attn_bwd_varlen launch phases 3, 4, 5 in order):
 *   phase 3 : the terms of phase 0, and zeroes the fp32 dQ accumulator
 *   phase 4 : dK, dV and the dQ accumulator (one pass per 128-key tile)
 *   phase 5 : dq = bf16(scale * accumulator)
 *   The workspace needs at least attn_bwd_workspace_bytes (dense) or
 *   attn_bwd_varlen_workspace_bytes (packed) bytes.
 * Phases must run in order on the same workspace and stream.  Other arguments as
 * attn_bwd_varlen; for the dense layout pass cu_seqlens = NULL, num_seqs = B,
 * max_seqlen = N and total_tokens = 0.
 */
ATTN_API int attn_bwd_phase(int phase, const void *q, const void *k, const void *v, const void *o,
                            const float *lse, const void *dout, void *dq, void *dk, void *dv,
                            int num_seqs, int total_tokens, int max_seqlen, int H, int d, float scale,
                            int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Block-sparse attention (codechina FlashAttention article, §7.1 variant algorithms,
 * Block-Sparse FlashAttention: only the important pairs are computed, a sparsity
 * pattern combined with the tiling).  Dense layout only, as attn_fwd / attn_bwd
 * with cu_seqlens = NULL and no key mask, plus:
 *   block_mask  device array of uint8 [H][nb][nb], nb = ceil(N / 128), shared by
 *               the B sequences.  Entry [h][i][j] == 0 leaves the pair (query rows
 *               128 i .. 128 i + 127, keys 128 j .. 128 j + 127) of head h out:
 *               those key/value tiles are never loaded or multiplied for those
 *               rows and their scores count as -inf.  Any nonzero value keeps the
 *               pair.  It combines with is_causal (a score must pass both).  A query
 *               row left with no key at all gets O = 0, lse = -inf and contributes
 *               no gradient; key rows that no query reaches get dK = dV = 0.
 *               Must not be NULL (ATTN_ERR_INVALID_ARG).  Owned by the caller, read
 *               during the call's kernels only.
 *   N <= 8192 (nb <= 64), else ATTN_ERR_UNSUPPORTED.
 * The backward takes the same workspace as attn_bwd (attn_bwd_workspace_bytes).
 */
ATTN_API int attn_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse,
                                  int B, int H, int N, int d, float scale, int is_causal,
                                  const uint8_t *block_mask, void *stream);
ATTN_API int attn_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o,
                                  const float *lse, const void *dout, void *dq, void *dk, void *dv,
                                  int B, int H, int N, int d, float scale, int is_causal,
                                  const uint8_t *block_mask, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * FP8 forward ("4.5 注意力优化实战：从PyTorch到CUDA的完整流程" / codechina
 * FlashAttention article §9, future directions: mixed precision with FP8 matrix
 * products and higher-precision accumulation).  The products Q K^T and P V run on
 * 8-bit floating-point operands with fp32 accumulation; the result is the same
 * attention as attn_fwd of the dequantised inputs, up to the rounding below.
 *   q, k, v  : DEVICE e4m3 codes (1 byte each: sign, 4 exponent bits with bias 7,
 *              3 mantissa bits; no infinities, 0x7F / 0xFF are NaN, largest
 *              finite 448), dense contiguous [B, H, N, d].
 *   q_scale, k_scale, v_scale : per-tensor dequantisation factors (finite, > 0):
 *              the element value is decode(code) * scale.
 *   o        : output (bf16) [B, H, N, d];  lse : output (fp32) [B, H, N], as for
 *              attn_fwd (natural-log logsumexp of the scaled dequantised scores).
 *   scale, is_causal : as for attn_fwd (dense layout, no key mask).
 * d must be 64 or 128 (ATTN_ERR_UNSUPPORTED otherwise).  Nothing is allocated and no
 * workspace is needed.  Rounding beyond attn_fwd's: the probabilities enter P V as
 * e4m3 (half an e4m3 step: 2^-4 relative, or 2^-10 absolute below 2^-6, on the
 * kernel's scale, where the row sum is at least 1), after exponentials accurate to
 * 1.1e-4 relative; the row sums and lse use the unrounded fp32 probabilities.
 */
ATTN_API int attn_fwd_fp8(const void *q, const void *k, const void *v, float q_scale, float k_scale,
                          float v_scale, void *o, float *lse, int B, int H, int N, int d, float scale,
                          int is_causal, void *stream);

/*
 * FP8 forward with a per-key padding mask (key_keep, nullable DEVICE uint8 [B, N],
 * as for attn_fwd_masked), dense layout.  Other arguments as attn_fwd_fp8.
 */
ATTN_API int attn_fwd_fp8_masked(const void *q, const void *k, const void *v, float q_scale, float k_scale,
                                 float v_scale, void *o, float *lse, int B, int H, int N, int d, float scale,
                                 int is_causal, const uint8_t *key_keep, void *stream);

/*
 * FP8 forward on the packed variable-length layout: q, k, v are e4m3 codes
 * [total_tokens, H, d], o is bf16 [total_tokens, H, d], lse fp32 [total_tokens, H];
 * num_seqs, total_tokens, max_seqlen, cu_seqlens (DEVICE int32, must not be NULL)
 * and key_keep (nullable, [total_tokens]) as for attn_fwd_varlen.  Other arguments
 * as attn_fwd_fp8.
 */
ATTN_API int attn_fwd_fp8_varlen(const void *q, const void *k, const void *v, float q_scale, float k_scale,
                                 float v_scale, void *o, float *lse, int num_seqs, int total_tokens, int max_seqlen,
                                 int H, int d, float scale, int is_causal, const int32_t *cu_seqlens,
                                 const uint8_t *key_keep, void *stream);

/*
 * FP8 forward with a block-sparse tile mask: attn_fwd_fp8's e4m3 operands, scales and
 * rounding combined with attn_fwd_blocksparse's tile mask (codechina FlashAttention
 * article, §7.1 Block-Sparse FlashAttention and §9 FP8).  Dense layout, no key mask.
 *   block_mask  DEVICE uint8 [H][nb][nb], nb = ceil(N / 128), as for
 *               attn_fwd_blocksparse (must not be NULL: ATTN_ERR_INVALID_ARG); a
 *               query row left with no key gets O = 0 and lse = -inf.
 *   N <= 8192, else ATTN_ERR_UNSUPPORTED.  Other arguments as attn_fwd_fp8.
 * Nothing is allocated and no workspace is needed.
 */
ATTN_API int attn_fwd_fp8_blocksparse(const void *q, const void *k, const void *v, float q_scale, float k_scale,
                                      float v_scale, void *o, float *lse, int B, int H, int N, int d, float scale,
                                      int is_causal, const uint8_t *block_mask, void *stream);

/* Size of the library-owned scratch array that attn_bwd_noalloc uses (8 MiB). */
#define ATTN_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * attn_bwd without a workspace argument, for callers that cannot allocate device
 * memory themselves: code running with a fixed memory budget or inside another
 * framework's allocator that forbids raw device allocations, or code that must
 * not allocate once it has started (no counterpart in the attention pages: this
 * is a deployment convenience, not part of the method).
 *
 * It runs the deterministic backward (attn_bwd_deterministic), whose scratch (two
 * fp32 terms per query row and head) lives instead in a fixed array of
 * ATTN_NOALLOC_SCRATCH_BYTES inside the library, one copy per GPU that loads the
 * library, kept until the process exits.  Nothing is allocated per call.
 * Arguments and layouts are those of attn_bwd (with cu_seqlens != NULL the
 * packed buffers must span B*N token rows).
 *   - The sizes may need at most ATTN_NOALLOC_SCRATCH_BYTES of scratch, i.e.
 *     attn_bwd_deterministic_workspace_bytes(B, H, N, d) <=
 *     ATTN_NOALLOC_SCRATCH_BYTES (B*H*N <= 1,048,576); larger sizes return
 *     ATTN_ERR_WORKSPACE without launching anything.
 *   - The first call on a device looks up that device's copy of the array (with
 *     the device current); make that first call before any stream capture.
 *   - Every call shares the array, which keeps the last call's contents.  Nothing
 *     in it needs to start at zero (each call writes every term it reads), but
 *     two calls whose kernels overlap on the GPU (different streams, no ordering
 *     between them) race on it.
 */
ATTN_API int attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                              const float *lse, const void *dout, void *dq, void *dk, void *dv,
                              int B, int H, int N, int d, float scale, int is_causal,
                              const int32_t *cu_seqlens, const uint8_t *key_keep, void *stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of the
 * current device: ATTN_OK, or ATTN_ERR_TIMEOUT if a kernel's bounded wait
 * expired since the last call, ATTN_ERR_UNSUPPORTED if a kernel found its shared
 * memory laid out in a way it cannot run with (and did nothing),
 * ATTN_ERR_DEBUG_CHECK if a pipeline consistency check of the debug library failed
 * (see attn_debug_checks), or ATTN_ERR_CUDA if synchronisation failed.
 */
ATTN_API int attn_status(void *stream);

/* Static, human-readable text for a status code (never NULL). */
ATTN_API const char *attn_strerror(int code);

/*
 * Sets the device-side wait limit in milliseconds for later launches from this
 * process (default 4000).  A kernel whose wait on a pipeline barrier exceeds the
 * limit stops, records ATTN_ERR_TIMEOUT and returns.  ms <= 0 restores the
 * default.  Returns the previous value.
 */
ATTN_API int attn_set_wait_limit_ms(int ms);

/*
 * Test hook for the failure-detection path.  For later launches from this
 * process, each CTA's tile loader skips one pipeline load: in the forward the
 * K/V stage load number `load_index` (counting the K and V tile loads of one CTA
 * from 0), in the backward the query-side load (Q and dO of one query tile)
 * number `load_index` of the dK/dV and of the dQ kernel.  That slot never fills,
 * the consumer's bounded wait expires, every kernel stops cleanly and
 * attn_status() reports ATTN_ERR_TIMEOUT.  -1 (the default) disables it.
 * Returns the previous value.  Nothing faults: all waits are time-limited.
 */
ATTN_API int attn_debug_skip_load(int load_index);

/*
 * Test hook for the exponential that the d = 64 and e4m3 forward kernels take from
 * the FMA pipe for part of their scores (a cubic in f = x - rint(x) on [-1/2, 1/2]
 * times 2^rint(x), with x clamped to -127 first).  Writes y[i] = that kernel's
 * 2^x[i] for i < n, on `stream`; x and y are DEVICE float arrays of n elements,
 * 16-byte aligned.  n must be even and > 0 (the kernels evaluate pairs).  Exposed
 * so that tests can hold the function to its stated accuracy: relative error
 * at most 1.02e-4 where 2^x is a normal float, exactly +0 for x <= -127 and for
 * -inf, exactly 2^x at integer x.  Returns an attn_status_t code.
 */
ATTN_API int attn_debug_ex2_poly(const float *x, float *y, long long n, void *stream);

/*
 * Test hook for the banded unit order.  When the data of the (sequence, head) slices
 * far exceeds the L2 cache, the single-pass backward (Q, dO and the fp32 dQ
 * accumulator beyond 512 MB) and the packed and block-sparse forwards (K and V
 * beyond 256 MB) walk their units in bands of slices that fit about half of the L2
 * cache, claiming units at run time.  For later launches from this process,
 * slices > 0 forces bands of that many slices (at most B*H) at any size, so that
 * tests can run those kernels on small problems; 0 (the default) restores the
 * automatic choice.  The results do not depend on the order (the backward's dQ up
 * to the order of its fp32 additions).  Returns the previous value.
 */
ATTN_API int attn_debug_force_band(int slices);

/*
 * 1 in the debug library (libattn_debug.so, built from the same sources with
 * LIBATTN_DEBUG=1), 0 in the release library.  The debug library runs the same kernels
 * with pipeline consistency checks; a failed check records ATTN_ERR_DEBUG_CHECK in the
 * status word (attn_status) and stops the kernel the way an expired wait does, never
 * with a trap or an assert.  The checks:
 *   - every bounded mbarrier wait: once phase k of a barrier is seen complete, phase
 *     k+1 must still be open (a producer two phases ahead of a consumer would make the
 *     parity protocol misread the phase; every kernel);
 *   - forward: each K/V ring fill carries a tag {unit rank, key tile, fill number}
 *     written by the TMA producer, which the MMA issuer compares with its own walk when
 *     the fill lands; at exit the producer, issuer and softmax warps must agree on the
 *     units, fills and S phases they processed;
 *   - single-pass backward: each Q stage fill carries a tag {unit rank, query tile, pair
 *     number} from the loader, checked by the issuer; at exit the loader, issuer, math
 *     and dQ-drain warps must agree on the units and tile pairs they processed.
 * Results are identical to the release library's.
 */
ATTN_API int attn_debug_checks(void);

/*
 * Test hook for the debug library's ring-tag check.  For later launches from this
 * process, the forward's TMA producer in every CTA writes a wrong tag for its K/V ring
 * fill number `fill_index` (counting the K and V tile loads of one CTA from 0), and the
 * single-pass backward's loader for its Q stage fill number `fill_index` (the CTA's
 * tile pairs, from 0); the issuer's check then fails, the kernel stops cleanly and
 * attn_status() reports ATTN_ERR_DEBUG_CHECK.  No effect in the release library, which writes no tags.  -1
 * (the default) disables it.  Returns the previous value.
 */
ATTN_API int attn_debug_corrupt_tag(int fill_index);

#ifdef __cplusplus
}
#endif

#endif /* LIBATTN_H */
