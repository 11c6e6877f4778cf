/*
 * fa.h -- C ABI of the exact, IO-aware attention library for B200 (sm_100a).
 *
 * The library computes exact scaled dot-product attention
 *     O = softmax(scale * Q K^T + causal mask) V
 * with optional attention dropout, tile by tile with the online-softmax
 * recurrence (running row maximum m_i and denominator l_i, earlier partial
 * sums rescaled when the maximum changes), without ever writing the N x N
 * score or probability matrix to device memory.
 *   - definition of the result: "Flash Attention" glossary (emergent.sh),
 *     section "Why Regular Attention Becomes a Bottleneck"; exactness:
 *     "DL0056 FlashAttention", Answer;
 *   - the recurrence: "DL0056 FlashAttention", Mathematical Formulation;
 *   - tiling / fusion: "FlashAttention" glossary (inferensys.com), Tiling and
 *     Kernel Optimization; "Flash Attention" glossary, How Flash Attention
 *     Works, steps 1-5;
 *   - backward by recomputation from stored per-row outputs: "FlashAttention"
 *     glossary, Recomputation; "Flash Attention" glossary, step 6;
 *   - causal mask and dropout inside the fused kernel: "FlashAttention"
 *     glossary, Causal Masking and Dropout bullets; the dropout pattern is
 *     regenerated, not stored: "Flash Attention" glossary, Key Components.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major [B, H, N, d] (strides H*N*d, N*d, d, 1) --
 *    except for the packed ``_varlen`` calls ([total, H, d]) and the paged
 *    decode cache ([num_pages, page_size, H_kv, d]) -- with 16-bit elements
 *    passed as void*: bfloat16 for fa_fwd / fa_bwd and their stages;
 *    bfloat16 or IEEE fp16 (binary16), as the ``dtype`` argument says, for
 *    every call that takes one.  All tensors of one call share the type.
 *    Per-row statistics (LSE) are fp32 [B, H, N]; every sum inside the
 *    kernels is fp32.
 *  - Every pointer argument is DEVICE memory owned by the caller, 16-byte
 *    aligned.  The library allocates nothing and keeps no per-call state.
 *  - Supported: d in {32, 64, 96, 128} (32 and 96 run on the 64- and
 *    128-column kernels: the columns past d are read as zeros and never
 *    stored); any N >= 1 (a partial last 128-row tile is handled inside the
 *    kernels); B*H*N < 2^31.  Queries and keys may differ
 *    in number (``_qk`` and ``_varlen`` entry points).
 *  - Causal mask with Nq queries and Nk keys: query i sits at key position
 *    i + Nk - Nq (bottom-right alignment; top-left when Nq = Nk) and sees the
 *    keys j <= i + Nk - Nq.  A query row that sees no key (Nk < Nq) gets
 *    O = 0 and LSE = -inf, and contributes nothing to the gradients.
 *  - ``stream`` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call only enqueues work on it and returns; results are
 *    ready when the stream reaches that point.
 *  - Argument errors are detected on the host before anything is enqueued:
 *    nothing is launched and no output is touched.  A failed launch returns
 *    FA_ERR_CUDA.  No entry point exits or aborts the process.
 *  - Device-side pipeline waits are bounded in time.  A wait that gives up
 *    records a flag in a device word and makes the kernel return early; the
 *    outputs of that call are then undefined and fa_last_device_error()
 *    reports FA_ERR_TIMEOUT.
 *  - LSE_i = m_i + ln(l_i) in natural-log units of the scaled scores:
 *    LSE_i = ln(sum_j exp(scale * Q_i . K_j)) over the unmasked j.  Dropout
 *    does not change it.
 *  - Dropout: keep(i, j) <=> u16(seed, b, h, i, j) >= t with
 *    t = round-half-even(p_drop * 65536); u16 comes from Philox4x32-10
 *    (Salmon et al., SC'11) with key (seed mod 2^32, seed >> 32), counter
 *    (j >> 3, i, h, b); key j takes 16 bits of output word (j >> 1) & 3, the
 *    low half for even j and the high half for odd j.  Kept probabilities are
 *    scaled by 1/(1 - p_drop).  p_drop = 0 disables dropout.
 */
#ifndef FA_SM100_H_
#define FA_SM100_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, non-positive size, p_drop outside [0,1), ... */
  FA_ERR_UNSUPPORTED = 2,  /* valid but not implemented: d not in {32,64,96,128}, B*H*N too large */
  FA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed (launch, tensor-map encoding, ...) */
  FA_ERR_TIMEOUT = 4       /* a bounded device-side wait gave up (reported by fa_last_device_error) */
} fa_status;

/* Element type of the 16-bit tensors of an ``_ex`` call. */
typedef enum {
  FA_DTYPE_BF16 = 0, /* bfloat16: 8 exponent bits, 7 stored mantissa bits */
  FA_DTYPE_F16 = 1   /* IEEE binary16: 5 exponent bits, 10 stored mantissa bits */
} fa_dtype;

/*
 * Forward pass.
 *   Q, K, V : in,  bf16 [B, H, N, d]
 *   O       : out, bf16 [B, H, N, d]   O = dropout(softmax(scale*QK^T + mask)) V
 *   LSE     : out, fp32 [B, H, N]      per-row log-sum-exp of the scaled scores
 *   causal  : nonzero -> key j > query i is masked (square, top-left aligned)
 *   scale   : finite score scale, usually 1/sqrt(d)
 *   p_drop  : dropout probability in [0, 1); seed keys the dropout mask
 * Source: the tiled forward ("FlashAttention" glossary, Tiling; "DL0056
 * FlashAttention", Mathematical Formulation; "Flash Attention" glossary, steps
 * 1-5).  O and LSE may not alias the inputs.
 */
fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE,
                 int B, int H, int N, int d, int causal, float scale,
                 float p_drop, uint64_t seed, void* stream);

/*
 * fa_fwd for either 16-bit input type: Q, K, V and O are all of ``dtype``
 * (FA_DTYPE_BF16 gives exactly fa_fwd).  The probabilities fed to the second
 * product are rounded to ``dtype`` too; LSE stays fp32.  An unknown dtype
 * returns FA_ERR_INVALID_ARG.
 */
fa_status fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, float* LSE,
                    int B, int H, int N, int d, int causal, float scale,
                    float p_drop, uint64_t seed, fa_dtype dtype, void* stream);

/*
 * Forward pass with Nq queries and Nk keys per (b, h): Q, O are [B, H, Nq, d],
 * K, V are [B, H, Nk, d], LSE is fp32 [B, H, Nq], all 16-bit tensors of
 * ``dtype``.  Causal alignment as stated above.  Otherwise as fa_fwd_ex.
 */
fa_status fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, float* LSE,
                    int B, int H, int Nq, int Nk, int d, int causal, float scale,
                    float p_drop, uint64_t seed, fa_dtype dtype, void* stream);

/*
 * Forward pass over a batch of B sequences of different lengths, packed
 * without padding ("variable length").
 *   Q, O     : [total_q, H, d] of ``dtype``; token rows of all sequences back to back
 *   K, V     : [total_k, H, d]
 *   LSE      : out, fp32 [H, total_q]
 *   cu_seqlens_q, cu_seqlens_k : DEVICE int32 [B + 1], 4-byte aligned:
 *              sequence b owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *              and key rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1; offsets start
 *              at 0, never decrease and end at total_q / total_k
 *   max_seqlen_q, max_seqlen_k : the largest sequence lengths (they size the
 *              launch); 1 <= max_seqlen <= total
 * Each sequence is an independent problem with Nq = its query count and
 * Nk = its key count (causal alignment as above).  Dropout draws use b = the
 * sequence index and i, j = positions within the sequence.  The offsets live
 * on the device, so the library cannot check them: offsets that break the
 * rules above give wrong results for the rows concerned (every access is still
 * clamped into the tensors and the workspace).  H*total < 2^31.
 */
fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                        int B, int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                        int d, int causal, float scale, float p_drop, uint64_t seed,
                        fa_dtype dtype, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: an fp32 dQ
 * accumulator [B, H, N, d], the fp32 row statistic D and the fp32 copy of
 * LSE in log2 units, both [B, H, Npad] with Npad = N rounded up to a multiple
 * of 128, each part rounded up to 256 bytes.
 * Linear in N ("FlashAttention" glossary: memory drops from O(N^2) to O(N)).
 * Returns 0 for non-positive sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass by recomputation ("FlashAttention" glossary, Recomputation;
 * "Flash Attention" glossary, step 6 and Key Components on regenerating the
 * dropout pattern).
 *   Q, K, V, O, dO : in, bf16 [B, H, N, d]  (O from fa_fwd on the same inputs)
 *   LSE            : in, fp32 [B, H, N]     (from fa_fwd)
 *   dQ, dK, dV     : out, bf16 [B, H, N, d] gradients of sum(dO * O)
 *   workspace      : device scratch of at least fa_bwd_workspace_size() bytes,
 *                    256-byte aligned, owned by the caller, contents on entry
 *                    ignored; it may be reused once the stream has passed
 *                    this call.
 * causal, scale, p_drop and seed must equal the values given to fa_fwd; the
 * library cannot check this.  Steps: D_i = sum_c dO_ic O_ic and zeroing of
 * the dQ accumulator; one pass over key tiles recomputing P from LSE and
 * producing dK, dV and fp32 atomic contributions to dQ; conversion of dQ to
 * bf16.
 */
fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV,
                 int B, int H, int N, int d, int causal, float scale,
                 float p_drop, uint64_t seed, void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * fa_bwd for either 16-bit input type: Q, K, V, O, dO, dQ, dK and dV are all
 * of ``dtype`` (FA_DTYPE_BF16 gives exactly fa_bwd); the workspace is the
 * same fp32 scratch of fa_bwd_workspace_size() bytes.  The recomputed P and
 * dS are rounded to ``dtype`` before their products.  An unknown dtype
 * returns FA_ERR_INVALID_ARG.
 */
fa_status fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, void* dQ, void* dK, void* dV,
                    int B, int H, int N, int d, int causal, float scale,
                    float p_drop, uint64_t seed, fa_dtype dtype, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * Deterministic mode (the ``deterministic`` argument of fa_bwd_qk and
 * fa_bwd_varlen; the pages ask only for exact results, this is an option of
 * this library).  dQ is a sum over key tiles that many thread blocks add into
 * an fp32 accumulator; by default the order of those additions depends on
 * scheduling, so dQ may differ in its last bits from run to run (O, LSE, dK
 * and dV never do).  With deterministic != 0 the additions into each query
 * tile happen in increasing key-tile order, enforced with one counter per
 * (b, h, query tile) in the workspace, so repeated calls on the same inputs
 * give bitwise-identical dQ.  It needs the slightly larger workspace the
 * ``_workspace_size`` functions return for deterministic != 0 and may run
 * somewhat slower.
 */

/*
 * Workspace for fa_bwd_qk: fa_bwd_workspace_size(B, H, Nq, d) bytes, plus
 * (deterministic != 0) one uint32 counter per (b, h, 128-row query tile)
 * rounded up to 256 bytes.  Returns 0 for non-positive sizes.
 */
size_t fa_bwd_qk_workspace_size(int B, int H, int Nq, int d, int deterministic);

/*
 * Backward pass of fa_fwd_qk: Q, O, dO, dQ are [B, H, Nq, d], K, V, dK, dV
 * are [B, H, Nk, d]; workspace of at least
 * fa_bwd_qk_workspace_size(B, H, Nq, d, deterministic) bytes.  Otherwise as
 * fa_bwd_ex.
 */
fa_status fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                    const float* LSE, void* dQ, void* dK, void* dV,
                    int B, int H, int Nq, int Nk, int d, int causal, float scale,
                    float p_drop, uint64_t seed, fa_dtype dtype, int deterministic,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace for fa_bwd_varlen: an fp32 dQ accumulator [H, total_q, d], the
 * fp32 D and LSE*log2(e) vectors [B, H, pad128(max_seqlen_q)] and (when
 * deterministic != 0) the uint32 counters [B, H, pad128(max_seqlen_q)/128],
 * each part rounded up to 256 bytes.  Returns 0 for non-positive sizes.
 */
size_t fa_bwd_varlen_workspace_size(int B, int H, int total_q, int max_seqlen_q, int d,
                                    int deterministic);

/*
 * Backward pass of fa_fwd_varlen: same packed layouts (dQ like Q, dK and dV
 * like K), same offsets and scalars; workspace of at least
 * fa_bwd_varlen_workspace_size() bytes, 256-byte aligned.
 */
fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                        const float* LSE, void* dQ, void* dK, void* dV,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                        int B, int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                        int d, int causal, float scale, float p_drop, uint64_t seed,
                        fa_dtype dtype, int deterministic, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * The three stages fa_bwd runs, in order, for callers that schedule or time
 * them separately.  Same conventions and argument meanings as fa_bwd; each
 * validates its own arguments and enqueues one kernel.
 *   fa_bwd_prepare: D_i = sum_c dO_ic O_ic, LSE_i * log2(e), zero the dQ
 *                   accumulator (all in ``workspace``);
 *   fa_bwd_tiles:   the fused pass over (key tile, query tile) pairs that
 *                   recomputes P from the prepared LSE, regenerates the
 *                   dropout mask, writes dK and dV and adds into the dQ
 *                   accumulator; needs a workspace fa_bwd_prepare filled on the
 *                   same stream (or one ordered before it);
 *   fa_bwd_finish:  dQ = bf16(scale * accumulator).
 */
fa_status fa_bwd_prepare(const void* O, const void* dO, const float* LSE, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, void* stream);
fa_status fa_bwd_tiles(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV,
                       int B, int H, int N, int d, int causal, float scale, float p_drop, uint64_t seed,
                       void* workspace, size_t workspace_bytes, void* stream);
fa_status fa_bwd_finish(void* dQ, int B, int H, int N, int d, float scale, const void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * One training step of attention (forward, then backward) on HOST buffers,
 * with the host<->device copies overlapped with the kernels.  The pages ask
 * that end-to-end throughput, not only kernel speed, be measured ("Flash
 * Attention" glossary, Practical Limits and Common Pitfalls); this call is
 * that end-to-end path.
 *   Q, K, V, dO : host, [B, H, N, d] of ``dtype``, contiguous (page-locked for
 *                 the copies to overlap; pageable memory works but serialises)
 *   O, LSE      : host outputs, [B, H, N, d] and fp32 [B, H, N]
 *   dQ, dK, dV  : host outputs, [B, H, N, d]
 *   groups      : the B*H (b, h) units are cut into this many groups of
 *                 consecutive units (at most B*H; a smaller last group);
 *                 group g is copied in on streams[0], computed (fa_fwd and
 *                 the three backward stages, the same kernels and results as
 *                 fa_fwd / fa_bwd) on streams[1] (odd groups: on a second
 *                 compute stream the call creates and releases itself, so
 *                 one group's kernels start while the previous group's last
 *                 wave runs) and copied out on streams[2], so group g+1's
 *                 copy-in and group g-1's copy-out overlap group g's kernels.
 *                 Dropout counters keep the whole problem's (b, h).
 *   workspace   : device, 256-byte aligned, at least
 *                 fa_fwd_bwd_host_workspace_size(B, H, N, d, groups) bytes:
 *                 four staging slots of one group's tensors plus two of one
 *                 group's backward workspaces.  Caller-owned.
 *   streams     : three CUDA streams (cudaStream_t), copy-in, compute,
 *                 copy-out; the same stream may be given more than once (the
 *                 step then runs without overlap, and without the second
 *                 compute stream).
 * Everything is enqueued asynchronously and starts after the work already
 * enqueued on streams[2] (so calls in a row on the same streams reuse the
 * staging slots safely); the outputs are complete when streams[2] has
 * reached the end of this call's work (synchronise it).
 * Validation as fa_bwd (FA_ERR_INVALID_ARG for null pointers, groups <= 0, a
 * workspace too small or misaligned, an unknown dtype).
 */
size_t fa_fwd_bwd_host_workspace_size(int B, int H, int N, int d, int groups);
fa_status fa_fwd_bwd_host(const void* Q, const void* K, const void* V, const void* dO, void* O, float* LSE,
                          void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale,
                          float p_drop, uint64_t seed, fa_dtype dtype, int groups, void* workspace,
                          size_t workspace_bytes, void* const* streams);

/*
 * Backward pass for callers that cannot allocate device memory.  (The pages
 * have no counterpart: this is an integration convenience of this library.)
 * Some callers may not call cudaMalloc at all -- a plugin running inside a
 * framework whose memory pool owns every device allocation, a latency-critical
 * loop that cannot take the synchronisation an allocation may cause, or a
 * deployment with a fixed, audited memory budget.  fa_bwd_noalloc computes
 * exactly what fa_bwd computes, with the same arguments minus the workspace:
 * its scratch (fp32 dQ accumulator, D and LSE*log2(e)) lives in a fixed array
 * of FA_NOALLOC_SCRATCH_BYTES in the library's static device memory, which
 * every GPU that loads the library holds until the process exits.  The caller
 * still owns and passes every input and output.
 *   - Limit: fa_bwd_workspace_size(B, H, N, d) must not exceed
 *     FA_NOALLOC_SCRATCH_BYTES; larger problems return FA_ERR_UNSUPPORTED
 *     (use fa_bwd with a caller-provided workspace); for N a multiple of
 *     128 that allows B*H*N <= 64512 rows at d = 128, <= 126976 at d = 64,
 *     <= 43136 at d = 192 and <= 32512 at d = 256.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  It calls no allocating routine.
 *   - All calls share the one array, and each call's first stage rewrites
 *     every word of it that the call later reads, so earlier contents do not
 *     matter; but calls that overlap on the GPU (for example on two streams
 *     at once) race on it and must be serialised by the caller.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                         const float* LSE, void* dQ, void* dK, void* dV,
                         int B, int H, int N, int d, int causal, float scale,
                         float p_drop, uint64_t seed, void* stream);

/*
 * Decoding over a paged key/value cache: exact attention of the newest Nq
 * queries of each sequence over all of its cached positions, with the cache
 * kept in fixed-size pages that need not be contiguous (the serving setting
 * of the "FlashAttention" glossary's vLLM / PagedAttention entries).
 *   Q, O        : [B, H, Nq, d] of ``dtype``; O = softmax(scale Q K^T + mask) V
 *   LSE         : out, fp32 [B, H, Nq]
 *   K_cache, V_cache : [num_pages, page_size, H_kv, d] of ``dtype``
 *   block_table : DEVICE int32 [B, max_pages_per_seq]; entry (b, n) is the
 *                 page holding positions n*page_size .. of sequence b (only
 *                 the entries covering seqlens_k[b] are read)
 *   seqlens_k   : DEVICE int32 [B], cached positions of each sequence
 *                 (clamped to [0, max_pages_per_seq * page_size])
 *   H_kv        : key/value heads; H must be a multiple of it and query head
 *                 h reads key/value head h / (H / H_kv)
 *   causal      : nonzero -> query i of sequence b is position
 *                 seqlens_k[b] - Nq + i and sees positions up to it
 *   max_seqlen_k: the largest seqlens_k entry (sizes the launch; a sequence
 *                 longer than it is read only up to max_seqlen_k rounded up
 *                 to a multiple of 128 positions)
 *   page_size   : 16, 32, 64 or 128; d in {32, 64, 96, 128}; no dropout
 *   num_splits  : how many parts each sequence's positions are cut into
 *                 (each a thread block, merged by log-sum-exp); 0 chooses
 *                 fa_decode_num_splits(); with more than one split the call
 *                 needs ``workspace`` of fa_decode_workspace_size() bytes,
 *                 256-byte aligned (with one split it may be NULL).
 * A row that sees no position gets O = 0 and LSE = -inf.  Page ids outside
 * [0, num_pages) read as zeros; the tables live on the device, so the library
 * cannot check them otherwise.
 */
int fa_decode_num_splits(int B, int H_kv, int H, int Nq, int max_seqlen_k);
size_t fa_decode_workspace_size(int B, int H, int Nq, int d, int num_splits);
fa_status fa_decode_paged(const void* Q, const void* K_cache, const void* V_cache,
                          const int32_t* block_table, const int32_t* seqlens_k,
                          void* O, float* LSE, int B, int H, int H_kv, int Nq, int d,
                          int num_pages, int page_size, int max_pages_per_seq, int max_seqlen_k,
                          int causal, float scale, int num_splits, fa_dtype dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Test/inspection export of the attention-dropout pattern.  Dropout is
 * Bernoulli per attention score, applied inside the softmax step, and its
 * pattern is regenerated during the backward recomputation instead of being
 * stored ("FlashAttention" glossary, Dropout bullet; "Flash Attention"
 * glossary, Key Components).  This call writes that pattern, the keep mask
 * Z (1 = kept, 0 = dropped), as uint8 [B, H, N, N] into caller-owned device
 * memory ``mask`` (row i, column j = query i, key j), computed by the same
 * device Philox4x32-10 and keep test the kernels use: counter
 * (j >> 3, i, h, b), key (seed mod 2^32, seed >> 32), keep <=> u16 >= t with
 * t = round-half-even(p_drop * 65536).  N only needs to be positive; the
 * buffer must hold B*H*N*N bytes.  FA_ERR_INVALID_ARG for a null mask,
 * non-positive sizes or p_drop outside [0, 1); FA_ERR_UNSUPPORTED when
 * B*H*N >= 2^31.  Asynchronous on ``stream``.
 */
fa_status fa_dropout_mask(uint8_t* mask, int B, int H, int N, float p_drop, uint64_t seed,
                          void* stream);

/*
 * Synchronises the device, then reads and clears the device error word.
 * FA_OK when no kernel recorded a problem since the last call; FA_ERR_TIMEOUT
 * when a bounded wait gave up; FA_ERR_CUDA when a kernel found its shared-
 * memory layout would not fit and returned without work, or the device could
 * not be read.
 */
fa_status fa_last_device_error(void);

/*
 * Failure-detection self-test: enqueues one tiny kernel whose single bounded
 * wait is on a barrier that nothing ever completes, with a limit of
 * ``limit_us`` microseconds (1 .. 1000000).  The wait gives up, records a
 * timeout in the device error word and the kernel returns normally, so the
 * next fa_last_device_error() reports FA_ERR_TIMEOUT and the CUDA context
 * stays usable.  It exercises the same bounded-wait code the attention
 * kernels use; it never faults or hangs the device.
 */
fa_status fa_selftest_wait_timeout(uint32_t limit_us, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* fa_status_string(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H_ */
