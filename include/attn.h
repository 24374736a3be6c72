/*
 * attn.h -- C ABI of the B200 (sm_100a) fused attention forward library (libattn.so).
 *
 * Operation (FlashAttention/ops-transformer article on ai6s.net):
 *   O = softmax(scale * Q K^T [+ causal mask]) V, per batch b and head h,
 * as defined in the section "传统注意力的显存陷阱" (scores = Q K^T / sqrt(d_k),
 * softmax over the key axis, output = probabilities . V), computed the way the
 * section "FlashAttention的核心逻辑" describes: Q blocks against streamed K/V
 * blocks with an online softmax (running row max and row sum, rescaling of the
 * partial output), one normalisation at the end, so the Nq x Nk score matrix
 * never exists in device memory.  The causal flag is the one of the article's
 * API example (section "如何使用", causal=True for GPT-style models).
 *
 * Readings where the article is silent:
 *   - the scale is an explicit argument (1/sqrt(d) is the caller's default);
 *   - causal with Nq != Nk is aligned to the bottom-right corner: key j is
 *     allowed for query i iff j <= i + (Nk - Nq);
 *   - a query row with no allowed key yields O = 0 and lse = -inf;
 *   - lse is the natural-log row log-sum-exp of the scaled, masked scores.
 *
 * Nothing here allocates host memory or keeps a caller's pointer after a call
 * returns.  All pointers except `stream` are DEVICE pointers on the current CUDA
 * device.  Per device, the library caches what it looks up on its first call
 * there (the device's properties, the kernels' shared-memory attributes, the
 * addresses of its status word and of the no-alloc array) for the life of the
 * process: do not keep using it on a device after cudaDeviceReset.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL means the legacy default stream. */
typedef struct CUstream_st* attn_stream_t;

/* Element type of q, k, v and out. */
typedef enum {
    ATTN_F16 = 0,   /* IEEE binary16 */
    ATTN_BF16 = 1   /* bfloat16 */
} attn_dtype_t;

/* Return codes.  Every entry point returns one of these (negative = error). */
typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = -1, /* null pointer, dimension <= 0, misaligned or overlapping
                                  buffers, non-finite scale, size beyond a stated limit */
    ATTN_ERR_UNSUPPORTED = -2, /* head_dim not in {64, 128}, unknown dtype, device not sm_100 */
    ATTN_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed (launch, allocation...) */
    ATTN_ERR_TIMEOUT = -4,     /* device side: a bounded pipeline wait gave up (see attn_get_status) */
    ATTN_ERR_RANGE = -5        /* device side: a bf16 V element has no fp16 value (see attn_fwd) */
} attn_status_t;

/*
 * attn_fwd -- fused scaled-dot-product attention forward.
 *
 *   q    [B, Nq, H, d]  contiguous, dtype        (read)
 *   k    [B, Nk, H, d]  contiguous, dtype        (read)
 *   v    [B, Nk, H, d]  contiguous, dtype        (read)
 *   out  [B, Nq, H, d]  contiguous, dtype        (written; must not overlap q, k, v, lse)
 *   lse  [B, H, Nq]     contiguous, float32      (written) or NULL = not written
 *   B, H, Nq, Nk >= 1;  d (head_dim) in {64, 128};  causal 0/1;  scale finite;
 *   dtype one of attn_dtype_t;  stream: the caller's stream.
 *
 * Alignment: q, k, v, out must be 16-byte aligned (tensor-memory-accelerator
 * copies); lse 4-byte aligned.
 *
 * Paths: Nq == 1 runs the split-KV decode kernels (partials + combine, with a
 * workspace of B*H*splits*(d+2)*4 bytes taken stream-ordered from the device's
 * default memory pool and returned on the same stream); every other shape runs
 * the tiled prefill kernel.  Both give the same result up to fp32 rounding.
 *
 * Value range (bf16 only): the tiled prefill multiplies P by V with both in
 * fp16 (fp16's 11-bit significand keeps the rounding of P small), converting
 * each bf16 V tile to fp16 on chip.  A V element of magnitude 65536 or more,
 * or an infinite or NaN one, has no fp16 value: the call then records
 * ATTN_ERR_RANGE in the status word read by attn_get_status(), and its O is
 * undefined.  Elements below 2^-14 in magnitude keep an absolute error under
 * 2^-25.  The decode path (Nq == 1) computes in fp32 and has no such limit.
 *
 * Asynchronous: the call validates its arguments on the host, enqueues the
 * kernels on `stream` and returns.  Argument errors return before anything is
 * enqueued.  A device-side failure (a bounded wait that expired, a V value out
 * of range) does not trap: it is recorded in a per-device status word read by
 * attn_get_status().
 * Since the call only enqueues work (and stream-ordered allocations) on
 * `stream`, it can be captured into a CUDA graph once a first call on the
 * device has run (that call sets the kernels' shared-memory attributes).
 *
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED or ATTN_ERR_CUDA.
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
             int B, int H, int Nq, int Nk, int d, int causal, float scale,
             int dtype, attn_stream_t stream);

/*
 * attn_fwd_prefill / attn_fwd_decode -- the two paths of attn_fwd, callable
 * directly (same arguments, same contract).  attn_fwd_decode requires Nq == 1
 * (ATTN_ERR_INVALID_ARG otherwise); `splits` = number of key ranges per
 * (b, h) row, 0 = automatic, otherwise 1 <= splits <= ceil(Nk / 128).
 */
ATTN_API int attn_fwd_prefill(const void* q, const void* k, const void* v, void* out, float* lse,
                     int B, int H, int Nq, int Nk, int d, int causal, float scale,
                     int dtype, attn_stream_t stream);
ATTN_API int attn_fwd_decode(const void* q, const void* k, const void* v, void* out, float* lse,
                    int B, int H, int Nk, int d, float scale, int dtype, int splits,
                    attn_stream_t stream);

/*
 * attn_fwd_decode_noalloc -- attn_fwd_decode without any device-memory allocation.
 * (An addition of this library; the article has no counterpart.)
 *
 * For callers that must not allocate device memory while they run: code hosted
 * inside another framework that owns all device memory and hands a plug-in only
 * its input and output buffers, serving loops that forbid allocation after
 * start-up so latency and footprint stay fixed, and processes at their memory
 * limit, where a per-call allocation could fail in the middle of a step.
 * attn_fwd_decode takes its split workspace from the stream-ordered pool; this
 * variant keeps the split partials in a fixed array compiled into the library
 * instead, and calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments, layouts and results are those of attn_fwd_decode; the caller
 * still passes q, k, v, out and lse.  Limit: B * H * splits * (d + 2) must not
 * exceed 1,048,576 floats (the array is 4 MiB; `splits` after the automatic
 * choice or the caller's value), otherwise the call returns
 * ATTN_ERR_INVALID_ARG and launches nothing.  Every GPU that loads the
 * library holds the 4 MiB array until the process exits.
 *
 * With splits = 0 the automatic choice only considers split counts whose
 * partials fit the array, so a shape that fits with fewer splits runs.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it for the life of the process; make that first
 * call before any stream capture, and do not keep using the library across a
 * reset of the device (cudaDeviceReset), which invalidates the cached address.
 * All calls share the one array and it keeps the last call's contents; nothing
 * in it has to start at zero, because every slot the combining kernel reads is
 * written earlier in the same call.  Calls whose kernels overlap on the GPU
 * (other streams, other host threads) race on the array and corrupt each
 * other's results: serialise them.
 */
ATTN_API int attn_fwd_decode_noalloc(const void* q, const void* k, const void* v, void* out,
                                     float* lse, int B, int H, int Nk, int d, float scale,
                                     int dtype, int splits, attn_stream_t stream);

/*
 * attn_fwd_decode_paged -- attn_fwd_decode over a paged key/value cache.
 *
 * One query row per request; request b's keys and values are its first
 * seq_lens[b] cache rows, stored page by page: keys [i*page_size,
 * (i+1)*page_size) of request b are rows [0, page_size) of cache page
 * block_table[b*max_blocks + i].  This is the decode metadata of the vLLM
 * MiniMax-M3 indexer page ("PR #45743 完整报告", section "关键源码片段":
 * per-request int32 seq_lens and a block table); the page size is the caller's.
 * The result equals attn_fwd_decode on each request's keys gathered densely.
 *
 *   q            [B, 1, H, d]                          dtype   (read)
 *   k_cache      [num_blocks, page_size, H, d]         dtype   (read)
 *   v_cache      [num_blocks, page_size, H, d]         dtype   (read)
 *   block_table  [B, max_blocks]                       int32   (read, DEVICE memory)
 *   seq_lens     [B]                                   int32   (read, DEVICE memory)
 *   out          [B, 1, H, d]                          dtype   (written)
 *   lse          [B, H] float32 (written) or NULL
 *   page_size: 8, 16, 32, 64 or a multiple of 128;  max_blocks * page_size and
 *   num_blocks * page_size below 2^31;  splits: 0 = automatic, else the number
 *   of key ranges per (b, h) (sized for max_blocks * page_size keys).
 *
 * seq_lens[b] is clamped to [0, max_blocks * page_size]; a request with no key
 * gets O = 0 and lse = -inf.  Table entries of pages holding keys below
 * seq_lens[b] must lie in [0, num_blocks) (others are clamped into it, so reads
 * stay inside the cache); entries past the sequence are not read.  Alignment
 * as attn_fwd, plus 4 bytes for block_table and seq_lens.  The workspace of
 * B*H*splits*(d+2)*4 bytes is taken stream-ordered as for attn_fwd_decode.
 *
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED (d, dtype, page
 * size or device) or ATTN_ERR_CUDA; asynchronous like attn_fwd.
 */
ATTN_API int attn_fwd_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                                   const int* block_table, const int* seq_lens, void* out,
                                   float* lse, int B, int H, int d, int num_blocks, int page_size,
                                   int max_blocks, float scale, int dtype, int splits,
                                   attn_stream_t stream);

/*
 * attn_fwd_paged -- several query tokens per request against a paged key/value
 * cache, on the tensor cores.
 *
 * The speculative-decoding step of the vLLM MiniMax-M3 indexer page ("PR #45743
 * 完整报告", section "功能与动机": the query tokens of one request are scored
 * together; section "关键源码片段": per-request int32 seq_lens and a block
 * table).  Request b's Lq query tokens are the last Lq positions of its
 * sequence of L = seq_lens[b] keys, stored page by page as for
 * attn_fwd_decode_paged.  With causal = 1, query i (0-based) sees keys
 * j <= L - Lq + i (the bottom-right alignment of attn_fwd); with causal = 0
 * every query sees all L keys.  A query with no key gets O = 0, lse = -inf.
 *
 *   q            [B, Lq, H, d]                         dtype   (read)
 *   k_cache      [num_blocks, page_size, H, d]         dtype   (read)
 *   v_cache      [num_blocks, page_size, H, d]         dtype   (read)
 *   block_table  [B, max_blocks]                       int32   (read, DEVICE memory)
 *   seq_lens     [B]                                   int32   (read, DEVICE memory)
 *   out          [B, Lq, H, d]                         dtype   (written)
 *   lse          [B, H, Lq] float32 (written) or NULL
 *   1 <= Lq <= 16; page_size, max_blocks, num_blocks, splits, seq_lens and
 *   table entries as attn_fwd_decode_paged; causal 0/1.
 *
 * The probabilities multiply V in fp16 (bf16 V tiles are converted to fp16 on
 * chip, as attn_fwd does; a bf16 V element of the sequence with no fp16 value,
 * magnitude 65536 or more, inf or NaN, makes the call record ATTN_ERR_RANGE in
 * the status word) and O is normalised by the sum of those rounded
 * probabilities.  The workspace of
 * B*H*splits*Lq*(d+2)*4 bytes is taken stream-ordered from the default pool.
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED or ATTN_ERR_CUDA;
 * asynchronous like attn_fwd.
 */
ATTN_API int attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                            const int* block_table, const int* seq_lens, void* out, float* lse,
                            int B, int H, int Lq, int d, int num_blocks, int page_size,
                            int max_blocks, int causal, float scale, int dtype, int splits,
                            attn_stream_t stream);

/*
 * attn_bwd -- gradients of attn_fwd (the backward pass).
 *
 * The step after the forward: the article notes (section "传统注意力的显存陷阱")
 * that eager attention keeps the N x N matrix for backpropagation.  Here the
 * probabilities are recomputed tile by tile from q, k and the forward's lse and
 * never stored; for an upstream gradient dO of O:
 *   P = exp(scale * Q K^T - lse) (masked entries 0),  dV = P^T dO,
 *   dS = P o (dO V^T - D) with D_i = sum_t dO_it O_it,
 *   dQ = scale * dS K,   dK = scale * dS^T Q.
 *
 *   q, o, dout   [B, Nq, H, d]   dtype      (read; o and lse as attn_fwd wrote them)
 *   k, v         [B, Nk, H, d]   dtype      (read)
 *   lse          [B, H, Nq]      float32    (read, required)
 *   dq           [B, Nq, H, d]   dtype      (written)
 *   dk, dv       [B, Nk, H, d]   dtype      (written)
 *   Sizes, causal rule, scale, dtype and alignment as attn_fwd; the outputs
 *   must not overlap each other or any input.  P and dS multiply on the tensor
 *   cores in the input type with fp32 accumulation; dQ is accumulated over key
 *   tiles in fp32.  A workspace of B*Nq*H*(d+1)*4 bytes (rounded up) is taken
 *   stream-ordered from the default pool and returned on the same stream.
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED or ATTN_ERR_CUDA;
 * asynchronous like attn_fwd.
 */
ATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk,
                      int d, int causal, float scale, int dtype, attn_stream_t stream);

/*
 * attn_fwd_relpos -- attention with a fused relative-position score term.
 *
 * The Granite-Speech conformer block attention of the vLLM page "PR #42933"
 * (sections "实现拆解" and "关键源码片段"): the scores carry, besides
 * q_i . k_j, the einsum of the queries with the relative-position embeddings
 * gathered by a distance table, both scaled, before masking and softmax:
 *   S[i, j] = scale * (q_i . k_j + q_i . emb[dist(i, j)]),
 *   dist(i, j) = clamp(i - j, -R, R) + R     (row R of emb is distance 0),
 * then O and lse exactly as attn_fwd.  The table is the conformer's clamped
 * relative distance, so it is given by R, not stored; a model whose table is
 * clamp(i - j, -R, R) + M passes emb + (M - R) * d.  The term is formed on the
 * tensor cores per 128 x 64 tile and never written to memory.
 *
 *   q, out       [B, Nq, H, d]   dtype      (read / written)
 *   k, v         [B, Nk, H, d]   dtype      (read)
 *   emb          [n_emb, d]      dtype      (read; n_emb >= 2R + 1; shared by
 *                                            every batch element and head)
 *   lse          [B, H, Nq]      float32    (written; may be NULL)
 *   B (batch x blocks), H, Nq, Nk, d, causal, scale, dtype and alignment as
 *   attn_fwd; emb 16-byte aligned, R >= 0.  For bf16 inputs P V runs in fp16 as
 *   in attn_fwd, with the same value-range status (ATTN_ERR_RANGE).
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED or ATTN_ERR_CUDA;
 * asynchronous like attn_fwd.
 */
ATTN_API int attn_fwd_relpos(const void* q, const void* k, const void* v, const void* emb, void* out,
                             float* lse, int B, int H, int Nq, int Nk, int d, int n_emb, int R,
                             int causal, float scale, int dtype, attn_stream_t stream);

/*
 * attn_indexer_score -- lightning-indexer score on the tensor cores.
 *
 * The aispot.cmou.io report on llama.cpp release b11372 (entry "compute the
 * indexer score with the lightning indexer"): each query token scores each
 * pooled key by the rectified dot product of every indexer head with the key,
 * weighted per head and summed over heads; keys have no head axis; an additive
 * f16 pool mask follows:
 *   score[b,t,p] = sum_h w[b,t,h] * max(0, q[b,t,h,:] . kp[b,p,:]) + mask[b,t,p]
 * (the report's unweighted form is w = 1/sqrt(d) for every head).
 *
 *   q      [B, T, H, d]  dtype            (read)
 *   kp     [B, P, d]     dtype            (read)
 *   w      [B, T, H]     float32          (read)
 *   mask   [B, T, P]     IEEE binary16 (0 or -inf), or NULL = no mask   (read)
 *   score  [B, T, P]     float32          (written; must not overlap the inputs)
 *   H a power of two <= 128; d in {64, 128}; alignment 16 bytes for q and kp,
 *   4 for w and score, 2 for mask.  Products accumulate in fp32.
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED or ATTN_ERR_CUDA;
 * asynchronous like attn_fwd.
 */
ATTN_API int attn_indexer_score(const void* q, const void* kp, const float* w, const void* mask,
                                float* score, int B, int T, int H, int P, int d, int dtype,
                                attn_stream_t stream);

/*
 * attn_topk -- positions of the k largest scores of each row.
 *
 * The selection the vLLM page "PR #45743 完整报告" (section "实现拆解") builds
 * on: only the order of the indexer scores matters.  For each of R rows of P
 * float32 scores, idx receives the positions of the k largest finite (or +inf)
 * scores, largest first; equal scores go lowest position first; -inf and NaN
 * are never chosen; slots past a row's chosen entries hold -1.
 *   score [R, P] float32 (read), idx [R, k] int32 (written); 1 <= k <= 2048.
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG or ATTN_ERR_CUDA; asynchronous.
 */
ATTN_API int attn_topk(const float* score, int R, int P, int k, int* idx, attn_stream_t stream);

/*
 * attn_get_status -- synchronises `stream`, then returns and clears the
 * current device's status word: ATTN_OK; ATTN_ERR_TIMEOUT if any kernel since
 * the last call gave up on a pipeline wait, or ATTN_ERR_RANGE if a bf16 prefill
 * met a V value with no fp16 value (the first such event is kept; the outputs
 * of the call it came from are undefined); or ATTN_ERR_CUDA if the
 * synchronisation itself failed.
 */
ATTN_API int attn_get_status(attn_stream_t stream);

/* attn_error_string -- static, human-readable text for a return code. */
ATTN_API const char* attn_error_string(int status);

/* attn_version -- library version as 10000*major + 100*minor + patch. */
ATTN_API int attn_version(void);

/*
 * attn_debug_set -- test hook for the failure-detection path.
 *   wait_timeout_ns: limit of every bounded device wait (0 = default, 2 s).
 *   inject: 0 = off; 1 = the prefill producer skips its first Q-tile load, so
 *   the matrix-multiply issuer's wait on it expires, the kernel records
 *   ATTN_ERR_TIMEOUT and every role exits without trapping.  Applies to the
 *   calls that follow on this host process; returns ATTN_OK.
 */
ATTN_API int attn_debug_set(int inject, unsigned long long wait_timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
