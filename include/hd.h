/*
 * hd.h -- C ABI of libhd, the B200 (sm_100a) hot path of Hidden Decoding.
 *
 * Hidden Decoding ("Hidden Decoding at Scale: Latent Computation Scaling for
 * Large Language Models"; review page section "Method", Tencent/Sequential-
 * Hidden-Decoding README section "Key Idea") expands every token into n
 * streams, each with its own embedding table, lays them out token-major as a
 * length-nL sequence (expanded position p = t*n + s for token t, stream s) and
 * runs Stream-Factorized Attention (SFA) over it:
 *
 *   within-stream layers: query (t,s) attends keys (t',s) with t' <= t
 *   cross-stream layers:  query p attends every expanded position p' <= p,
 *                         so the intermediate streams' K/V stay as context.
 *
 * The library exports the three steps of that path: the n-table expansion,
 * SFA prefill in either mode, and SFA decode of the n new positions of one
 * token against the retained expanded KV cache.  Around them: the
 * cross-stream sliding window, the transient-intermediate-streams control
 * mask, chunked prefill and decode over a contiguous or paged cache (serving),
 * and the training-side pieces (final-stream rows, the tables' gradient, the
 * SFA backward).
 *
 * Conventions (every entry point):
 *   - All data pointers are DEVICE pointers into memory the caller owns and
 *     keeps alive until the work on `stream` has finished.  No call allocates
 *     device memory (the one array the library owns is described at
 *     sfa_decode_fwd_noalloc), no call synchronises, and each returns as soon
 *     as the work is enqueued on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).
 *   - Tensors are dense, row-major, with the shapes given below; bf16 is IEEE
 *     bfloat16 (16-bit storage).  Every tensor pointer must be 16-byte aligned.
 *   - Shape or alignment errors are detected on the host and returned before
 *     anything is launched.  Data-dependent errors (a token id out of range, a
 *     wait that timed out inside a kernel) never trap: the kernel ORs a bit
 *     into *dev_status (a device int32 the caller zeroes; may be NULL) and
 *     writes a defined result (zero rows for bad ids).
 *   - Supported: head_dim D in {64, 128}; Hq a multiple of Hkv (query head h
 *     reads KV head h / (Hq/Hkv)); 1 <= n <= 16; d_model a multiple of 8.
 *   - softmax_scale <= 0 selects 1/sqrt(D).
 */
#ifndef HD_H
#define HD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side return codes. */
typedef enum hd_status {
    HD_OK = 0,
    HD_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size    */
    HD_ERR_UNSUPPORTED = 2,   /* valid but not implemented (D, n, Hq % Hkv ...) */
    HD_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned               */
    HD_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed              */
    HD_ERR_WORKSPACE = 5      /* workspace missing or smaller than required     */
} hd_status;

/* Bits ORed into *dev_status by the kernels. */
#define HD_DEV_ID_RANGE 0x1   /* hd_expand_embed met an id outside [0, V)       */
#define HD_DEV_TIMEOUT 0x2    /* a bounded wait inside a kernel gave up         */
/* (HD_DEV_BAD_LENGTH 0x4 and HD_DEV_PAGE_RANGE 0x8: see sfa_decode_paged_fwd
 * and sfa_prefill_chunk_paged_fwd) */

/* SFA attention pattern of a layer. */
typedef enum sfa_mode {
    SFA_WITHIN = 0,           /* intra-stream: same stream, earlier-or-same token */
    SFA_CROSS = 1,            /* cross-stream: all earlier-or-same positions      */
    /* 2: cross-stream sliding window (the *_window_* and paged entry points)      */
    SFA_TRANSIENT = 3         /* PHD-style control: earlier tokens only through   */
                              /* their final stream n-1, the current token's      */
                              /* streams s' <= s (review "Prior limitations")     */
} sfa_mode;

/* Human-readable name of a hd_status value (static string). */
const char *hd_status_str(int status);

/* Message of the last CUDA error seen by this thread's library calls. */
const char *hd_last_cuda_error(void);

/* Library ABI version: (major << 16) | minor. */
int hd_version(void);

/*
 * hd_expand_embed -- token expansion into n streams with independent
 * embedding tables (review "Method"; README "Key Idea", item 1).
 *
 *   ids    : int64 [B][L], token ids.
 *   tables : HOST array of n DEVICE pointers; tables[s] is bf16 [V][d].
 *   out    : bf16 [B][L*n][d]; row t*n+s of batch b := tables[s][ids[b][t]].
 *
 * An id outside [0, V) produces a zero row and sets HD_DEV_ID_RANGE.
 * Bit-exact copy.  Returns HD_ERR_INVALID_ARG for B, L < 0, n outside
 * [1, 16], V < 1, d < 8 or d % 8 != 0.  B*L == 0 launches nothing.
 */
hd_status hd_expand_embed(const int64_t *ids, int64_t B, int64_t L,
                          const void *const *tables, int n, int64_t V,
                          int64_t d, void *out, int32_t *dev_status,
                          void *stream);

/*
 * hd_final_stream_rows -- the rows that feed the LM head and the loss: only
 * the final stream predicts the next token (review "Method": cross-entropy at
 * the final-stream positions only; README "Key Idea", item 3).
 *
 *   x   : bf16 [B][L*n][d]     expanded hidden states
 *   out : bf16 [B][L][d]       out[b][t] := x[b][t*n + n-1]  (bit-exact copy)
 */
hd_status hd_final_stream_rows(const void *x, int64_t B, int64_t L, int n,
                               int64_t d, void *out, void *stream);

/*
 * hd_expand_embed_backward -- gradient of hd_expand_embed with respect to the
 * n embedding tables:
 *   grad_tables[s][ids[b][t]] += grad_out[b][t*n + s]   for every (b, t, s).
 *
 *   ids         : int64 [B][L]
 *   grad_out    : bf16 [B][L*n][d]  gradient of the expanded rows
 *   grad_tables : HOST array of n DEVICE pointers, each fp32 [V][d],
 *                 ACCUMULATED into (zero them first for a plain gradient)
 *
 * fp32 atomic accumulation: the summation order over repeated ids is not
 * fixed, so results may differ in the last bits between runs.  Ids outside
 * [0, V) add nothing and set HD_DEV_ID_RANGE.  d % 8 == 0, n <= 16.
 */
hd_status hd_expand_embed_backward(const int64_t *ids, const void *grad_out,
                                   int64_t B, int64_t L, int n, int64_t V,
                                   int64_t d, float *const *grad_tables,
                                   int32_t *dev_status, void *stream);

/*
 * sfa_prefill_fwd -- Stream-Factorized Attention forward over the expanded
 * sequence of N = n*L positions (review "Method": most layers attend only
 * within their stream, O(nL^2); a few mix streams, O(n^2 L^2); README "Key
 * Idea").
 *
 *   q   : bf16 [B][N][Hq][D]   (post-projection, post-RoPE queries)
 *   k,v : bf16 [B][N][Hkv][D]
 *   o   : bf16 [B][N][Hq][D]   out
 *   lse : fp32 [B][Hq][N]      out, natural-log sum-exp of the scaled logits
 *                              of each row (may be NULL, except in the
 *                              transient mode: HD_ERR_INVALID_ARG)
 *   mode: SFA_WITHIN, SFA_CROSS or SFA_TRANSIENT (masks above).
 *
 * The transient mode runs two kernels: a pre-pass attends each row to its own
 * token's streams 0..s and leaves that normalised part in o and its
 * log-sum-exp in lse; the main kernel starts every row from that state and
 * adds the earlier tokens' final streams.
 *
 * o[b,p,h] = sum_{p' allowed} softmax(scale * q[b,p,h].k[b,p',g]) v[b,p',g],
 * g = h / (Hq/Hkv).  bf16 inputs, fp32 accumulation and softmax, bf16 output.
 * N = 0 launches nothing.  o must not alias q, k or v.
 */
hd_status sfa_prefill_fwd(const void *q, const void *k, const void *v, void *o,
                          float *lse, int64_t B, int64_t L, int n, int Hq,
                          int Hkv, int D, int mode, float softmax_scale,
                          int32_t *dev_status, void *stream);

/*
 * sfa_prefill_chunk_fwd -- SFA prefill of a chunk of C new tokens that follow
 * a cached prefix of P tokens (chunked prefill / prefix caching for serving;
 * the retained expanded cache is what later tokens read, review "Method").
 * The chunk's K/V rows must already be in the cache (append, then attend), so
 * the result equals rows n*P .. n*(P+C)-1 of sfa_prefill_fwd over the first
 * P + C tokens.
 *
 *   q, o    : bf16 [B][n*C][Hq][D]        the chunk's queries / outputs
 *   k_cache : bf16 [B][n*T_max][Hkv][D]   rows 0 .. n*(P+C)-1 are read
 *   v_cache : same layout
 *   lse     : fp32 [B][Hq][n*C] or NULL
 *   mode    : SFA_WITHIN, SFA_CROSS, or 2 = cross-stream sliding window of
 *             `window` tokens (ignored otherwise)
 *
 * P >= 0, C >= 0 (C = 0 launches nothing), P + C <= T_max.  C = 1 is a
 * decode step (sfa_decode_fwd is the memory-bound kernel for that case).
 */
hd_status sfa_prefill_chunk_fwd(const void *q, const void *k_cache,
                                const void *v_cache, void *o, float *lse,
                                int64_t B, int64_t P, int64_t C, int64_t T_max,
                                int n, int Hq, int Hkv, int D, int mode,
                                int64_t window, float softmax_scale,
                                int32_t *dev_status, void *stream);

/*
 * sfa_prefill_bwd -- gradients of SFA prefill (training through the SFA
 * layers; review "Method": the loss sits at the final-stream positions and
 * the model is trained end to end, so every within- and cross-stream layer
 * passes gradients back).  With P the softmax of the forward pass on the
 * allowed pairs:
 *   dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),
 *   dQ = scale dS K,  dK = scale dS^T Q,
 * dK / dV of a KV head summed over the query heads of its group.
 *
 *   q, o, dout, dq : bf16 [B][n*L][Hq][D]   (o: the forward output)
 *   k, v, dk, dv   : bf16 [B][n*L][Hkv][D]
 *   lse            : fp32 [B][Hq][n*L], the forward pass's log-sum-exp
 *                    (natural log), required
 *   mode           : SFA_WITHIN, SFA_CROSS, or 2 = cross-stream sliding window
 *                    of `window` tokens (ignored otherwise)
 *   workspace      : device scratch of sfa_prefill_bwd_workspace_bytes(), 16-byte
 *                    aligned, owned by the caller; overwritten
 *
 * Every output row is written by exactly one CTA (no atomics): the result is
 * deterministic.  dq / dk / dv are written, not accumulated into.
 * Errors: as sfa_prefill_fwd; HD_ERR_WORKSPACE if the workspace is short.
 */
size_t sfa_prefill_bwd_workspace_bytes(int64_t B, int64_t L, int n, int Hq,
                                       int mode);
hd_status sfa_prefill_bwd(const void *q, const void *k, const void *v,
                          const void *o, const void *dout, const float *lse,
                          void *dq, void *dk, void *dv, int64_t B, int64_t L,
                          int n, int Hq, int Hkv, int D, int mode,
                          int64_t window, float softmax_scale,
                          void *workspace, size_t workspace_bytes,
                          int32_t *dev_status, void *stream);

/*
 * sfa_prefill_chunk_paged_fwd -- sfa_prefill_chunk_fwd over a paged K/V pool
 * (README "Serving": a server keeps each request's expanded cache in pages):
 * sequence b has a cached prefix of prefix_tokens[b] tokens followed by the
 * chunk's C tokens, whose K/V rows are already in its pages.  Expanded
 * position r of sequence b is row r % page_rows of page
 * page_table[b * max_pages_per_seq + r / page_rows].
 *
 *   q, o          : bf16 [B][n*C][Hq][D]
 *   k/v_pages     : bf16 [num_pages][page_rows][Hkv][D]
 *   page_table    : int32 [B][max_pages_per_seq], device
 *   prefix_tokens : int32 [B], device; prefix + chunk tokens must fit the table
 *   chunk_tokens  : int32 [B], device, or NULL: sequence b's chunk is its first
 *                   chunk_tokens[b] <= C tokens (a variable-length batch padded
 *                   to C); o rows past it hold unspecified values and
 *                   their lse is not written.  NULL: every chunk has C
 *                   tokens.
 *   lse           : fp32 [B][Hq][n*C] or NULL
 *   mode          : SFA_WITHIN, SFA_CROSS, or 2 (sliding window of `window` tokens)
 *
 * page_rows must be a multiple of n; cross-stream modes also need whole
 * 128-position tiles per page (page_rows % 128 == 0); the within-stream mode
 * needs page_rows / n tokens per page to divide 128 or be a multiple of 128
 * (and a multiple of 8): else HD_ERR_UNSUPPORTED.  Rows of a sequence's last
 * page past its length may hold anything (they are never used).  A prefix
 * that does not fit, or a chunk length outside [0, C], sets HD_DEV_BAD_LENGTH
 * and leaves that sequence's rows unwritten; a page id outside
 * [0, num_pages) sets HD_DEV_PAGE_RANGE and its rows read as zeros.
 * The within-stream mode runs at contiguous-cache speed with pages of at
 * least 128 tokens; smaller pages take two half-height copies per K/V tile.
 */
hd_status sfa_prefill_chunk_paged_fwd(const void *q, const void *k_pages,
                                      const void *v_pages,
                                      const int32_t *page_table,
                                      int64_t max_pages_per_seq,
                                      int64_t num_pages, int64_t page_rows,
                                      const int32_t *prefix_tokens,
                                      const int32_t *chunk_tokens, void *o,
                                      float *lse, int64_t B, int64_t C, int n,
                                      int Hq, int Hkv, int D, int mode,
                                      int64_t window, float softmax_scale,
                                      int32_t *dev_status, void *stream);

/*
 * Bytes of device workspace sfa_decode_fwd needs for these shapes (may be 0).
 */
size_t sfa_decode_workspace_bytes(int64_t B, int n, int Hq, int Hkv, int D,
                                  int64_t T);

/*
 * sfa_decode_fwd -- one decode step of Hidden Decoding: the n new expanded
 * positions of token T (p = n*(T-1) + s, s = 0..n-1) attend the retained
 * expanded KV cache (review "Method": intermediate streams' KV is retained;
 * "Limitations": the retained cache is the serving cost) under the layer's
 * SFA mask.  The K/V rows of the n new positions must already be in the
 * cache (append, then attend), so the result equals the last n rows of
 * sfa_prefill_fwd over the first n*T positions.
 *
 *   q          : bf16 [B][n][Hq][D]    queries of the n new positions
 *   k_cache    : bf16 [B][n*T_max][Hkv][D]; rows 0 .. n*T_b-1 of sequence b
 *                are read
 *   v_cache    : same layout as k_cache
 *   seq_tokens : device int32 [B] or NULL.  NULL: every sequence holds T
 *                tokens.  Otherwise sequence b holds seq_tokens[b] tokens
 *                (1 .. T, the new one included): its new positions are
 *                n*(T_b-1)+s, and T only bounds the lengths (it sizes the
 *                work split and the workspace).  A count outside [1, T] sets
 *                HD_DEV_BAD_LENGTH and gives that sequence zero output.
 *   o          : bf16 [B][n][Hq][D]    out
 *   lse        : fp32 [B][Hq][n]       out (may be NULL)
 *   workspace  : device scratch of at least sfa_decode_workspace_bytes(...)
 *                bytes (may be NULL when that is 0); contents need not be
 *                initialised; must not be shared by calls in flight together.
 *
 * mode: SFA_WITHIN, SFA_CROSS or SFA_TRANSIENT.  1 <= T <= T_max.  Returns
 * HD_ERR_WORKSPACE if the workspace is too small, HD_ERR_MISALIGNED if
 * seq_tokens is not 4-byte aligned.
 */
hd_status sfa_decode_fwd(const void *q, const void *k_cache,
                         const void *v_cache, const int32_t *seq_tokens,
                         void *o, float *lse, int64_t B, int64_t T,
                         int64_t T_max, int n, int Hq, int Hkv, int D,
                         int mode, float softmax_scale, void *workspace,
                         size_t workspace_bytes, int32_t *dev_status,
                         void *stream);

/*
 * Cross-stream layers with a sliding window.  The pages give the mixing
 * layers the base model's own attention pattern, full or sliding-window (the
 * 80B model has 23 sliding-window cross-stream layers of 49; review
 * "Method"); the window's size is not given, so it is an argument here, in
 * tokens: query position p (token t) attends every p' <= p whose token t'
 * satisfies t' > t - window, i.e. all n streams of the last `window` tokens,
 * causally within the current token.  window >= the sequence length is the
 * plain cross-stream mask.  Arguments are those of the non-window entry
 * points with `mode` replaced by `window` (>= 1; HD_ERR_INVALID_ARG
 * otherwise).
 */
hd_status sfa_prefill_window_fwd(const void *q, const void *k, const void *v,
                                 void *o, float *lse, int64_t B, int64_t L,
                                 int n, int Hq, int Hkv, int D, int64_t window,
                                 float softmax_scale, int32_t *dev_status,
                                 void *stream);

size_t sfa_decode_window_workspace_bytes(int64_t B, int n, int Hq, int Hkv,
                                         int D, int64_t T, int64_t window);

/* Decode of token T over the window: only cache rows n*(T-window) .. n*T-1
 * are read (all of them while T <= window). */
hd_status sfa_decode_window_fwd(const void *q, const void *k_cache,
                                const void *v_cache, void *o, float *lse,
                                int64_t B, int64_t T, int64_t T_max, int n,
                                int Hq, int Hkv, int D, int64_t window,
                                float softmax_scale, void *workspace,
                                size_t workspace_bytes, int32_t *dev_status,
                                void *stream);

/*
 * Decode over a variable-length, paged retained cache (for serving: the
 * retained per-stream KV is the serving cost; review "Limitations"; the
 * serving patch manages expanded sequence lengths; README "Patch Contents").
 *
 * The cache is a pool of pages, k_pages / v_pages bf16
 * [num_pages][page_rows][Hkv][D]: cache row r of sequence b (expanded
 * position r) lives in page page_table[b * max_pages_per_seq + r / page_rows]
 * at row r % page_rows.  page_table may be NULL: then page b holds sequence
 * b (a contiguous cache with a page stride of page_rows rows).  With a page
 * table, page_rows must be a multiple of 64 and max_pages_per_seq * page_rows
 * must cover n * T_bound rows.
 *
 *   seq_tokens : device int32 [B], tokens of each sequence including the
 *                new one (1 .. T_bound), or NULL for T_bound everywhere.
 *                Sequence b's new positions are n*(T_b-1)+s.
 *   T_bound    : the largest token count (sizes the work split).
 *   mode       : SFA_WITHIN, SFA_CROSS, or 2 = cross-stream sliding window of
 *                `window` tokens (window ignored otherwise).
 *
 * Only rows of a sequence's valid range (its window, if any) take part; rows
 * past the range may hold anything.  A token count outside [1, T_bound] sets
 * HD_DEV_BAD_LENGTH and gives that sequence zero output; a page id outside
 * [0, num_pages) sets HD_DEV_PAGE_RANGE and reads as zeros.  Other arguments
 * as sfa_decode_fwd; the workspace size comes from
 * sfa_decode_paged_workspace_bytes.
 */
#define HD_DEV_BAD_LENGTH 0x4
#define HD_DEV_PAGE_RANGE 0x8

size_t sfa_decode_paged_workspace_bytes(int64_t B, int n, int Hq, int Hkv,
                                        int D, int64_t T_bound, int mode,
                                        int64_t window);

hd_status sfa_decode_paged_fwd(const void *q, const void *k_pages,
                               const void *v_pages, const int32_t *page_table,
                               int max_pages_per_seq, int64_t num_pages,
                               int64_t page_rows, const int32_t *seq_tokens,
                               int64_t T_bound, void *o, float *lse, int64_t B,
                               int n, int Hq, int Hkv, int D, int mode,
                               int64_t window, float softmax_scale,
                               void *workspace, size_t workspace_bytes,
                               int32_t *dev_status, void *stream);

/*
 * Self-checks of device building blocks (for tests; no counterpart on the
 * pages).
 *
 * hd_selftest_ex2: y_poly[i] = the library's FMA-pipe exp2 of x[i] (range
 * reduction plus a cubic, used for part of the prefill softmax) and
 * y_mufu[i] = the hardware ex2.approx of x[i]; fp32 device arrays of n.
 *
 * hd_selftest_timeout: one CTA waits on an mbarrier that nothing arrives on,
 * with the kernels' bounded-wait routine and a limit of limit_clocks SM
 * clocks (at most 2^31); the wait gives up and ORs HD_DEV_TIMEOUT into
 * *dev_status (a device int32, required).  Exercises the failure path
 * without faulting or hanging the GPU.
 */
hd_status hd_selftest_ex2(const float *x, float *y_poly, float *y_mufu,
                          int64_t n, void *stream);
hd_status hd_selftest_timeout(int32_t *dev_status, long long limit_clocks,
                              void *stream);

/*
 * sfa_decode_fwd_noalloc -- sfa_decode_fwd for callers that cannot provide
 * device scratch memory.  (An addition of this library: the paper has no
 * counterpart.)
 *
 * Some host programs cannot hand a library a workspace: plugin interfaces of
 * inference engines pass a kernel only its input and output buffers, and
 * serving runtimes that reserve all device memory at start-up forbid
 * allocation on the request path (cudaMalloc may synchronise the device and
 * its latency is unbounded).  This entry point takes the arguments of
 * sfa_decode_fwd minus seq_tokens (every sequence holds T tokens) and the
 * workspace, and keeps the key-split partial results
 * in one fixed device array of HD_DECODE_NOALLOC_SCRATCH_BYTES inside the
 * library instead.  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *
 *   - Limit: shapes whose sfa_decode_workspace_bytes(...) exceeds
 *     HD_DECODE_NOALLOC_SCRATCH_BYTES are rejected with HD_ERR_WORKSPACE
 *     before anything is launched.  Shapes that need no workspace never touch
 *     the array.
 *   - Memory: every GPU on which the library is used holds the array until
 *     the process exits.
 *   - Set-up: the first call on a device (with that device current) looks up
 *     the array's device address once; make that first call before any
 *     stream capture begins.  The address is kept for the life of the
 *     process: a cudaDeviceReset() ends the context that owns the array and
 *     leaves the kept address dangling, so do not call this entry point on a
 *     device after resetting it.
 *   - Sharing: all calls use the same array and it keeps the contents the
 *     last call left.  Nothing in it has to start at zero (every partial
 *     result is written before it is read), but two calls whose work overlaps
 *     on the GPU (different streams, or different host threads) race on it and
 *     give wrong results: serialise them.
 */
#define HD_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* Size of the fixed scratch array (HD_DECODE_NOALLOC_SCRATCH_BYTES). */
size_t sfa_decode_noalloc_scratch_bytes(void);

hd_status sfa_decode_fwd_noalloc(const void *q, const void *k_cache,
                                 const void *v_cache, void *o, float *lse,
                                 int64_t B, int64_t T, int64_t T_max, int n,
                                 int Hq, int Hkv, int D, int mode,
                                 float softmax_scale, int32_t *dev_status,
                                 void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HD_H */
