// hd_kernels.cuh -- launch interfaces between libhd's host layer (hd_api.cu)
// and its kernels.  Internal: not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "hd_ptx.cuh"

namespace hd {

constexpr int kMaxStreams = 16;

struct ExpandTables {
  const void *ptr[kMaxStreams];
};

struct GradTables {
  float *ptr[kMaxStreams];
};

cudaError_t launch_final_stream_rows(const void *x, int64_t B, int64_t L, int n, int64_t d,
                                     void *out, cudaStream_t stream, int num_sms);

cudaError_t launch_expand_embed_backward(const int64_t *ids, const void *grad, int64_t B,
                                         int64_t L, int n, int64_t V, int64_t d,
                                         const GradTables &tables, int32_t *dev_status,
                                         cudaStream_t stream, int num_sms);

cudaError_t launch_expand_embed(const int64_t *ids, int64_t B, int64_t L, const ExpandTables &tables,
                                int n, int64_t V, int64_t d, void *out, int32_t *dev_status,
                                cudaStream_t stream, int num_sms);

// ------------------------------------------------------------------ prefill
struct PrefillParams {
  int64_t B, L, N;      // N = n * L expanded positions
  int n, Hq, Hkv, G;    // G = Hq / Hkv
  int mode;             // 0 within-stream, 1 cross-stream, 2 cross-stream sliding window,
                        // 3 transient intermediate streams (PHD-style control)
  int seq;              // per-problem query sequence length: L (within) or N (cross)
  int q_off;            // queries' offset among the keys (a chunk after a cached prefix)
  int q_tiles;          // ceil(seq / 128)
  int64_t problems;     // B * Hq * (within ? n : 1)
  // Work order: problems are taken in chunks of this many (whole KV groups,
  // sized so a chunk's K/V stays in L2), each chunk's query-tile pairs
  // heaviest first.
  int64_t chunk_problems;
  float scale_log2;     // softmax_scale * log2(e)
  int window;           // sliding window in tokens (mode 2), at most the key tokens
  // q [B][N][Hq][D], k/v [B][N][Hkv][D] (read directly by the transient pre-pass)
  const __nv_bfloat16 *q, *k, *v;
  // mode 3: the pre-pass's output for the current token's streams (the o
  // buffer) and its log-sum-exp (lse, required), the state each row starts from
  const __nv_bfloat16 *o_own;
  float *lse;           // [B][Hq][N] or nullptr
  int32_t *dev_status;
  // Paged K/V (chunked prefill over a page pool; page_table == nullptr
  // otherwise): sequence b's expanded position r is row r % page_rows of page
  // page_table[b * max_pages + r / page_rows]; its prefix is prefix[b] tokens.
  const int32_t *page_table;
  const int32_t *prefix;
  const int32_t *chunk_len;  // per-sequence chunk tokens (<= L) or nullptr
  int max_pages, num_pages, page_rows;
  int page_tokens;      // page_rows / n: tokens per page (within-stream view)
  int box_tokens;       // rows of one within-stream pool box: min(128, page_tokens)
};

cudaError_t launch_sfa_prefill(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                               const CUtensorMap &tm_v, const CUtensorMap &tm_o,
                               const PrefillParams &p, int D, cudaStream_t stream);
// Transient mode pre-pass: the current token's streams 0..s of every row, into
// o (normalised) and p.lse.
cudaError_t launch_transient_own(const PrefillParams &p, __nv_bfloat16 *o, int D,
                                 cudaStream_t stream);

// ------------------------------------------------------------------ backward
struct BwdParams {
  int64_t B, N;         // N = n * L expanded positions per batch
  int n, Hq, Hkv, G;    // G = Hq / Hkv
  int mode;             // 0 within-stream, 1 cross-stream, 2 cross-stream sliding window
  int seq;              // per-problem sequence length: L (within) or N (cross)
  int seq_pad;          // seq rounded up to 128: row stride of the row statistics
  int tiles;            // ceil(seq / 128)
  int window;           // sliding window in tokens (mode 2), at most L
  int64_t problems_q;   // B * Hq * (within ? n : 1)
  int64_t problems_kv;  // B * Hkv * (within ? n : 1)
  float scale;          // softmax scale (dQ and dK carry it)
  float scale_log2;     // softmax scale * log2(e)
  const __nv_bfloat16 *o, *dout;  // [B][N][Hq][D], for the row statistics
  const float *lse;     // [B][Hq][N], natural log, from the forward pass
  float *nlse;          // [problems_q][seq_pad]: -lse * log2(e)
  float *ndelta;        // [problems_q][seq_pad]: -<dO, O>
  int32_t *dev_status;
};

// Row statistics, then dK/dV (one CTA per 128-key tile), then dQ (one CTA per
// 128-query tile), in stream order.  Maps: 128-row boxes of Q, dO, K, V (the
// tiles a CTA keeps and the chunks it streams) and of the three gradients.
cudaError_t launch_sfa_backward(const CUtensorMap &q_t, const CUtensorMap &do_t,
                                const CUtensorMap &k_t, const CUtensorMap &v_t,
                                const CUtensorMap &dq_t, const CUtensorMap &dk_t,
                                const CUtensorMap &dv_t, const BwdParams &p, int D,
                                cudaStream_t stream, int num_sms);

// ------------------------------------------------------------------ decode
constexpr int kDecodeTileKeys = 64;
constexpr int kDecodeRows = 16;  // query rows (stream x head-in-group) per CTA
constexpr int kDecodeMaxSplits = 64;

struct DecodeParams {
  const __nv_bfloat16 *q;  // [B][n][Hq][D]
  __nv_bfloat16 *o;        // [B][n][Hq][D]
  float *lse;              // [B][Hq][n] or nullptr
  float *ws_o;             // [B][Hkv][RG][splits][16][D] partial outputs
  float *ws_lse;           // [B][Hkv][RG][splits][16] partial log2-sum-exp
  int B, n, Hq, Hkv, G, R, RG;  // R = n*G query rows per KV head, RG = ceil(R/16)
  int splits, tiles_per_split, ntiles;  // ntiles: tiles streamed per sequence (upper bound)
  int64_t T;               // tokens per sequence (the bound, when seq_tokens is given)
  const int32_t *seq_tokens;  // [B] tokens of each sequence, or nullptr (all T)
  // Cache storage: a pool of pages [num_pages][page_rows][Hkv][D] (the tensor
  // maps).  page_table [B][max_pages] maps a sequence's row block r / page_rows
  // to a page; nullptr means page b holds sequence b.
  const int32_t *page_table;
  int max_pages;
  int64_t num_pages, page_rows;
  int64_t window;          // sliding window in tokens (mode 2)
  int mode;                // 0 within-stream, 1 cross-stream, 2 cross-stream window
  float scale_log2;
  int32_t *dev_status;
};

struct DecodePlan {
  int splits, tiles_per_split, ntiles, RG;
  size_t ws_bytes;
};

// rows: cache rows streamed per sequence (an upper bound over the sequences).
DecodePlan plan_sfa_decode(int64_t B, int n, int Hq, int Hkv, int D, int64_t rows, int num_sms);

cudaError_t launch_sfa_decode(const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                              const DecodeParams &p, int D, cudaStream_t stream);

}  // namespace hd
