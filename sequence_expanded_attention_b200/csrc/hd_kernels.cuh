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

cudaError_t launch_expand_embed(const int64_t *ids, int64_t B, int64_t L, const ExpandTables &tables,
                                int n, int64_t V, int64_t d, void *out, int32_t *dev_status,
                                cudaStream_t stream, int num_sms);

// ------------------------------------------------------------------ prefill
struct PrefillParams {
  int64_t B, L, N;      // N = n * L expanded positions
  int n, Hq, Hkv, G;    // G = Hq / Hkv
  int mode;             // 0 within-stream, 1 cross-stream, 2 cross-stream sliding window
  int seq;              // per-problem sequence length: L (within) or N (cross)
  int q_tiles;          // ceil(seq / 128)
  int64_t problems;     // B * Hq * (within ? n : 1)
  float scale_log2;     // softmax_scale * log2(e)
  int64_t window;       // sliding window in tokens (mode 2)
  float *lse;           // [B][Hq][N] or nullptr
  int32_t *dev_status;
};

cudaError_t launch_sfa_prefill(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                               const CUtensorMap &tm_v, const CUtensorMap &tm_o,
                               const PrefillParams &p, int D, cudaStream_t stream);

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
  int splits, tiles_per_split, ntiles;
  int64_t T, nkeys;        // nkeys = n*T valid cache rows
  int64_t key_lo;          // first key row streamed: the sliding window's first row, else 0
  int mode;                // 0 within-stream, 1 cross-stream, 2 cross-stream window
  float scale_log2;
  int32_t *dev_status;
};

struct DecodePlan {
  int splits, tiles_per_split, ntiles, RG;
  size_t ws_bytes;
};

// key_lo: first key row the queries may attend (0 without a sliding window).
DecodePlan plan_sfa_decode(int64_t B, int n, int Hq, int Hkv, int D, int64_t T, int num_sms,
                           int64_t key_lo = 0);

cudaError_t launch_sfa_decode(const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                              const DecodeParams &p, int D, cudaStream_t stream);

}  // namespace hd
