// hd_api.cu -- the C ABI of libhd (include/hd.h): argument validation, TMA
// tensor-map construction and kernel launches on the caller's stream.  The
// host layer never allocates device memory and never synchronises.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "../../include/hd.h"
#include "hd_kernels.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";

hd_status cuda_fail(cudaError_t e, const char *where) {
  snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s (%s)", where,
           cudaGetErrorName(e), cudaGetErrorString(e));
  return HD_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library needs no link-time dependency on libcuda.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tiled map, 128B swizzle.  dims / box innermost first; strides are the
// byte strides of dims 1 .. rank-1.
hd_status make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
                   const uint64_t *strides, const uint32_t *box) {
  auto fn = encode_fn();
  if (!fn) {
    snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
             "cuTensorMapEncodeTiled entry point unavailable");
    return HD_ERR_CUDA;
  }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled failed (%d)",
             (int)r);
    return HD_ERR_CUDA;
  }
  return HD_OK;
}

// Views of an expanded tensor X[B][n * L_stride][H][D] whose first n * L
// rows of each batch are valid (L = L_stride for a plain activation tensor):
//   within-stream: 5-D [B][L][n][H][D], box (64 d, 1 head, 1 stream, 128 tokens, 1)
//   cross-stream:  4-D [B][nL][H][D],   box (64 d, 1 head, 128 positions, 1)
hd_status make_prefill_map(CUtensorMap *m, const void *base, int64_t B, int64_t L,
                           int64_t L_stride, int n, int H, int D, bool within,
                           uint32_t box_rows = 128) {
  const uint64_t e = 2;  // bf16 bytes
  const uint64_t N = (uint64_t)n * L;
  const uint64_t Ns = (uint64_t)n * L_stride;
  if (within) {
    const uint64_t dims[5] = {(uint64_t)D, (uint64_t)H, (uint64_t)n, (uint64_t)L, (uint64_t)B};
    const uint64_t strides[4] = {D * e, (uint64_t)H * D * e, (uint64_t)n * H * D * e,
                                 Ns * H * D * e};
    const uint32_t box[5] = {64, 1, 1, box_rows, 1};
    return make_map(m, base, 5, dims, strides, box);
  }
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, N, (uint64_t)B};
  const uint64_t strides[3] = {D * e, (uint64_t)H * D * e, Ns * H * D * e};
  const uint32_t box[4] = {64, 1, box_rows, 1};
  return make_map(m, base, 4, dims, strides, box);
}

// Decode cache view: a pool of pages [num_pages][page_rows][Hkv][D] of which
// rows 0 .. extent-1 of each page may be read; rows past `extent` read as
// zeros.  Box (64 d, 1 head, 64 keys, 1 page).
hd_status make_cache_map(CUtensorMap *m, const void *base, int64_t num_pages, int64_t extent,
                         int64_t page_rows, int Hkv, int D) {
  const uint64_t e = 2;
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)extent, (uint64_t)num_pages};
  const uint64_t strides[3] = {D * e, (uint64_t)Hkv * D * e, (uint64_t)page_rows * Hkv * D * e};
  const uint32_t box[4] = {64, 1, (uint32_t)hd::kDecodeTileKeys, 1};
  return make_map(m, base, 4, dims, strides, box);
}

float resolve_scale(float s, int D) { return s > 0.f ? s : 1.0f / std::sqrt((float)D); }

// Problems per chunk of the prefill work order: whole KV groups (G query
// heads reading one K/V sequence of key_rows rows) whose K and V together
// take at most kL2ChunkBytes, so that a chunk's K/V stays in the 126 MB L2
// while all of its query tiles read it.
constexpr int64_t kL2ChunkBytes = 32ll << 20;

int64_t l2_chunk_problems(int64_t problems, int G, int64_t key_rows, int D) {
  const int64_t group_bytes = 2 * key_rows * D * 2;
  int64_t groups = kL2ChunkBytes / (group_bytes > 0 ? group_bytes : 1);
  if (groups < 1) groups = 1;
  const int64_t c = groups * G;
  return c < problems ? c : problems;
}

constexpr float kLog2e = 1.4426950408889634f;

// Shared body of the prefill entry points; mode 2 = cross-stream sliding
// window, 3 = transient intermediate streams.  The queries are L tokens that
// follow a cached prefix of P tokens: keys are the first P + L tokens of
// k / v, whose batch stride is T_kv tokens (P = 0, T_kv = L for a plain
// prefill).
hd_status prefill_impl(const void *q, const void *k, const void *v, void *o, float *lse, int64_t B,
                       int64_t L, int n, int Hq, int Hkv, int D, int mode, int64_t window,
                       int64_t P, int64_t T_kv, float softmax_scale, int32_t *dev_status,
                       void *stream) {
  if (B < 0 || L < 0 || n < 1 || Hq < 1 || Hkv < 1) return HD_ERR_INVALID_ARG;
  if (n > hd::kMaxStreams || (D != 64 && D != 128) || Hq % Hkv != 0) return HD_ERR_UNSUPPORTED;
  if (B * L == 0) return HD_OK;
  if (!q || !k || !v || !o) return HD_ERR_INVALID_ARG;
  // The transient mode carries the current token's part between its two
  // kernels in o and lse.
  if (mode == SFA_TRANSIENT && !lse) return HD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return HD_ERR_MISALIGNED;
  const int64_t N = (int64_t)n * L;
  // within-stream views for the within-stream mode and the transient mode
  const bool within = (mode == SFA_WITHIN || mode == SFA_TRANSIENT);
  // TMA coordinates are 32-bit and the grid is one CTA per (problem, tile pair).
  if ((int64_t)n * T_kv > (1LL << 30) || B > (1LL << 20)) return HD_ERR_UNSUPPORTED;
  hd::PrefillParams p{};
  p.B = B;
  p.L = L;
  p.N = N;
  p.n = n;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.mode = mode;
  p.window = (int)(window < P + L ? window : P + L);  // a longer window is the full mask
  p.seq = (int)(within ? L : N);
  p.q_off = (int)(within ? P : (int64_t)n * P);
  p.q_tiles = (p.seq + 127) / 128;
  p.problems = B * Hq * (within ? n : 1);
  p.chunk_problems = l2_chunk_problems(p.problems, p.G, within ? P + L : (int64_t)n * (P + L), D);
  p.scale_log2 = resolve_scale(softmax_scale, D) * kLog2e;
  p.lse = lse;
  p.dev_status = dev_status;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.k = static_cast<const __nv_bfloat16 *>(k);
  p.v = static_cast<const __nv_bfloat16 *>(v);
  CUtensorMap tq, tk, tv, to;
  hd_status st;
  if ((st = make_prefill_map(&tq, q, B, L, L, n, Hq, D, within)) != HD_OK) return st;
  if ((st = make_prefill_map(&tk, k, B, P + L, T_kv, n, Hkv, D, within)) != HD_OK) return st;
  if ((st = make_prefill_map(&tv, v, B, P + L, T_kv, n, Hkv, D, within)) != HD_OK) return st;
  if ((st = make_prefill_map(&to, o, B, L, L, n, Hq, D, within)) != HD_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (mode == SFA_TRANSIENT) {
    p.o_own = static_cast<const __nv_bfloat16 *>(o);
    const cudaError_t e0 = hd::launch_transient_own(p, static_cast<__nv_bfloat16 *>(o), D, cs);
    if (e0 != cudaSuccess) return cuda_fail(e0, "transient pre-pass launch");
  }
  cudaError_t e = hd::launch_sfa_prefill(tq, tk, tv, to, p, D, cs);
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "sfa_prefill launch");
}

// First key row the n new positions of token T may attend under a sliding
// window of `window` tokens: the n streams of tokens T-window .. T-1.
int64_t window_key_lo(int n, int64_t T, int64_t window) {
  const int64_t t0 = T - window;
  return t0 > 0 ? (int64_t)n * t0 : 0;
}

// Where the decode reads the cache from.
struct CacheStorage {
  const int32_t *seq_tokens;  // nullable: all sequences have T tokens
  const int32_t *page_table;  // nullable: page b is sequence b
  int max_pages;
  int64_t num_pages;          // pages in the pool
  int64_t page_rows;          // rows per page (the stride between pages)
  int64_t page_extent;        // rows of a page that may be read (<= page_rows)
  int64_t stream_rows;        // rows streamed per sequence, upper bound (the plan)
};

// Shared body of the decode entry points; mode 2 = cross-stream sliding window.
hd_status decode_impl(const void *q, const void *k_cache, const void *v_cache, void *o,
                      float *lse, int64_t B, int64_t T, int n, int Hq, int Hkv, int D, int mode,
                      int64_t window, const CacheStorage &cs, float softmax_scale,
                      void *workspace, size_t workspace_bytes, int32_t *dev_status, void *stream) {
  if (!q || !k_cache || !v_cache || !o) return HD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || !aligned16(workspace))
    return HD_ERR_MISALIGNED;
  const hd::DecodePlan pl = hd::plan_sfa_decode(B, n, Hq, Hkv, D, cs.stream_rows, device_sms());
  if (pl.ws_bytes > 0 && (!workspace || workspace_bytes < pl.ws_bytes)) return HD_ERR_WORKSPACE;
  hd::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.lse = lse;
  p.B = (int)B;
  p.n = n;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.R = n * p.G;
  p.RG = pl.RG;
  p.splits = pl.splits;
  p.tiles_per_split = pl.tiles_per_split;
  p.ntiles = pl.ntiles;
  p.T = T;
  p.seq_tokens = cs.seq_tokens;
  p.page_table = cs.page_table;
  p.max_pages = cs.max_pages;
  p.num_pages = cs.num_pages;
  p.page_rows = cs.page_rows;
  p.window = window;
  p.mode = mode;
  p.scale_log2 = resolve_scale(softmax_scale, D) * kLog2e;
  p.dev_status = dev_status;
  if (pl.ws_bytes > 0) {
    const size_t rows = (size_t)B * Hkv * pl.RG * pl.splits * hd::kDecodeRows;
    p.ws_o = static_cast<float *>(workspace);
    p.ws_lse = p.ws_o + rows * D;
  }
  CUtensorMap tk, tv;
  hd_status st;
  if ((st = make_cache_map(&tk, k_cache, cs.num_pages, cs.page_extent, cs.page_rows, Hkv, D)) !=
      HD_OK)
    return st;
  if ((st = make_cache_map(&tv, v_cache, cs.num_pages, cs.page_extent, cs.page_rows, Hkv, D)) !=
      HD_OK)
    return st;
  cudaError_t e = hd::launch_sfa_decode(tk, tv, p, D, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "sfa_decode launch");
}

// Shape checks common to the decode entry points.
hd_status decode_shape_check(int64_t B, int64_t T, int n, int Hq, int Hkv, int D) {
  if (B < 0 || n < 1 || Hq < 1 || Hkv < 1 || T < 1) return HD_ERR_INVALID_ARG;
  if (n > hd::kMaxStreams || (D != 64 && D != 128) || Hq % Hkv != 0) return HD_ERR_UNSUPPORTED;
  if (B > 65535) return HD_ERR_UNSUPPORTED;  // one grid z-slice per sequence
  return HD_OK;
}

// Contiguous per-sequence cache [B][n*T_max] read for the first n*T rows.
CacheStorage contiguous_storage(int64_t B, int64_t T, int64_t T_max, int n, int64_t key_lo) {
  CacheStorage cs{};
  cs.num_pages = B;
  cs.page_rows = (int64_t)n * T_max;
  cs.page_extent = (int64_t)n * T;
  cs.stream_rows = (int64_t)n * T - key_lo;
  return cs;
}

}  // namespace

extern "C" {

const char *hd_status_str(int status) {
  switch (status) {
    case HD_OK: return "ok";
    case HD_ERR_INVALID_ARG: return "invalid argument";
    case HD_ERR_UNSUPPORTED: return "unsupported configuration";
    case HD_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case HD_ERR_CUDA: return "CUDA error";
    case HD_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

const char *hd_last_cuda_error(void) { return g_last_cuda_error; }

int hd_version(void) { return (2 << 16) | 0; }

hd_status hd_expand_embed(const int64_t *ids, int64_t B, int64_t L, const void *const *tables,
                          int n, int64_t V, int64_t d, void *out, int32_t *dev_status,
                          void *stream) {
  if (B < 0 || L < 0 || n < 1 || n > hd::kMaxStreams || V < 1 || d < 8 || d % 8 != 0)
    return HD_ERR_INVALID_ARG;
  if (B * L == 0) return HD_OK;
  if (!ids || !tables || !out) return HD_ERR_INVALID_ARG;
  hd::ExpandTables t{};
  for (int s = 0; s < n; ++s) {
    if (!tables[s]) return HD_ERR_INVALID_ARG;
    if (!aligned16(tables[s])) return HD_ERR_MISALIGNED;
    t.ptr[s] = tables[s];
  }
  if (!aligned16(out) || (reinterpret_cast<uintptr_t>(ids) & 7u)) return HD_ERR_MISALIGNED;
  cudaError_t e = hd::launch_expand_embed(ids, B, L, t, n, V, d, out, dev_status,
                                          static_cast<cudaStream_t>(stream), device_sms());
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "hd_expand_embed launch");
}

hd_status hd_final_stream_rows(const void *x, int64_t B, int64_t L, int n, int64_t d, void *out,
                               void *stream) {
  if (B < 0 || L < 0 || n < 1 || d < 8 || d % 8 != 0) return HD_ERR_INVALID_ARG;
  if (B * L == 0) return HD_OK;
  if (!x || !out) return HD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return HD_ERR_MISALIGNED;
  cudaError_t e = hd::launch_final_stream_rows(x, B, L, n, d, out,
                                               static_cast<cudaStream_t>(stream), device_sms());
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "hd_final_stream_rows launch");
}

hd_status hd_expand_embed_backward(const int64_t *ids, const void *grad_out, int64_t B, int64_t L,
                                   int n, int64_t V, int64_t d, float *const *grad_tables,
                                   int32_t *dev_status, void *stream) {
  if (B < 0 || L < 0 || n < 1 || n > hd::kMaxStreams || V < 1 || d < 8 || d % 8 != 0)
    return HD_ERR_INVALID_ARG;
  if (B * L == 0) return HD_OK;
  if (!ids || !grad_out || !grad_tables) return HD_ERR_INVALID_ARG;
  hd::GradTables t{};
  for (int s = 0; s < n; ++s) {
    if (!grad_tables[s]) return HD_ERR_INVALID_ARG;
    if (!aligned16(grad_tables[s])) return HD_ERR_MISALIGNED;
    t.ptr[s] = grad_tables[s];
  }
  if (!aligned16(grad_out) || (reinterpret_cast<uintptr_t>(ids) & 7u)) return HD_ERR_MISALIGNED;
  cudaError_t e = hd::launch_expand_embed_backward(ids, grad_out, B, L, n, V, d, t, dev_status,
                                                   static_cast<cudaStream_t>(stream),
                                                   device_sms());
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "hd_expand_embed_backward launch");
}

hd_status sfa_prefill_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                          int64_t B, int64_t L, int n, int Hq, int Hkv, int D, int mode,
                          float softmax_scale, int32_t *dev_status, void *stream) {
  if (mode != SFA_WITHIN && mode != SFA_CROSS && mode != SFA_TRANSIENT) return HD_ERR_INVALID_ARG;
  return prefill_impl(q, k, v, o, lse, B, L, n, Hq, Hkv, D, mode, 0, 0, L, softmax_scale,
                      dev_status, stream);
}

hd_status sfa_prefill_window_fwd(const void *q, const void *k, const void *v, void *o,
                                 float *lse, int64_t B, int64_t L, int n, int Hq, int Hkv, int D,
                                 int64_t window, float softmax_scale, int32_t *dev_status,
                                 void *stream) {
  if (window < 1) return HD_ERR_INVALID_ARG;
  return prefill_impl(q, k, v, o, lse, B, L, n, Hq, Hkv, D, 2, window, 0, L, softmax_scale,
                      dev_status, stream);
}

hd_status sfa_prefill_chunk_fwd(const void *q, const void *k_cache, const void *v_cache, void *o,
                                float *lse, int64_t B, int64_t P, int64_t C, int64_t T_max, int n,
                                int Hq, int Hkv, int D, int mode, int64_t window,
                                float softmax_scale, int32_t *dev_status, void *stream) {
  if (mode != SFA_WITHIN && mode != SFA_CROSS && mode != 2) return HD_ERR_INVALID_ARG;
  if (mode == 2 && window < 1) return HD_ERR_INVALID_ARG;
  if (P < 0 || C < 0 || P + C > T_max) return HD_ERR_INVALID_ARG;
  return prefill_impl(q, k_cache, v_cache, o, lse, B, C, n, Hq, Hkv, D, mode, window, P, T_max,
                      softmax_scale, dev_status, stream);
}

hd_status sfa_prefill_chunk_paged_fwd(const void *q, const void *k_pages, const void *v_pages,
                                      const int32_t *page_table, int64_t max_pages_per_seq,
                                      int64_t num_pages, int64_t page_rows,
                                      const int32_t *prefix_tokens,
                                      const int32_t *chunk_tokens, void *o, float *lse,
                                      int64_t B, int64_t C, int n, int Hq, int Hkv, int D,
                                      int mode, int64_t window, float softmax_scale,
                                      int32_t *dev_status, void *stream) {
  if (mode != SFA_WITHIN && mode != SFA_CROSS && mode != 2) return HD_ERR_INVALID_ARG;
  if (mode == 2 && window < 1) return HD_ERR_INVALID_ARG;
  if (B < 0 || C < 0 || n < 1 || Hq < 1 || Hkv < 1 || max_pages_per_seq < 1 || num_pages < 1 ||
      page_rows < 1)
    return HD_ERR_INVALID_ARG;
  if (n > hd::kMaxStreams || (D != 64 && D != 128) || Hq % Hkv != 0) return HD_ERR_UNSUPPORTED;
  const bool within = (mode == SFA_WITHIN);
  // Whole 128-position tiles per page (cross-stream); whole tokens per page and
  // boxes of a power-of-two token count (within-stream).
  if (page_rows % n != 0) return HD_ERR_UNSUPPORTED;
  const int64_t page_tokens = page_rows / n;
  if (!within && page_rows % 128 != 0) return HD_ERR_UNSUPPORTED;
  if (within && (page_tokens % 8 != 0 ||
                 (page_tokens < 128 ? 128 % page_tokens != 0 : page_tokens % 128 != 0)))
    return HD_ERR_UNSUPPORTED;
  if (B * C == 0) return HD_OK;
  if (!q || !k_pages || !v_pages || !o || !page_table || !prefix_tokens) return HD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(page_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(prefix_tokens) & 3u) ||
      (reinterpret_cast<uintptr_t>(chunk_tokens) & 3u))
    return HD_ERR_MISALIGNED;
  if (max_pages_per_seq * page_rows > (1LL << 30) || num_pages > (1LL << 30) ||
      (int64_t)n * C > (1LL << 30) || B > (1LL << 20))
    return HD_ERR_UNSUPPORTED;
  hd::PrefillParams p{};
  p.B = B;
  p.L = C;
  p.N = (int64_t)n * C;
  p.n = n;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.mode = mode;
  const int64_t cap_tokens = max_pages_per_seq * page_tokens;
  p.window = (int)(window < cap_tokens ? window : cap_tokens);
  p.seq = (int)(within ? C : (int64_t)n * C);
  p.q_off = 0;  // per sequence, from prefix_tokens
  p.q_tiles = (p.seq + 127) / 128;
  p.problems = B * Hq * (within ? n : 1);
  p.chunk_problems =
      l2_chunk_problems(p.problems, p.G, within ? cap_tokens : (int64_t)n * cap_tokens, D);
  p.scale_log2 = resolve_scale(softmax_scale, D) * kLog2e;
  p.lse = lse;
  p.dev_status = dev_status;
  p.page_table = page_table;
  p.prefix = prefix_tokens;
  p.chunk_len = chunk_tokens;
  p.max_pages = (int)max_pages_per_seq;
  p.num_pages = (int)num_pages;
  p.page_rows = (int)page_rows;
  p.page_tokens = (int)page_tokens;
  p.box_tokens = (int)(page_tokens < 128 ? page_tokens : 128);
  CUtensorMap tq, tk, tv, to;
  hd_status st;
  if ((st = make_prefill_map(&tq, q, B, C, C, n, Hq, D, within)) != HD_OK) return st;
  if ((st = make_prefill_map(&to, o, B, C, C, n, Hq, D, within)) != HD_OK) return st;
  // The pool: [num_pages][page_rows][Hkv][D], viewed as 4-D (cross-stream) or
  // as 5-D [num_pages][page_tokens][n][Hkv][D] (within-stream).
  const uint64_t e = 2;
  for (int t = 0; t < 2; ++t) {
    CUtensorMap *m = t ? &tv : &tk;
    const void *base = t ? v_pages : k_pages;
    if (within) {
      const uint64_t dims[5] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)n, (uint64_t)page_tokens,
                                (uint64_t)num_pages};
      const uint64_t strides[4] = {D * e, (uint64_t)Hkv * D * e, (uint64_t)n * Hkv * D * e,
                                   (uint64_t)page_rows * Hkv * D * e};
      const uint32_t box[5] = {64, 1, 1, (uint32_t)p.box_tokens, 1};
      if ((st = make_map(m, base, 5, dims, strides, box)) != HD_OK) return st;
    } else {
      const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)page_rows,
                                (uint64_t)num_pages};
      const uint64_t strides[3] = {D * e, (uint64_t)Hkv * D * e,
                                   (uint64_t)page_rows * Hkv * D * e};
      const uint32_t box[4] = {64, 1, 128, 1};
      if ((st = make_map(m, base, 4, dims, strides, box)) != HD_OK) return st;
    }
  }
  cudaError_t err = hd::launch_sfa_prefill(tq, tk, tv, to, p, D, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? HD_OK : cuda_fail(err, "sfa_prefill_chunk_paged launch");
}

// Row statistics of the backward pass: -LSE * log2(e) and -<dO, O> per query
// row (two fp32 arrays), rows of each problem padded to a multiple of 128.
static int64_t bwd_seq(int64_t L, int n, int mode) {
  return mode == SFA_WITHIN ? L : (int64_t)n * L;
}

size_t sfa_prefill_bwd_workspace_bytes(int64_t B, int64_t L, int n, int Hq, int mode) {
  if (B < 1 || L < 1 || n < 1 || n > hd::kMaxStreams || Hq < 1 || mode < 0 || mode > 2) return 0;
  const int64_t seq_pad = (bwd_seq(L, n, mode) + 127) / 128 * 128;
  const int64_t problems = B * Hq * (mode == SFA_WITHIN ? n : 1);
  return (size_t)(problems * seq_pad) * 8;
}

hd_status sfa_prefill_bwd(const void *q, const void *k, const void *v, const void *o,
                          const void *dout, const float *lse, void *dq, void *dk, void *dv,
                          int64_t B, int64_t L, int n, int Hq, int Hkv, int D, int mode,
                          int64_t window, float softmax_scale, void *workspace,
                          size_t workspace_bytes, int32_t *dev_status, void *stream) {
  if (B < 0 || L < 0 || n < 1 || Hq < 1 || Hkv < 1) return HD_ERR_INVALID_ARG;
  if (mode != SFA_WITHIN && mode != SFA_CROSS && mode != 2) return HD_ERR_INVALID_ARG;
  if (mode == 2 && window < 1) return HD_ERR_INVALID_ARG;
  if (n > hd::kMaxStreams || (D != 64 && D != 128) || Hq % Hkv != 0) return HD_ERR_UNSUPPORTED;
  if (B * L == 0) return HD_OK;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace)
    return HD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return HD_ERR_MISALIGNED;
  const int64_t N = (int64_t)n * L;
  if (N > (1LL << 30) || B > (1LL << 20)) return HD_ERR_UNSUPPORTED;
  if (workspace_bytes < sfa_prefill_bwd_workspace_bytes(B, L, n, Hq, mode))
    return HD_ERR_WORKSPACE;
  const bool within = (mode == SFA_WITHIN);
  hd::BwdParams p{};
  p.B = B;
  p.N = N;
  p.n = n;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.mode = mode;
  p.seq = (int)bwd_seq(L, n, mode);
  p.seq_pad = (p.seq + 127) / 128 * 128;
  p.tiles = p.seq_pad / 128;
  p.window = (int)(window < L ? window : L);
  p.problems_q = B * Hq * (within ? n : 1);
  p.problems_kv = B * Hkv * (within ? n : 1);
  p.scale = resolve_scale(softmax_scale, D);
  p.scale_log2 = p.scale * kLog2e;
  p.o = static_cast<const __nv_bfloat16 *>(o);
  p.dout = static_cast<const __nv_bfloat16 *>(dout);
  p.lse = lse;
  p.nlse = static_cast<float *>(workspace);
  p.ndelta = p.nlse + p.problems_q * p.seq_pad;
  p.dev_status = dev_status;
  CUtensorMap q_t, do_t, k_t, v_t, dq_t, dk_t, dv_t;
  hd_status st;
  if ((st = make_prefill_map(&q_t, q, B, L, L, n, Hq, D, within)) != HD_OK ||
      (st = make_prefill_map(&do_t, dout, B, L, L, n, Hq, D, within)) != HD_OK ||
      (st = make_prefill_map(&k_t, k, B, L, L, n, Hkv, D, within)) != HD_OK ||
      (st = make_prefill_map(&v_t, v, B, L, L, n, Hkv, D, within)) != HD_OK ||
      (st = make_prefill_map(&dq_t, dq, B, L, L, n, Hq, D, within)) != HD_OK ||
      (st = make_prefill_map(&dk_t, dk, B, L, L, n, Hkv, D, within)) != HD_OK ||
      (st = make_prefill_map(&dv_t, dv, B, L, L, n, Hkv, D, within)) != HD_OK)
    return st;
  cudaError_t e = hd::launch_sfa_backward(q_t, do_t, k_t, v_t, dq_t, dk_t, dv_t, p, D,
                                          static_cast<cudaStream_t>(stream), device_sms());
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "sfa_prefill_bwd");
}

size_t sfa_decode_workspace_bytes(int64_t B, int n, int Hq, int Hkv, int D, int64_t T) {
  if (B < 1 || decode_shape_check(B, T, n, Hq, Hkv, D) != HD_OK) return 0;
  return hd::plan_sfa_decode(B, n, Hq, Hkv, D, (int64_t)n * T, device_sms()).ws_bytes;
}

size_t sfa_decode_window_workspace_bytes(int64_t B, int n, int Hq, int Hkv, int D, int64_t T,
                                         int64_t window) {
  if (B < 1 || window < 1 || decode_shape_check(B, T, n, Hq, Hkv, D) != HD_OK) return 0;
  return hd::plan_sfa_decode(B, n, Hq, Hkv, D, (int64_t)n * T - window_key_lo(n, T, window),
                             device_sms())
      .ws_bytes;
}

hd_status sfa_decode_fwd(const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *seq_tokens, void *o, float *lse, int64_t B, int64_t T,
                         int64_t T_max, int n, int Hq, int Hkv, int D, int mode,
                         float softmax_scale, void *workspace, size_t workspace_bytes,
                         int32_t *dev_status, void *stream) {
  if (mode != SFA_WITHIN && mode != SFA_CROSS && mode != SFA_TRANSIENT) return HD_ERR_INVALID_ARG;
  hd_status st = decode_shape_check(B, T, n, Hq, Hkv, D);
  if (st != HD_OK) return st;
  if (T > T_max) return HD_ERR_INVALID_ARG;
  if ((int64_t)n * T_max > (1LL << 31)) return HD_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(seq_tokens) & 3u) return HD_ERR_MISALIGNED;
  if (B == 0) return HD_OK;
  // T bounds every sequence's length: the plan and the cache view cover n*T rows
  CacheStorage cs = contiguous_storage(B, T, T_max, n, 0);
  cs.seq_tokens = seq_tokens;
  return decode_impl(q, k_cache, v_cache, o, lse, B, T, n, Hq, Hkv, D, mode, 0, cs,
                     softmax_scale, workspace, workspace_bytes, dev_status, stream);
}

hd_status sfa_decode_window_fwd(const void *q, const void *k_cache, const void *v_cache, void *o,
                                float *lse, int64_t B, int64_t T, int64_t T_max, int n, int Hq,
                                int Hkv, int D, int64_t window, float softmax_scale,
                                void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                void *stream) {
  if (window < 1) return HD_ERR_INVALID_ARG;
  hd_status st = decode_shape_check(B, T, n, Hq, Hkv, D);
  if (st != HD_OK) return st;
  if (T > T_max) return HD_ERR_INVALID_ARG;
  if ((int64_t)n * T_max > (1LL << 31)) return HD_ERR_UNSUPPORTED;
  if (B == 0) return HD_OK;
  return decode_impl(q, k_cache, v_cache, o, lse, B, T, n, Hq, Hkv, D, 2, window,
                     contiguous_storage(B, T, T_max, n, window_key_lo(n, T, window)),
                     softmax_scale, workspace, workspace_bytes, dev_status, stream);
}

// Rows a sequence of at most T_bound tokens streams in the paged decode.
static int64_t paged_stream_rows(int n, int64_t T_bound, int mode, int64_t window) {
  const int64_t all = (int64_t)n * T_bound;
  if (mode != 2) return all;
  const int64_t w = (int64_t)n * window + hd::kDecodeTileKeys - 1;  // window + tile rounding
  return w < all ? w : all;
}

size_t sfa_decode_paged_workspace_bytes(int64_t B, int n, int Hq, int Hkv, int D, int64_t T_bound,
                                        int mode, int64_t window) {
  if (B < 1 || mode < 0 || mode > 2 || (mode == 2 && window < 1) ||
      decode_shape_check(B, T_bound, n, Hq, Hkv, D) != HD_OK)
    return 0;
  return hd::plan_sfa_decode(B, n, Hq, Hkv, D, paged_stream_rows(n, T_bound, mode, window),
                             device_sms())
      .ws_bytes;
}

hd_status sfa_decode_paged_fwd(const void *q, const void *k_pages, const void *v_pages,
                               const int32_t *page_table, int max_pages_per_seq,
                               int64_t num_pages, int64_t page_rows, const int32_t *seq_tokens,
                               int64_t T_bound, void *o, float *lse, int64_t B, int n, int Hq,
                               int Hkv, int D, int mode, int64_t window, float softmax_scale,
                               void *workspace, size_t workspace_bytes, int32_t *dev_status,
                               void *stream) {
  if (mode < 0 || mode > 2 || (mode == 2 && window < 1)) return HD_ERR_INVALID_ARG;
  hd_status st = decode_shape_check(B, T_bound, n, Hq, Hkv, D);
  if (st != HD_OK) return st;
  if (num_pages < 1 || page_rows < 1 || num_pages > (1LL << 31) || page_rows > (1LL << 31))
    return HD_ERR_INVALID_ARG;
  if (page_table) {
    if (max_pages_per_seq < 1 || page_rows % hd::kDecodeTileKeys != 0) return HD_ERR_INVALID_ARG;
    if ((int64_t)max_pages_per_seq * page_rows < (int64_t)n * T_bound) return HD_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(page_table) & 3u) return HD_ERR_MISALIGNED;
  } else {
    // page b holds sequence b
    if (num_pages < B || page_rows < (int64_t)n * T_bound) return HD_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(seq_tokens) & 3u) return HD_ERR_MISALIGNED;
  if (B == 0) return HD_OK;
  CacheStorage cs{};
  cs.seq_tokens = seq_tokens;
  cs.page_table = page_table;
  cs.max_pages = page_table ? max_pages_per_seq : 0;
  cs.num_pages = num_pages;
  cs.page_rows = page_rows;
  cs.page_extent = page_rows;
  cs.stream_rows = paged_stream_rows(n, T_bound, mode, window);
  return decode_impl(q, k_pages, v_pages, o, lse, B, T_bound, n, Hq, Hkv, D, mode, window, cs,
                     softmax_scale, workspace, workspace_bytes, dev_status, stream);
}

}  // extern "C"
