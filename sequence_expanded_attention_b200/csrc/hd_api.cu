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

// Views of an expanded tensor X[B][N = n*L][H][D] for one SFA problem:
//   within-stream: 5-D [B][L][n][H][D], box (64 d, 1 head, 1 stream, 128 tokens, 1)
//   cross-stream:  4-D [B][N][H][D],    box (64 d, 1 head, 128 positions, 1)
hd_status make_prefill_map(CUtensorMap *m, const void *base, int64_t B, int64_t L, int n, int H,
                           int D, bool within) {
  const uint64_t e = 2;  // bf16 bytes
  const uint64_t N = (uint64_t)n * L;
  if (within) {
    const uint64_t dims[5] = {(uint64_t)D, (uint64_t)H, (uint64_t)n, (uint64_t)L, (uint64_t)B};
    const uint64_t strides[4] = {D * e, (uint64_t)H * D * e, (uint64_t)n * H * D * e,
                                 N * H * D * e};
    const uint32_t box[5] = {64, 1, 1, 128, 1};
    return make_map(m, base, 5, dims, strides, box);
  }
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, N, (uint64_t)B};
  const uint64_t strides[3] = {D * e, (uint64_t)H * D * e, N * H * D * e};
  const uint32_t box[4] = {64, 1, 128, 1};
  return make_map(m, base, 4, dims, strides, box);
}

// Decode cache view [B][n*T valid rows][Hkv][D] with batch stride n*T_max rows;
// rows past n*T read as zeros.  Box (64 d, 1 head, 64 keys, 1).
hd_status make_cache_map(CUtensorMap *m, const void *base, int64_t B, int64_t nkeys,
                         int64_t nrows_max, int Hkv, int D) {
  const uint64_t e = 2;
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)nkeys, (uint64_t)B};
  const uint64_t strides[3] = {D * e, (uint64_t)Hkv * D * e, (uint64_t)nrows_max * Hkv * D * e};
  const uint32_t box[4] = {64, 1, (uint32_t)hd::kDecodeTileKeys, 1};
  return make_map(m, base, 4, dims, strides, box);
}

float resolve_scale(float s, int D) { return s > 0.f ? s : 1.0f / std::sqrt((float)D); }

constexpr float kLog2e = 1.4426950408889634f;

// Shared body of the prefill entry points; mode 2 = cross-stream sliding window.
hd_status prefill_impl(const void *q, const void *k, const void *v, void *o, float *lse, int64_t B,
                       int64_t L, int n, int Hq, int Hkv, int D, int mode, int64_t window,
                       float softmax_scale, int32_t *dev_status, void *stream) {
  if (B < 0 || L < 0 || n < 1 || Hq < 1 || Hkv < 1) return HD_ERR_INVALID_ARG;
  if (n > hd::kMaxStreams || (D != 64 && D != 128) || Hq % Hkv != 0) return HD_ERR_UNSUPPORTED;
  if (B * L == 0) return HD_OK;
  if (!q || !k || !v || !o) return HD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return HD_ERR_MISALIGNED;
  const int64_t N = (int64_t)n * L;
  const bool within = (mode == SFA_WITHIN);
  // TMA coordinates are 32-bit and the grid is one CTA per (problem, tile pair).
  if (N > (1LL << 30) || B > (1LL << 20)) return HD_ERR_UNSUPPORTED;
  hd::PrefillParams p{};
  p.B = B;
  p.L = L;
  p.N = N;
  p.n = n;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.mode = mode;
  p.window = window;
  p.seq = (int)(within ? L : N);
  p.q_tiles = (p.seq + 127) / 128;
  p.problems = B * Hq * (within ? n : 1);
  p.scale_log2 = resolve_scale(softmax_scale, D) * kLog2e;
  p.lse = lse;
  p.dev_status = dev_status;
  CUtensorMap tq, tk, tv, to;
  hd_status st;
  if ((st = make_prefill_map(&tq, q, B, L, n, Hq, D, within)) != HD_OK) return st;
  if ((st = make_prefill_map(&tk, k, B, L, n, Hkv, D, within)) != HD_OK) return st;
  if ((st = make_prefill_map(&tv, v, B, L, n, Hkv, D, within)) != HD_OK) return st;
  if ((st = make_prefill_map(&to, o, B, L, n, Hq, D, within)) != HD_OK) return st;
  cudaError_t e = hd::launch_sfa_prefill(tq, tk, tv, to, p, D, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "sfa_prefill launch");
}

// First key row the n new positions of token T may attend under a sliding
// window of `window` tokens: the n streams of tokens T-window .. T-1.
int64_t window_key_lo(int n, int64_t T, int64_t window) {
  const int64_t t0 = T - window;
  return t0 > 0 ? (int64_t)n * t0 : 0;
}

// Shared body of the decode entry points; mode 2 = cross-stream sliding window.
hd_status decode_impl(const void *q, const void *k_cache, const void *v_cache, void *o,
                      float *lse, int64_t B, int64_t T, int64_t T_max, int n, int Hq, int Hkv,
                      int D, int mode, int64_t window, float softmax_scale, void *workspace,
                      size_t workspace_bytes, int32_t *dev_status, void *stream) {
  if (B < 0 || n < 1 || Hq < 1 || Hkv < 1 || T < 1 || T > T_max) return HD_ERR_INVALID_ARG;
  if (n > hd::kMaxStreams || (D != 64 && D != 128) || Hq % Hkv != 0) return HD_ERR_UNSUPPORTED;
  if (B == 0) return HD_OK;
  if (!q || !k_cache || !v_cache || !o) return HD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || !aligned16(workspace))
    return HD_ERR_MISALIGNED;
  if ((int64_t)n * T_max > (1LL << 31) || B > (1LL << 16)) return HD_ERR_UNSUPPORTED;
  const int64_t key_lo = (mode == 2) ? window_key_lo(n, T, window) : 0;
  const hd::DecodePlan pl = hd::plan_sfa_decode(B, n, Hq, Hkv, D, T, device_sms(), key_lo);
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
  p.nkeys = (int64_t)n * T;
  p.key_lo = key_lo;
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
  if ((st = make_cache_map(&tk, k_cache, B, p.nkeys, (int64_t)n * T_max, Hkv, D)) != HD_OK)
    return st;
  if ((st = make_cache_map(&tv, v_cache, B, p.nkeys, (int64_t)n * T_max, Hkv, D)) != HD_OK)
    return st;
  cudaError_t e = hd::launch_sfa_decode(tk, tv, p, D, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HD_OK : cuda_fail(e, "sfa_decode launch");
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

int hd_version(void) { return (1 << 16) | 0; }

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

hd_status sfa_prefill_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                          int64_t B, int64_t L, int n, int Hq, int Hkv, int D, int mode,
                          float softmax_scale, int32_t *dev_status, void *stream) {
  if (mode != SFA_WITHIN && mode != SFA_CROSS) return HD_ERR_INVALID_ARG;
  return prefill_impl(q, k, v, o, lse, B, L, n, Hq, Hkv, D, mode, 0, softmax_scale, dev_status,
                      stream);
}

hd_status sfa_prefill_window_fwd(const void *q, const void *k, const void *v, void *o,
                                 float *lse, int64_t B, int64_t L, int n, int Hq, int Hkv, int D,
                                 int64_t window, float softmax_scale, int32_t *dev_status,
                                 void *stream) {
  if (window < 1) return HD_ERR_INVALID_ARG;
  return prefill_impl(q, k, v, o, lse, B, L, n, Hq, Hkv, D, 2, window, softmax_scale,
                      dev_status, stream);
}

size_t sfa_decode_workspace_bytes(int64_t B, int n, int Hq, int Hkv, int D, int64_t T) {
  if (B < 1 || n < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || T < 1 || (D != 64 && D != 128))
    return 0;
  return hd::plan_sfa_decode(B, n, Hq, Hkv, D, T, device_sms()).ws_bytes;
}

size_t sfa_decode_window_workspace_bytes(int64_t B, int n, int Hq, int Hkv, int D, int64_t T,
                                         int64_t window) {
  if (B < 1 || n < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || T < 1 || window < 1 ||
      (D != 64 && D != 128))
    return 0;
  return hd::plan_sfa_decode(B, n, Hq, Hkv, D, T, device_sms(), window_key_lo(n, T, window))
      .ws_bytes;
}

hd_status sfa_decode_fwd(const void *q, const void *k_cache, const void *v_cache, void *o,
                         float *lse, int64_t B, int64_t T, int64_t T_max, int n, int Hq, int Hkv,
                         int D, int mode, float softmax_scale, void *workspace,
                         size_t workspace_bytes, int32_t *dev_status, void *stream) {
  if (mode != SFA_WITHIN && mode != SFA_CROSS) return HD_ERR_INVALID_ARG;
  return decode_impl(q, k_cache, v_cache, o, lse, B, T, T_max, n, Hq, Hkv, D, mode, 0,
                     softmax_scale, workspace, workspace_bytes, dev_status, stream);
}

hd_status sfa_decode_window_fwd(const void *q, const void *k_cache, const void *v_cache, void *o,
                                float *lse, int64_t B, int64_t T, int64_t T_max, int n, int Hq,
                                int Hkv, int D, int64_t window, float softmax_scale,
                                void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                void *stream) {
  if (window < 1) return HD_ERR_INVALID_ARG;
  return decode_impl(q, k_cache, v_cache, o, lse, B, T, T_max, n, Hq, Hkv, D, 2, window,
                     softmax_scale, workspace, workspace_bytes, dev_status, stream);
}

}  // extern "C"
