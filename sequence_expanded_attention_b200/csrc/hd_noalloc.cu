// hd_noalloc.cu -- sfa_decode_fwd_noalloc: the decode step for callers that
// cannot provide device scratch memory.
//
// Some host programs cannot hand this library a workspace: plugin interfaces
// of inference engines that give a kernel only its input and output buffers,
// and serving runtimes that reserve all device memory when they start and
// forbid allocation on the request path (cudaMalloc may synchronise the
// device and its latency is unbounded).  For them the key-split partial
// results live in one file-scope device array of fixed size, which every GPU
// that loads this library keeps until the process exits.
#include <mutex>

#include "../../include/hd.h"
#include "hd_kernels.cuh"

namespace {

constexpr size_t kScratchBytes = HD_DECODE_NOALLOC_SCRATCH_BYTES;  // 32 MiB

// The shared scratch.  In host code this name is only a stand-in for the
// device array, not its address: the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device, looked up once
// per device (with that device current).
hd_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return HD_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return HD_OK;
}

}  // namespace

extern "C" {

size_t sfa_decode_noalloc_scratch_bytes(void) { return kScratchBytes; }

hd_status sfa_decode_fwd_noalloc(const void *q, const void *k_cache, const void *v_cache, void *o,
                                 float *lse, int64_t B, int64_t T, int64_t T_max, int n, int Hq,
                                 int Hkv, int D, int mode, float softmax_scale,
                                 int32_t *dev_status, void *stream) {
  const size_t need = sfa_decode_workspace_bytes(B, n, Hq, Hkv, D, T);
  if (need > kScratchBytes) return HD_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (need > 0) {
    const hd_status st = scratch_address(&scratch);
    if (st != HD_OK) return st;
  }
  return sfa_decode_fwd(q, k_cache, v_cache, nullptr, o, lse, B, T, T_max, n, Hq, Hkv, D, mode,
                        softmax_scale, scratch, need > 0 ? kScratchBytes : 0, dev_status, stream);
}

}  // extern "C"
