// k_expand_embed.cu -- Hidden Decoding token expansion: every token id picks
// one row from each of n independent embedding tables, and the n rows are
// written token-major (expanded position t*n + s holds table s's row).
// ("Hidden Decoding at Scale" review, "Method"; Tencent/Sequential-Hidden-
// Decoding README, "Key Idea" item 1.)
//
// Pure data movement, bound by HBM: each output row is read once from a table
// and written once.  One warp moves one row with 16-byte vector accesses; a
// lane keeps kUnroll loads in flight before storing.  Table reads use the
// read-only path (hot Zipf ids then hit L2); output stores are streaming.
#include "hd_kernels.cuh"

namespace hd {

namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 8;

__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_cs_v4(uint4 *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__global__ void __launch_bounds__(kWarps * 32)
    expand_embed_kernel(const int64_t *__restrict__ ids, ExpandTables tables, int n, int64_t V,
                        int64_t vec_per_row, int64_t rows, uint4 *__restrict__ out,
                        int32_t *__restrict__ dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t warp_stride = (int64_t)gridDim.x * kWarps;
  for (int64_t row = warp_global; row < rows; row += warp_stride) {
    const int64_t token = row / n;
    const int s = (int)(row - token * n);
    const int64_t x = __ldg(ids + token);
    uint4 *dst = out + row * vec_per_row;
    if (x < 0 || x >= V) {
      const uint4 z = make_uint4(0, 0, 0, 0);
      for (int64_t v = lane; v < vec_per_row; v += 32) st_cs_v4(dst + v, z);
      if (lane == 0 && s == 0) report(dev_status, kDevIdRange);
      continue;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(tables.ptr[s]) + x * vec_per_row;
    int64_t v = lane;
    for (; v + 32 * (kUnroll - 1) < vec_per_row; v += 32 * kUnroll) {
      uint4 buf[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) buf[u] = ld_nc_v4(src + v + 32 * u);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) st_cs_v4(dst + v + 32 * u, buf[u]);
    }
    for (; v < vec_per_row; v += 32) st_cs_v4(dst + v, ld_nc_v4(src + v));
  }
}

}  // namespace

cudaError_t launch_expand_embed(const int64_t *ids, int64_t B, int64_t L, const ExpandTables &tables,
                                int n, int64_t V, int64_t d, void *out, int32_t *dev_status,
                                cudaStream_t stream, int num_sms) {
  const int64_t rows = B * L * n;
  if (rows == 0) return cudaSuccess;
  const int64_t vec_per_row = d / 8;  // 8 bf16 per 16-byte vector
  // Enough resident warps to keep ~kUnroll x 16 B x 32 lanes in flight per
  // warp on every SM; a grid-stride loop covers the rest.
  int64_t blocks = (rows + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)num_sms * 16;
  if (blocks > cap) blocks = cap;
  expand_embed_kernel<<<(unsigned)blocks, kWarps * 32, 0, stream>>>(
      ids, tables, n, V, vec_per_row, rows, reinterpret_cast<uint4 *>(out), dev_status);
  return cudaGetLastError();
}

}  // namespace hd
