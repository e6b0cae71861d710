// k_train_embed.cu -- the training-side ends of the Hidden Decoding path
// ("Hidden Decoding at Scale" review, "Method": next-token cross-entropy is
// applied only at the final-stream positions, the first n-1 streams get no
// loss; README "Key Idea" item 3):
//
//   final_stream_rows       out[b, t, :] = x[b, t*n + n-1, :]  (the rows that
//                           feed the LM head and the loss)
//   expand_embed_backward   grad_table_s[ids[b, t], :] += grad_x[b, t*n+s, :]
//                           (gradient of the n-table expansion)
//
// Both are HBM-bound.  The row copy moves 16-byte vectors, one warp per row.
// The gradient reads each bf16 gradient row once and adds it into its table
// row with vector fp32 reductions (red.global.add.v4.f32, resolved in L2);
// repeated ids (Zipf-hot tokens) meet in the same table row and the L2
// serialises their reductions.
#include "hd_kernels.cuh"

namespace hd {

namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__global__ void __launch_bounds__(kWarps * 32)
    final_stream_rows_kernel(const uint4 *__restrict__ x, int n, int64_t vec_per_row,
                             int64_t rows, uint4 *__restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t warp_stride = (int64_t)gridDim.x * kWarps;
  for (int64_t row = warp_global; row < rows; row += warp_stride) {
    const uint4 *src = x + (row * n + n - 1) * vec_per_row;  // row = b*L + t
    uint4 *dst = out + row * vec_per_row;
    int64_t v = lane;
    // four 16-byte loads in flight per lane, then the tail
    for (; v + 96 < vec_per_row; v += 128) {
      const uint4 a = ld_nc_v4(src + v), b = ld_nc_v4(src + v + 32);
      const uint4 c = ld_nc_v4(src + v + 64), d = ld_nc_v4(src + v + 96);
      dst[v] = a;
      dst[v + 32] = b;
      dst[v + 64] = c;
      dst[v + 96] = d;
    }
    for (; v < vec_per_row; v += 32) dst[v] = ld_nc_v4(src + v);
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __launch_bounds__(kWarps * 32)
    expand_embed_backward_kernel(const int64_t *__restrict__ ids, const uint4 *__restrict__ grad,
                                 GradTables tables, int n, int64_t V, int64_t vec_per_row,
                                 int64_t rows, int32_t *__restrict__ dev_status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t warp_stride = (int64_t)gridDim.x * kWarps;
  for (int64_t row = warp_global; row < rows; row += warp_stride) {  // row = (b*L + t)*n + s
    const int64_t token = row / n;
    const int s = (int)(row - token * n);
    const int64_t x = __ldg(ids + token);
    if (x < 0 || x >= V) {
      if (lane == 0 && s == 0) report(dev_status, kDevIdRange);
      continue;
    }
    const uint4 *src = grad + row * vec_per_row;
    float *dst = tables.ptr[s] + x * vec_per_row * 8;
    for (int64_t v = lane; v < vec_per_row; v += 32) {
      const uint4 g = ld_nc_v4(src + v);
      red_add_v4(dst + v * 8, bf16_lo(g.x), bf16_hi(g.x), bf16_lo(g.y), bf16_hi(g.y));
      red_add_v4(dst + v * 8 + 4, bf16_lo(g.z), bf16_hi(g.z), bf16_lo(g.w), bf16_hi(g.w));
    }
  }
}

int64_t grid_for(int64_t rows, int num_sms) {
  int64_t blocks = (rows + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)num_sms * 16;
  return blocks > cap ? cap : blocks;
}

}  // namespace

cudaError_t launch_final_stream_rows(const void *x, int64_t B, int64_t L, int n, int64_t d,
                                     void *out, cudaStream_t stream, int num_sms) {
  const int64_t rows = B * L;
  if (rows == 0) return cudaSuccess;
  final_stream_rows_kernel<<<(unsigned)grid_for(rows, num_sms), kWarps * 32, 0, stream>>>(
      static_cast<const uint4 *>(x), n, d / 8, rows, static_cast<uint4 *>(out));
  return cudaGetLastError();
}

cudaError_t launch_expand_embed_backward(const int64_t *ids, const void *grad, int64_t B,
                                         int64_t L, int n, int64_t V, int64_t d,
                                         const GradTables &tables, int32_t *dev_status,
                                         cudaStream_t stream, int num_sms) {
  const int64_t rows = B * L * n;
  if (rows == 0) return cudaSuccess;
  expand_embed_backward_kernel<<<(unsigned)grid_for(rows, num_sms), kWarps * 32, 0, stream>>>(
      ids, static_cast<const uint4 *>(grad), tables, n, V, d / 8, rows, dev_status);
  return cudaGetLastError();
}

}  // namespace hd
