// k_sfa_decode.cu -- SFA decode: the n new expanded positions of one token
// attend the retained expanded KV cache (review "Method": intermediate
// streams' KV is kept as context; "Limitations"/"Notes": in small-batch
// decode the retained cache is the cost, and the streams' extra arithmetic
// rides on otherwise idle compute).
//
// Bound by HBM: every valid cache row of a (batch, KV head) is read exactly
// once, in both modes.  One CTA owns one (batch, KV head, row group, key
// split): its 16 query rows are the n streams x (Hq/Hkv) heads that share the
// KV head, so each K/V tile serves all of them (within-stream mode masks each
// row down to its own stream: row s keeps keys p' with p' % n == s).
//
// Pipeline: a producer warp streams 64-key K/V tiles with TMA (128B swizzle)
// through a ring of shared-memory stages; four consumer warps each take 16
// keys of a tile and run QK^T and PV on warp-level bf16 tensor-core MMAs
// (m16n8k16, fp32 accumulate) with an online softmax whose row max is reduced
// across the quad of lanes that share a row by warp shuffles.  The four warps'
// partial results merge in shared memory; with several key splits a small
// combine kernel merges the splits through their log-sum-exp.
#include <algorithm>
#include <cfloat>

#include "hd_kernels.cuh"

namespace hd {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct DecodeCfg {
  static constexpr int kBoxes = D / 64;                 // 64-wide (128 B) TMA boxes per row
  static constexpr int kTileBytes = kBoxes * kDecodeTileKeys * 128;  // one K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = (D == 128) ? 3 : 6;   // ~96 KB: two CTAs per SM
};

template <int D>
constexpr size_t decode_smem_bytes() {
  return 1024 /* alignment slack */ + (size_t)DecodeCfg<D>::kStages * DecodeCfg<D>::kStageBytes +
         2 * DecodeCfg<D>::kStages * sizeof(uint64_t) + 4 * kConsumerWarps * kDecodeRows * sizeof(float);
}

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16 *p) {
  return *reinterpret_cast<const uint32_t *>(p);
}

template <int D>
__global__ void __launch_bounds__(kThreads)
    sfa_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using Cfg = DecodeCfg<D>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *smem = smem_raw + pad;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * Cfg::kStageBytes);
  uint64_t *empty = full + S;
  float *red_m = reinterpret_cast<float *>(empty + S);  // [warps][16]
  float *red_l = red_m + kConsumerWarps * kDecodeRows;  // [warps][16]
  float *row_M = red_l + kConsumerWarps * kDecodeRows;  // [16]
  float *row_L = row_M + kDecodeRows;                   // [16]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Row groups fastest: the CTAs of one (KV head, key split) that differ only
  // in their query rows launch together and share each K/V tile through L2.
  const int rg = blockIdx.x % p.RG, split = blockIdx.x / p.RG;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int tile0 = split * p.tiles_per_split;
  // This sequence's extent: its token count (variable lengths), the first row
  // its queries may attend (sliding window), and the first row streamed (with
  // a page table rounded down to a tile, so no tile straddles two pages).
  int64_t Tb = p.T;
  if (p.seq_tokens) {
    const int32_t t = p.seq_tokens[b];
    if (t < 1 || t > p.T) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) report(p.dev_status, kDevBadLength);
      Tb = 0;  // defined output: zero rows
    } else {
      Tb = t;
    }
  }
  const int64_t nkeys_b = (int64_t)p.n * Tb;
  const int64_t key_lo_b = (p.mode == 2 && Tb > p.window) ? (int64_t)p.n * (Tb - p.window) : 0;
  const int64_t key_base_b = p.page_table ? key_lo_b / kDecodeTileKeys * kDecodeTileKeys : key_lo_b;
  const int tiles_b =
      nkeys_b > key_base_b ? (int)((nkeys_b - key_base_b + kDecodeTileKeys - 1) / kDecodeTileKeys) : 0;
  const int tile1 = min(tile0 + p.tiles_per_split, min(tiles_b, p.ntiles));
  const int ntl = max(0, tile1 - tile0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int i = 0; i < ntl; ++i) {
        const int st = i % S;
        if (!mbar_wait(&empty[st], ((i / S) & 1) ^ 1)) {
          report(p.dev_status, kDevTimeout);
          break;
        }
        mbar_arrive_expect_tx(&full[st], Cfg::kStageBytes);
        // Logical cache row of the tile -> (page, row inside the page).  A page
        // id outside the pool reads as zeros (TMA fill) and is reported.
        const int64_t row0 = key_base_b + (int64_t)(tile0 + i) * kDecodeTileKeys;
        int page = b;
        int64_t prow = row0;
        if (p.page_table) {
          const int64_t blk = row0 / p.page_rows;
          const int32_t pg = blk < p.max_pages ? p.page_table[(int64_t)b * p.max_pages + blk] : -1;
          if (pg < 0 || pg >= p.num_pages) {
            report(p.dev_status, kDevPageRange);
            page = (int)p.num_pages;
          } else {
            page = pg;
          }
          prow = row0 - blk * p.page_rows;
        }
        uint8_t *kt = smem + st * Cfg::kStageBytes;
        uint8_t *vt = kt + Cfg::kTileBytes;
#pragma unroll
        for (int c = 0; c < Cfg::kBoxes; ++c) {
          tma_load_4d(kt + c * kDecodeTileKeys * 128, &tm_k, &full[st], c * 64, g, (int)prow, page);
          tma_load_4d(vt + c * kDecodeTileKeys * 128, &tm_v, &full[st], c * 64, g, (int)prow, page);
        }
        issued = i + 1;
      }
      // Before the CTA may exit, every issued copy must have landed (normally
      // they all have: the consumers waited for them).
      for (int i = max(0, issued - S); i < issued; ++i)
        if (!mbar_wait(&full[i % S], (i / S) & 1)) {
          report(p.dev_status, kDevTimeout);
          break;
        }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int qr[2] = {lane >> 2, (lane >> 2) + 8};
    bool valid[2];
    int srow[2];
    int64_t pq[2];
    const __nv_bfloat16 *qrow[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int rglob = rg * kDecodeRows + qr[j];
      valid[j] = rglob < p.R;
      const int s = valid[j] ? rglob / p.G : 0;
      const int h = g * p.G + (valid[j] ? rglob % p.G : 0);
      srow[j] = s;
      pq[j] = (int64_t)p.n * (Tb - 1) + s;
      qrow[j] = p.q + (((int64_t)b * p.n + s) * p.Hq + h) * D;
    }
    uint32_t qf[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int col = kk * 16 + 2 * (lane & 3);
      qf[kk][0] = valid[0] ? ld_u32(qrow[0] + col) : 0u;
      qf[kk][1] = valid[1] ? ld_u32(qrow[1] + col) : 0u;
      qf[kk][2] = valid[0] ? ld_u32(qrow[0] + col + 8) : 0u;
      qf[kk][3] = valid[1] ? ld_u32(qrow[1] + col + 8) : 0u;
    }

    float oacc[D / 8][4];
#pragma unroll
    for (int dn = 0; dn < D / 8; ++dn) oacc[dn][0] = oacc[dn][1] = oacc[dn][2] = oacc[dn][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};

    // Streams of this thread's four key offsets {0, 1, 8, 9} within its 16
    // keys of the tile; a tile advances them by kDecodeTileKeys mod n, so
    // they are stepped with a compare-subtract instead of a division per key.
    const int kmod = (int)((key_base_b + (int64_t)tile0 * kDecodeTileKeys + warp * 16 +
                            2 * (lane & 3)) % p.n);
    const int kmod_step = kDecodeTileKeys % p.n;
    int kst[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) kst[t] = (kmod + (t >> 1) * 8 + (t & 1)) % p.n;
    for (int i = 0; i < ntl; ++i) {
      const int st = i % S;
      if (!mbar_wait(&full[st], (i / S) & 1)) {
        report(p.dev_status, kDevTimeout);
        break;
      }
      const uint32_t kt = smem_u32(smem + st * Cfg::kStageBytes);
      const uint32_t vt = kt + Cfg::kTileBytes;

      // S = Q K^T for this warp's 16 keys (two n-tiles of 8).
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int mi = lane >> 3;
        const uint32_t key = warp * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t chunk = 2 * kk + (mi & 1);
          uint32_t b00, b01, b10, b11;
          ldmatrix_x4(kt + (chunk >> 3) * (kDecodeTileKeys * 128) + sw128_offset(key, chunk & 7),
                      b00, b01, b10, b11);
          mma_bf16_16816(sacc[0], qf[kk], b00, b01);
          mma_bf16_16816(sacc[1], qf[kk], b10, b11);
        }
      }

      // Mask, scale into the log2 domain, online softmax.
      const int64_t kbase =
          key_base_b + (int64_t)(tile0 + i) * kDecodeTileKeys + warp * 16 + 2 * (lane & 3);
      float x[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = e >> 1;
          const int off = nt * 8 + (e & 1);
          const int64_t pk = kbase + off;
          bool ok = valid[j] && pk < nkeys_b && pk <= pq[j] && pk >= key_lo_b;
          const int kstream = kst[nt * 2 + (e & 1)];
          if (p.mode == 0) {
            ok = ok && kstream == srow[j];
          } else if (p.mode == 3) {
            // earlier tokens only through their final stream; the new token's
            // own streams up to s (pk <= pq above)
            ok = ok && (pk >= nkeys_b - p.n || kstream == p.n - 1);
          }
          x[nt][e] = ok ? sacc[nt][e] * p.scale_log2 : -INFINITY;
        }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        kst[t] += kmod_step;
        if (kst[t] >= p.n) kst[t] -= p.n;
      }
      float mx[2];
      mx[0] = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      mx[1] = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 1));
        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], 2));
      }
      float alpha[2], base[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float mn = fmaxf(m[j], mx[j]);
        base[j] = (mn == -INFINITY) ? 0.f : mn;
        alpha[j] = ex2_approx(m[j] - base[j]);
        m[j] = mn;
      }
      float pr[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[nt][e] = ex2_approx(x[nt][e] - base[e >> 1]);
      l[0] = l[0] * alpha[0] + (pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1]);
      l[1] = l[1] * alpha[1] + (pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3]);
#pragma unroll
      for (int dn = 0; dn < D / 8; ++dn) {
        oacc[dn][0] *= alpha[0];
        oacc[dn][1] *= alpha[0];
        oacc[dn][2] *= alpha[1];
        oacc[dn][3] *= alpha[1];
      }
      uint32_t pa[4];
      pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
      pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
      pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
      pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);

      // V rows of this warp's 16 keys outside [key_lo_b, nkeys_b) may hold
      // anything (stale pages, unwritten rows): zero them so that a zero
      // probability cannot meet a NaN in the sum.
      {
        const int64_t r0w = key_base_b + (int64_t)(tile0 + i) * kDecodeTileKeys + warp * 16;
        if (r0w < key_lo_b || r0w + 16 > nkeys_b) {
          uint8_t *vgen = smem + st * Cfg::kStageBytes + Cfg::kTileBytes;
          for (int idx = lane; idx < 16 * Cfg::kBoxes * 8; idx += 32) {
            const int r = idx / (Cfg::kBoxes * 8), rem = idx % (Cfg::kBoxes * 8);
            const int64_t row = r0w + r;
            if (row < key_lo_b || row >= nkeys_b)
              *reinterpret_cast<uint4 *>(vgen + (rem >> 3) * (kDecodeTileKeys * 128) +
                                         sw128_offset(warp * 16 + r, rem & 7)) =
                  make_uint4(0, 0, 0, 0);
          }
          // These generic-proxy stores precede the next TMA (async-proxy)
          // write into this stage once it is released: order them for it.
          fence_proxy_async_smem();
          __syncwarp();
        }
      }
      // O += P V over the same 16 keys.
      {
        const int mi = lane >> 3;
        const uint32_t key = warp * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          const uint32_t chunk = 2 * dp + (mi >> 1);
          uint32_t v0, v1, v2, v3;
          ldmatrix_x4_trans(
              vt + (chunk >> 3) * (kDecodeTileKeys * 128) + sw128_offset(key, chunk & 7), v0, v1,
              v2, v3);
          mma_bf16_16816(oacc[2 * dp], pa, v0, v1);
          mma_bf16_16816(oacc[2 * dp + 1], pa, v2, v3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }

    // Merge the four warps: row max, rescale, sum in shared memory.
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      l[j] += __shfl_xor_sync(0xffffffffu, l[j], 1);
      l[j] += __shfl_xor_sync(0xffffffffu, l[j], 2);
    }
    if ((lane & 3) == 0) {
      red_m[warp * kDecodeRows + qr[0]] = m[0];
      red_m[warp * kDecodeRows + qr[1]] = m[1];
      red_l[warp * kDecodeRows + qr[0]] = l[0];
      red_l[warp * kDecodeRows + qr[1]] = l[1];
    }
    // The merge buffer overlays stage 0: every consumer warp must be done
    // reading its last tile (which may sit in stage 0) before it is cleared.
    named_bar_sync(1, kConsumerWarps * 32);
    float *obuf = reinterpret_cast<float *>(smem);  // [16][D]
    for (int idx = threadIdx.x; idx < kDecodeRows * D; idx += kConsumerWarps * 32) obuf[idx] = 0.f;
    named_bar_sync(1, kConsumerWarps * 32);
    if (threadIdx.x < kDecodeRows) {
      const int r = threadIdx.x;
      float M = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red_m[w * kDecodeRows + r]);
      float Lsum = 0.f;
      if (M != -INFINITY)
        for (int w = 0; w < kConsumerWarps; ++w)
          Lsum += red_l[w * kDecodeRows + r] * ex2_approx(red_m[w * kDecodeRows + r] - M);
      row_M[r] = M;
      row_L[r] = Lsum;
    }
    float f[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float M = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red_m[w * kDecodeRows + qr[j]]);
      f[j] = (M == -INFINITY) ? 0.f : ex2_approx(m[j] - M);
    }
#pragma unroll
    for (int dn = 0; dn < D / 8; ++dn) {
      const int col = dn * 8 + 2 * (lane & 3);
      atomicAdd(&obuf[qr[0] * D + col], oacc[dn][0] * f[0]);
      atomicAdd(&obuf[qr[0] * D + col + 1], oacc[dn][1] * f[0]);
      atomicAdd(&obuf[qr[1] * D + col], oacc[dn][2] * f[1]);
      atomicAdd(&obuf[qr[1] * D + col + 1], oacc[dn][3] * f[1]);
    }
    named_bar_sync(1, kConsumerWarps * 32);

    const bool final_out = (p.splits == 1);
    const int64_t ws_row0 =
        ((((int64_t)b * p.Hkv + g) * p.RG + rg) * p.splits + split) * kDecodeRows;
    for (int idx = threadIdx.x; idx < kDecodeRows * D; idx += kConsumerWarps * 32) {
      const int r = idx / D, col = idx % D;
      const int rglob = rg * kDecodeRows + r;
      if (rglob >= p.R) continue;
      const float Lr = row_L[r];
      const float val = Lr > 0.f ? obuf[idx] / Lr : 0.f;
      if (final_out) {
        const int s = rglob / p.G, h = g * p.G + rglob % p.G;
        p.o[(((int64_t)b * p.n + s) * p.Hq + h) * D + col] = __float2bfloat16_rn(val);
        if (col == 0 && p.lse)
          p.lse[((int64_t)b * p.Hq + h) * p.n + s] = (row_M[r] + __log2f(Lr)) * kLn2;
      } else {
        p.ws_o[(ws_row0 + r) * D + col] = val;
        if (col == 0) p.ws_lse[ws_row0 + r] = Lr > 0.f ? row_M[r] + __log2f(Lr) : -INFINITY;
      }
    }
  }
}

// Merge the key splits of one query row through their log2-sum-exp:
// o = sum_i 2^(lse_i - M) o_i / sum_i 2^(lse_i - M).  One CTA per row of a
// (batch, KV head, row group); the splits' LSEs are staged in shared memory
// and every thread owns one output column.
template <int D>
__global__ void __launch_bounds__(D) sfa_decode_combine_kernel(const DecodeParams p) {
  __shared__ float lse_s[kDecodeMaxSplits];
  __shared__ float stat[2];
  const int r = blockIdx.x % kDecodeRows;
  const int unit = blockIdx.x / kDecodeRows;  // ((b * Hkv + g) * RG + rg)
  const int rg = unit % p.RG;
  const int g = (unit / p.RG) % p.Hkv;
  const int b = unit / (p.RG * p.Hkv);
  const int rglob = rg * kDecodeRows + r;
  if (rglob >= p.R) return;  // padding row of the last row group (whole CTA)
  const int64_t base = (int64_t)unit * p.splits;
  for (int i = threadIdx.x; i < p.splits; i += D) lse_s[i] = p.ws_lse[(base + i) * kDecodeRows + r];
  __syncthreads();
  if (threadIdx.x < 32) {
    float M = -INFINITY;
    for (int i = threadIdx.x; i < p.splits; i += 32) M = fmaxf(M, lse_s[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Lsum = 0.f;
    for (int i = threadIdx.x; i < p.splits; i += 32) Lsum += ex2_approx(lse_s[i] - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    if (threadIdx.x == 0) {
      stat[0] = M;
      stat[1] = Lsum;
    }
  }
  __syncthreads();
  const float M = stat[0], Lsum = stat[1];
  const int col = threadIdx.x;
  const int s = rglob / p.G, h = g * p.G + rglob % p.G;
  if (M == -INFINITY) {  // no split saw an allowed key (an invalid sequence length)
    p.o[(((int64_t)b * p.n + s) * p.Hq + h) * D + col] = __float2bfloat16_rn(0.f);
    if (col == 0 && p.lse) p.lse[((int64_t)b * p.Hq + h) * p.n + s] = -INFINITY;
    return;
  }
  const float *src = p.ws_o + (base * kDecodeRows + r) * D + col;
  float acc = 0.f;
#pragma unroll 4
  for (int i = 0; i < p.splits; ++i)
    acc += ex2_approx(lse_s[i] - M) * src[(int64_t)i * kDecodeRows * D];
  p.o[(((int64_t)b * p.n + s) * p.Hq + h) * D + col] = __float2bfloat16_rn(acc / Lsum);
  if (col == 0 && p.lse) p.lse[((int64_t)b * p.Hq + h) * p.n + s] = (M + __log2f(Lsum)) * kLn2;
}

template <int D>
int decode_ctas_per_sm() {
  static int cached = 0;
  if (cached == 0) {
    int nb = 0;
    cudaFuncSetAttribute(sfa_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)decode_smem_bytes<D>());
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, sfa_decode_kernel<D>, kThreads,
                                                      decode_smem_bytes<D>()) != cudaSuccess ||
        nb < 1)
      nb = 1;
    cached = nb;
  }
  return cached;
}

}  // namespace

DecodePlan plan_sfa_decode(int64_t B, int n, int Hq, int Hkv, int D, int64_t rows,
                           int num_sms) {
  DecodePlan pl{};
  const int G = Hq / Hkv;
  const int R = n * G;
  pl.RG = (R + kDecodeRows - 1) / kDecodeRows;
  pl.ntiles = (int)((rows + kDecodeTileKeys - 1) / kDecodeTileKeys);
  const int64_t units = B * Hkv * pl.RG;
  // Two resident CTAs per SM (the stage ring is sized for it).  Pick the split
  // count with the smallest modelled time, in units of one tile streamed by
  // one CTA at its share of HBM bandwidth:
  //   waves(s) * (kFixedTiles + tiles_per_split(s)) + combine(s)
  // kFixedTiles is a CTA's start-up and merge cost (pipeline fill, Q load,
  // partial write); the combine term charges the split partials' traffic.
  constexpr double kFixedTiles = 5.0;
  const int64_t slots = (int64_t)num_sms * 2;
  const int max_splits = std::max(1, std::min(pl.ntiles, kDecodeMaxSplits));
  int best = 1;
  double best_cost = 1e300;
  for (int s = 1; s <= max_splits; ++s) {
    const int tps = (pl.ntiles + s - 1) / s;
    if ((pl.ntiles + tps - 1) / tps != s) continue;  // s splits would leave one empty
    const int64_t ctas = units * s;
    const int64_t waves = (ctas + slots - 1) / slots;
    const double cost = (double)waves * (kFixedTiles + tps) +
                        (s > 1 ? 0.5 * (double)s * (double)units / (double)slots : 0.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  pl.splits = best;
  pl.tiles_per_split = (pl.ntiles + best - 1) / best;
  if (pl.splits > 1) {
    const size_t rows = (size_t)units * pl.splits * kDecodeRows;
    pl.ws_bytes = rows * D * sizeof(float) + rows * sizeof(float);
  } else {
    pl.ws_bytes = 0;
  }
  return pl;
}

cudaError_t launch_sfa_decode(const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                              const DecodeParams &p, int D, cudaStream_t stream) {
  const dim3 grid(p.splits * p.RG, p.Hkv, p.B);
  if (D == 128) {
    decode_ctas_per_sm<128>();
    sfa_decode_kernel<128><<<grid, kThreads, decode_smem_bytes<128>(), stream>>>(tm_k, tm_v, p);
    if (p.splits > 1)
      sfa_decode_combine_kernel<128><<<p.B * p.Hkv * p.RG * kDecodeRows, 128, 0, stream>>>(p);
  } else {
    decode_ctas_per_sm<64>();
    sfa_decode_kernel<64><<<grid, kThreads, decode_smem_bytes<64>(), stream>>>(tm_k, tm_v, p);
    if (p.splits > 1)
      sfa_decode_combine_kernel<64><<<p.B * p.Hkv * p.RG * kDecodeRows, 64, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace hd
