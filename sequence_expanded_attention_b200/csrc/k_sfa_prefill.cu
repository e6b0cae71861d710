// k_sfa_prefill.cu -- Stream-Factorized Attention forward on tcgen05 tensor
// cores ("Hidden Decoding at Scale" review, "Method": most layers attend only
// within their own stream, O(nL^2); a few mix streams causally over the whole
// expanded sequence, O(n^2 L^2); README "Key Idea").
//
// One CTA computes one 128-row query tile of one attention problem:
//   within-stream: problem = (batch, query head, stream s); its sequence is
//     the L tokens of stream s, read through a 5-D TMA view
//     [B][L][n][H][D] of the token-major expanded tensor, so no copy or
//     transpose is made and each stream is a plain causal problem of length L
//     (the n-fold cost the pages give, not n^2);
//   cross-stream: problem = (batch, query head); its sequence is all N = nL
//     expanded positions, read through a 4-D view [B][N][H][D].
// Only causal (unmasked or diagonal) KV tiles are visited; the grid is
// ordered longest-first so the hardware scheduler balances the triangle.
//
// Roles (256 threads):
//   warp 0      TMA producer: Q once, then K_j / V_j tiles into a ring of
//               shared-memory stages (128B swizzle), completion on mbarriers.
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_j = Q K_j^T   tcgen05.mma SS, M=128 N=128 K=D  -> TMEM
//                 O  += P_j V_j   tcgen05.mma TS, A = P_j in TMEM (bf16, in
//                                 place of S_j), B = V_j (MN-major smem)
//               issue order S_0, S_1, PV_0, S_2, PV_1, ... so the tensor core
//               computes S_{j+1} while the softmax works on S_j.
//   warps 4..7  softmax, one thread per query row (TMEM lane = row): load
//               S_j, scale into the log2 domain, mask the diagonal tile, online
//               max/sum, write P_j (bf16) back to TMEM, rescale O in TMEM only
//               when the running max grew by more than 2^8, and finally
//               normalise O, stage it in shared memory and TMA-store it.
// TMEM: S double buffer in columns [0,128) and [128,256), O in [256,256+D).
#include <cfloat>

#include "hd_kernels.cuh"

namespace hd {

namespace {

constexpr int kBM = 128;      // query rows per tile (MMA M)
constexpr int kBN = 128;      // keys per KV tile
constexpr int kThreads = 256;
constexpr int kStages = 2;    // K/V ring depth
constexpr int kSoftmaxWarp0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr int kBoxBytes = 128 * 128;  // 128 rows x 128 B (64 bf16)
constexpr float kLn2 = 0.6931471805599453f;
// Rescale O only when the running row max grows by more than this (log2 units).
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct PCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // Q, K or V tile
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemK = kSmemQ + kTileBytes;
  static constexpr int kSmemV = kSmemK + kStages * kTileBytes;
  static constexpr int kSmemBar = kSmemV + kStages * kTileBytes;
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 1;
  static constexpr int kSmemTmemPtr = kSmemBar + kNumBars * 8;
  static constexpr int kSmemBytes = kSmemTmemPtr + 16;
  static constexpr size_t kDynSmem = 1024 + kSmemBytes;
};

struct Bars {
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_full, *mma_done;
};

__device__ __forceinline__ Bars carve_bars(uint8_t *base) {
  uint64_t *b = reinterpret_cast<uint64_t *>(base);
  Bars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = r.k_full + kStages;
  r.v_full = r.k_empty + kStages;
  r.v_empty = r.v_full + kStages;
  r.s_full = r.v_empty + kStages;  // [2]
  r.p_full = r.s_full + 2;         // [1]
  r.o_full = r.p_full + 1;         // [1]
  r.mma_done = r.o_full + 1;       // [1]
  return r;
}

// TMA coordinates of row `row0` of the problem's sequence for head `head`.
__device__ __forceinline__ void load_tile(void *dst, const CUtensorMap *m, uint64_t *bar, int dcol,
                                          int head, int stream, int row0, int batch, bool within) {
  if (within)
    tma_load_5d(dst, m, bar, dcol, head, stream, row0, batch);
  else
    tma_load_4d(dst, m, bar, dcol, head, row0, batch);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sfa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, const PrefillParams p) {
  using Cfg = PCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *smem = smem_raw + pad;
  uint8_t *sQ = smem + Cfg::kSmemQ;
  uint8_t *sK = smem + Cfg::kSmemK;
  uint8_t *sV = smem + Cfg::kSmemV;
  const Bars bar = carve_bars(smem + Cfg::kSmemBar);
  uint32_t *tmem_ptr_smem = reinterpret_cast<uint32_t *>(smem + Cfg::kSmemTmemPtr);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool within = (p.mode == 0);

  // Work item: heaviest query tiles first, heads of one KV group adjacent.
  const int64_t per = p.problems;
  const int qt = p.q_tiles - 1 - (int)(blockIdx.x / per);
  int64_t prob = blockIdx.x % per;
  const int h = (int)(prob % p.Hq);
  prob /= p.Hq;
  const int s = within ? (int)(prob % p.n) : 0;
  const int b = within ? (int)(prob / p.n) : (int)prob;
  const int g = h / p.G;
  const int q0 = qt * kBM;
  const int nt = qt + 1;  // causal: KV tiles 0 .. qt

  if (threadIdx.x == 0) {
    mbar_init(bar.q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar.k_full[i], 1);
      mbar_init(&bar.k_empty[i], 1);
      mbar_init(&bar.v_full[i], 1);
      mbar_init(&bar.v_empty[i], 1);
    }
    mbar_init(&bar.s_full[0], 1);
    mbar_init(&bar.s_full[1], 1);
    mbar_init(bar.p_full, 128);
    mbar_init(bar.o_full, 1);
    mbar_init(bar.mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_ptr_smem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr_smem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
      mbar_arrive_expect_tx(bar.q_full, Cfg::kTileBytes);
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c)
        load_tile(sQ + c * kBoxBytes, &tm_q, bar.q_full, c * 64, h, s, q0, b, within);
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int j = 0; j < nt; ++j) {
        const int st = j % kStages;
        const uint32_t ph = ((j / kStages) & 1) ^ 1;
        uint8_t *kd = sK + st * Cfg::kTileBytes;
        uint8_t *vd = sV + st * Cfg::kTileBytes;
        if (!(ok = mbar_wait(&bar.k_empty[st], ph))) break;
        mbar_arrive_expect_tx(&bar.k_full[st], Cfg::kTileBytes);
#pragma unroll
        for (int c = 0; c < Cfg::kBoxes; ++c)
          load_tile(kd + c * kBoxBytes, &tm_k, &bar.k_full[st], c * 64, g, s, j * kBN, b, within);
        k_issued = j + 1;
        if (!(ok = mbar_wait(&bar.v_empty[st], ph))) break;
        mbar_arrive_expect_tx(&bar.v_full[st], Cfg::kTileBytes);
#pragma unroll
        for (int c = 0; c < Cfg::kBoxes; ++c)
          load_tile(vd + c * kBoxBytes, &tm_v, &bar.v_full[st], c * 64, g, s, j * kBN, b, within);
        v_issued = j + 1;
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      // Every copy issued must land before the CTA can exit (in the normal
      // path the consumers have already waited for all of them).
      bool drained = mbar_wait(bar.q_full, 0);
      for (int j = max(0, k_issued - kStages); j < k_issued && drained; ++j)
        drained = mbar_wait(&bar.k_full[j % kStages], (j / kStages) & 1);
      for (int j = max(0, v_issued - kStages); j < v_issued && drained; ++j)
        drained = mbar_wait(&bar.v_full[j % kStages], (j / kStages) & 1);
      if (!drained) report(p.dev_status, kDevTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t k_base = smem_u32(sK);
      const uint32_t v_base = smem_u32(sV);
      bool ok = mbar_wait(bar.q_full, 0);
      auto issue_qk = [&](int j) -> bool {
        const int st = j % kStages;
        if (!mbar_wait(&bar.k_full[st], (j / kStages) & 1)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + ((j & 1) ? kColS1 : kColS0);
        const uint32_t kb = k_base + st * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_ss(d_tmem, smem_desc_sw128(q_base + off, 16, 1024),
                 smem_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.s_full[j & 1]);
        mma_commit(&bar.k_empty[st]);
        return true;
      };
      if (ok) {
        tc_fence_after();
        ok = issue_qk(0);
      }
      for (int j = 0; j < nt && ok; ++j) {
        if (j + 1 < nt && !(ok = issue_qk(j + 1))) break;
        const int st = j % kStages;
        if (!(ok = mbar_wait(bar.p_full, j & 1))) break;
        if (!(ok = mbar_wait(&bar.v_full[st], (j / kStages) & 1))) break;
        tc_fence_after();
        const uint32_t p_tmem = tmem + ((j & 1) ? kColS1 : kColS0);
        const uint32_t vb = v_base + st * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(tmem + kColO, p_tmem + kk * 8, smem_desc_sw128(vb + kk * 2048, kBoxBytes, 1024),
                 idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar.v_empty[st]);
        mma_commit(bar.o_full);
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      // All MMAs this thread issued must finish before TMEM is released.
      mma_commit(bar.mma_done);
      if (!mbar_wait(bar.mma_done, 0)) report(p.dev_status, kDevTimeout);
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ softmax
    const int wq = warp - kSoftmaxWarp0;  // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;       // query row inside the tile
    const int qpos = q0 + row;            // position inside the problem's sequence
    const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const uint32_t s_tmem = tmem + lane_addr + ((j & 1) ? kColS1 : kColS0);
      if (!(ok = mbar_wait(&bar.s_full[j & 1], (j >> 1) & 1))) break;
      tc_fence_after();
      float x[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(s_tmem + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(r[i]) * p.scale_log2;
      }
      if (j == nt - 1) {  // diagonal tile: keys after the query are masked
        const int lim = qpos - j * kBN;
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i > lim) x[i] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int i = 1; i < kBN; ++i) mx = fmaxf(mx, x[i]);
      const float m_cand = fmaxf(m, mx);
      const bool need = m_cand > m + kRescaleThreshold;
      const float m_new = need ? m_cand : m;
      const float base = (m_new == -INFINITY) ? 0.f : m_new;
      // P_j = 2^(x - base) in bf16, written over S_j: keys 64c .. 64c+63 pack
      // into the 32 columns starting at 32c (two keys per 32-bit column).
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kBN / 64; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2_approx(x[c * 64 + 2 * i] - base);
          const float p1 = ex2_approx(x[c * 64 + 2 * i + 1] - base);
          rs += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_tmem + c * 32, pk);
      }
      const float alpha = ex2_approx(m - base);
      l = l * alpha + rs;
      if (j > 0) {
        // O must hold PV_{j-1} before it is rescaled for the new max.
        if (!(ok = mbar_wait(bar.o_full, (j - 1) & 1))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            const uint32_t o_tmem = tmem + lane_addr + kColO + c * 32;
            tmem_ld32(o_tmem, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(o_tmem, r);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar.p_full);
      m = m_new;
    }
    if (ok) ok = mbar_wait(bar.o_full, (nt - 1) & 1);
    if (!ok) report(p.dev_status, kDevTimeout);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + kColO + c * 32, r);
        tmem_wait_ld();
        // 32 fp32 -> 16 packed bf16x2 = four 16-byte chunks of this row.
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l,
                              __uint_as_float(r[2 * i + 1]) * inv_l);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = c * 32 + q * 8;  // first element of the chunk
          uint8_t *dst = sQ + (col >> 6) * kBoxBytes + sw128_offset(row, (col & 63) >> 3);
          *reinterpret_cast<uint4 *>(dst) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                                                       pk[4 * q + 3]);
        }
      }
      if (p.lse && qpos < p.seq) {
        const int64_t pos = within ? (int64_t)qpos * p.n + s : (int64_t)qpos;
        p.lse[((int64_t)b * p.Hq + h) * p.N + pos] = (m + __log2f(l)) * kLn2;
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    if (ok && warp == kSoftmaxWarp0 && lane == 0) {
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c) {
        if (within)
          tma_store_5d(&tm_o, sQ + c * kBoxBytes, c * 64, h, s, q0, b);
        else
          tma_store_4d(&tm_o, sQ + c * kBoxBytes, c * 64, h, q0, b);
      }
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t prepare_prefill() {
  static int done_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (done_dev == dev) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(sfa_prefill_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PCfg<D>::kDynSmem);
  if (e == cudaSuccess) done_dev = dev;
  return e;
}

}  // namespace

cudaError_t launch_sfa_prefill(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                               const CUtensorMap &tm_v, const CUtensorMap &tm_o,
                               const PrefillParams &p, int D, cudaStream_t stream) {
  const int64_t ctas = p.problems * p.q_tiles;
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaError_t e;
  if (D == 128) {
    if ((e = prepare_prefill<128>()) != cudaSuccess) return e;
    sfa_prefill_kernel<128><<<(unsigned)ctas, kThreads, PCfg<128>::kDynSmem, stream>>>(
        tm_q, tm_k, tm_v, tm_o, p);
  } else {
    if ((e = prepare_prefill<64>()) != cudaSuccess) return e;
    sfa_prefill_kernel<64><<<(unsigned)ctas, kThreads, PCfg<64>::kDynSmem, stream>>>(
        tm_q, tm_k, tm_v, tm_o, p);
  }
  return cudaGetLastError();
}

}  // namespace hd
