// k_sfa_backward.cu -- Stream-Factorized Attention backward on tcgen05 tensor
// cores ("Hidden Decoding at Scale" review, "Method": the model trains end to
// end with the next-token loss at the final-stream positions, so gradients
// pass back through every within-stream and cross-stream layer).
//
// For each attention problem (the within-stream (batch, head, stream)
// problems or the cross-stream (batch, head) problems of the forward pass),
// with P = exp(scale Q K^T - LSE) on the allowed pairs:
//   dV = P^T dO,  dP = dO V^T,  Delta = rowsum(dO * O),
//   dS = P * (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three launches, in stream order:
//   bwd_rowstat   per query row: -LSE * log2(e) and -Delta, two arrays in
//                 problem order with the rows padded to a multiple of 128
//                 (padding: -LSE = -inf, so every padded row has P = 0).
//   sfa_bwd_dkdv  one CTA per (KV problem, 128-key tile): K and V stay in
//                 shared memory; the CTA streams every 64-row query chunk that
//                 sees the tile, for each query head of the KV head's group,
//                 and accumulates dV and dK in TMEM.
//   sfa_bwd_dq    one CTA per (query problem, 128-query tile): Q and dO stay in
//                 shared memory; the CTA streams the 64-row key chunks the
//                 tile sees and accumulates dQ in TMEM.
// Each output row is written by exactly one CTA: no atomics, and the result
// does not depend on scheduling.  S and dP are recomputed in both kernels
// (7 tile GEMMs per pair of tiles instead of 5); in exchange dQ needs no
// fp32 accumulation buffer in HBM and no reduction traffic through L2.
//
// Roles (320 threads), the same in both kernels:
//   warps 0-7  two threads per row of the resident tile (TMEM lane = row;
//              warps w and w+4 share lane quarter w and split the chunk's 64
//              columns in halves): P = 2^(S*scale*log2e - LSE2) and
//              dS = P (dP - Delta) in packed fp32 pairs, written back to TMEM
//              in bf16 inside the half's own columns (the bf16 pairs of
//              columns 32h .. 32h+31 go to columns 32h .. 32h+15), so the
//              two halves never overwrite what the other still reads
//   warp 8     TMA producer: the resident tile once, then 64-row chunks into
//              a 4-stage ring (128B swizzle)
//   warp 9     TMEM owner and MMA issuer (one thread).  Per chunk c, with S/dP
//              double-buffered in TMEM so the tensor core computes chunk c+1
//              while warps 0-3 work on chunk c:
//     dK/dV:  S^T = K Q_c^T, dP^T = V dO_c^T          (SS, M=128, N=64, K=D)
//             dV += P^T dO_c, dK += dS^T Q_c         (TS, M=128, N=D,  K=64)
//     dQ:     S = Q K_c^T,   dP = dO V_c^T           (SS, M=128, N=64, K=D)
//             dQ += dS K_c                            (TS, M=128, N=D,  K=64)
// TMEM columns: buffer b holds S at 128b + [0,64) and dP at 128b + [64,128);
// accumulators at 256 (dV or dQ) and 256 + D (dK).
#include "hd_kernels.cuh"

namespace hd {

namespace {

constexpr int kRows = 128;    // rows of the resident tile (MMA M)
constexpr int kChunk = 64;    // rows of a streamed chunk
constexpr int kThreads = 320;
constexpr int kCompute = 256;  // threads of warps 0-7
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kStages = 4;
constexpr uint32_t kTmemCols = 512;
constexpr int kBox128 = 128 * 128;  // 128 rows x 128 B (64 bf16)
constexpr int kBox64 = 64 * 128;    // 64 rows x 128 B
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTile = kBoxes * kBox128;       // one 128-row operand
  static constexpr int kChunkBytes = kBoxes * kBox64;  // one 64-row operand
  static constexpr int kStageBytes = 2 * kChunkBytes;  // two operands per stage
  static constexpr int kSmemRes = 0;                   // two resident 128-row operands
  static constexpr int kSmemStage = 2 * kTile;
  static constexpr int kSmemStat = kSmemStage + kStages * kStageBytes;
  static constexpr int kSmemBar = kSmemStat + kStages * kChunk * 8;  // -LSE2[64], -Delta[64]
  static constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 1 + 1;
  static constexpr int kSmemTmemPtr = kSmemBar + kNumBars * 8;
  static constexpr int kSmemBytes = kSmemTmemPtr + 16;
  static constexpr size_t kDynSmem = 1024 + kSmemBytes;
  __host__ __device__ static constexpr uint32_t col_s(int b) { return (uint32_t)b * 128u; }
  __host__ __device__ static constexpr uint32_t col_dp(int b) { return (uint32_t)b * 128u + 64u; }
  static constexpr uint32_t kColAcc0 = 256;      // dV (dK/dV kernel) or dQ (dQ kernel)
  static constexpr uint32_t kColAcc1 = 256 + D;  // dK (dK/dV kernel)
  // dQ kernel: its Q and dO tiles staged in TMEM as the A operands of S and dP
  static constexpr uint32_t kColQ = 256 + D;
  static constexpr uint32_t kColDO = 256 + D + D / 2;
  static_assert(kSmemStage + 2 * kTile <= kSmemStat, "epilogue staging must fit the ring");
};

struct Bars {
  uint64_t *res_full, *in_full, *in_empty, *s_full, *p_full, *acc_done, *a_ready;
};

__device__ __forceinline__ Bars carve_bars(uint8_t *base) {
  uint64_t *b = reinterpret_cast<uint64_t *>(base);
  Bars r;
  r.res_full = b;
  r.in_full = b + 1;
  r.in_empty = r.in_full + kStages;
  r.s_full = r.in_empty + kStages;  // [2]
  r.p_full = r.s_full + 2;          // [2]
  r.acc_done = r.p_full + 2;        // [1]
  r.a_ready = r.acc_done + 1;       // [1] (dQ kernel: Q, dO staged in TMEM)
  return r;
}

__device__ __forceinline__ void init_bars(const Bars &bar) {
  mbar_init(bar.res_full, 1);
  for (int i = 0; i < kStages; ++i) {
    mbar_init(&bar.in_full[i], 1);
    mbar_init(&bar.in_empty[i], 1);
  }
  for (int x = 0; x < 2; ++x) {
    mbar_init(&bar.s_full[x], 1);
    mbar_init(&bar.p_full[x], kCompute);
  }
  mbar_init(bar.acc_done, 1);
  mbar_init(bar.a_ready, kCompute);
  fence_barrier_init();
}

// Untiled bulk copy global -> shared, completion on an mbarrier (16-byte
// aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// One box of rows [row0, row0 + box rows) of head `head` (stream `stream` in
// the within-stream view) at column `dcol`.
__device__ __forceinline__ void load_rows(void *dst, const CUtensorMap *m, uint64_t *bar, int dcol,
                                          int head, int stream, int row0, int batch,
                                          bool within) {
  if (within)
    tma_load_5d(dst, m, bar, dcol, head, stream, row0, batch);
  else
    tma_load_4d(dst, m, bar, dcol, head, row0, batch);
}

// TMEM column (relative to the buffer) of the bf16 A operand of k-step kk:
// half h of the chunk's columns holds its 32 values packed in 16 columns at 32h.
__device__ __forceinline__ uint32_t a_col(int kk) { return (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8); }

// First key position a query at `pos` may attend in the sliding-window mode.
__device__ __forceinline__ int window_lo(const BwdParams &p, int pos) {
  const int t0 = pos / p.n - p.window + 1;
  return t0 > 0 ? t0 * p.n : 0;
}

// Problem decomposition shared by the kernels.
struct Problem {
  int b, s, head;  // batch, stream (0 cross-stream), head (query head or KV head)
};

__device__ __forceinline__ Problem decode_problem(int64_t prob, int heads, int n, bool within) {
  Problem r;
  r.head = (int)(prob % heads);
  prob /= heads;
  r.s = within ? (int)(prob % n) : 0;
  r.b = within ? (int)(prob / n) : (int)prob;
  return r;
}

// Index of query problem (b, s, h) in the order decode_problem reads it.
__device__ __forceinline__ int64_t q_problem(const BwdParams &p, int b, int h, int s, bool within) {
  return within ? ((int64_t)b * p.n + s) * p.Hq + h : (int64_t)b * p.Hq + h;
}

// The producer's tail: every copy it issued must land before the CTA exits.
__device__ __forceinline__ bool drain_ring(const Bars &bar, int issued) {
  bool ok = mbar_wait(bar.res_full, 0);
  for (int it = max(0, issued - kStages); it < issued && ok; ++it)
    ok = mbar_wait(&bar.in_full[it % kStages], (it / kStages) & 1);
  return ok;
}

// Rows of a resident 128-row accumulator in TMEM -> bf16 (times `mul`) into a
// 128B-swizzled staging tile laid out like a TMA box sequence.
template <int D>
__device__ __forceinline__ void stage_rows(uint32_t t_acc, uint8_t *stage, int row, float mul,
                                           int half) {
#pragma unroll
  for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
    uint32_t r[32];
    tmem_ld32(t_acc + c * 32, r);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = c * 32 + q * 8;
      uint8_t *dst = stage + (col >> 6) * kBox128 + sw128_offset(row, (col & 63) >> 3);
      *reinterpret_cast<uint4 *>(dst) =
          make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  }
}

// ---------------------------------------------------------------- row statistics

// One row of D bf16 per kTpr threads (16-byte vectors of 8 elements); a warp
// takes 32 / kTpr rows per step.
template <int D>
__global__ void __launch_bounds__(256) bwd_rowstat_kernel(const BwdParams p) {
  constexpr int kTpr = D / 8;
  constexpr int kRpw = 32 / kTpr;
  const bool within = (p.mode == 0);
  const int lane = threadIdx.x & 31;
  const int sub = lane / kTpr, part = lane % kTpr;
  const int64_t rows = p.problems_q * p.seq_pad;
  const int64_t stride = (int64_t)gridDim.x * 8 * kRpw;
  for (int64_t row0 = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * kRpw; row0 < rows;
       row0 += stride) {
    const int64_t row = row0 + sub;
    float acc = 0.f, lse = INFINITY;  // padding rows: -LSE2 = -inf, -Delta = 0
    if (row < rows) {
      const int64_t prob = row / p.seq_pad;
      const int t = (int)(row - prob * p.seq_pad);
      if (t < p.seq) {
        const Problem pr = decode_problem(prob, p.Hq, p.n, within);
        const int64_t pos = within ? (int64_t)t * p.n + pr.s : (int64_t)t;
        const int64_t base = (((int64_t)pr.b * p.N + pos) * p.Hq + pr.head) * D + part * 8;
        const uint4 a = *reinterpret_cast<const uint4 *>(p.o + base);
        const uint4 g = *reinterpret_cast<const uint4 *>(p.dout + base);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(gw[e] << 16), acc);
          acc = fmaf(__uint_as_float(aw[e] & 0xffff0000u), __uint_as_float(gw[e] & 0xffff0000u),
                     acc);
        }
        lse = p.lse[((int64_t)pr.b * p.Hq + pr.head) * p.N + pos] * kLog2e;
      }
    }
#pragma unroll
    for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (part == 0 && row < rows) {
      p.nlse[row] = -lse;
      p.ndelta[row] = -acc;
    }
  }
}

// ---------------------------------------------------------------- dK / dV

template <int D, bool kWindow>
__global__ void __launch_bounds__(kThreads, 1)
    sfa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,   // 64-row boxes
                        const __grid_constant__ CUtensorMap tm_do,  // 64-row boxes
                        const __grid_constant__ CUtensorMap tm_k,   // 128-row boxes
                        const __grid_constant__ CUtensorMap tm_v,   // 128-row boxes
                        const __grid_constant__ CUtensorMap tm_dk,  // 128-row boxes (store)
                        const __grid_constant__ CUtensorMap tm_dv,  // 128-row boxes (store)
                        const BwdParams p) {
  using Cfg = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *smem = smem_raw + pad;
  uint8_t *sK = smem + Cfg::kSmemRes;
  uint8_t *sV = sK + Cfg::kTile;
  uint8_t *sRing = smem + Cfg::kSmemStage;
  float *sStat = reinterpret_cast<float *>(smem + Cfg::kSmemStat);
  const Bars bar = carve_bars(smem + Cfg::kSmemBar);
  uint32_t *tmem_ptr_smem = reinterpret_cast<uint32_t *>(smem + Cfg::kSmemTmemPtr);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool within = (p.mode == 0);

  // Work item: key tile j (ascending: tile 0 sees the most query chunks).
  const int64_t per = p.problems_kv;
  const int j = (int)(blockIdx.x / per);
  const Problem pr = decode_problem(blockIdx.x % per, p.Hkv, p.n, within);
  const int g = pr.head;
  const int k0 = j * kRows;
  // Query chunks that see any key of the tile: from the chunk holding k0 to
  // the end of the sequence, or (sliding window) to the last query whose
  // window still reaches the tile's last key.
  int q_end = p.seq;
  if (kWindow) {
    const int tk_last = min(k0 + kRows - 1, p.seq - 1) / p.n;
    q_end = min(p.seq, (tk_last + p.window) * p.n);
  }
  const int c_lo = k0 / kChunk;
  const int nch = (q_end + kChunk - 1) / kChunk - c_lo;
  const int nit = p.G * nch;  // (query head in group, chunk) pairs

  if (threadIdx.x == 0) init_bars(bar);
  if (warp == kWarpMma) {
    tmem_alloc(tmem_ptr_smem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr_smem;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar.res_full, 2 * Cfg::kTile);
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c) {
        load_rows(sK + c * kBox128, &tm_k, bar.res_full, c * 64, g, pr.s, k0, pr.b, within);
        load_rows(sV + c * kBox128, &tm_v, bar.res_full, c * 64, g, pr.s, k0, pr.b, within);
      }
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < nit; ++it) {
        const int st = it % kStages;
        if (!(ok = mbar_wait(&bar.in_empty[st], ((it / kStages) & 1) ^ 1))) break;
        const int h = g * p.G + it / nch;
        const int c = c_lo + it % nch;
        uint8_t *dq = sRing + st * Cfg::kStageBytes;
        uint8_t *ddo = dq + Cfg::kChunkBytes;
        mbar_arrive_expect_tx(&bar.in_full[st], Cfg::kStageBytes + kChunk * 8);
#pragma unroll
        for (int cc = 0; cc < Cfg::kBoxes; ++cc) {
          load_rows(dq + cc * kBox64, &tm_q, &bar.in_full[st], cc * 64, h, pr.s, c * kChunk,
                    pr.b, within);
          load_rows(ddo + cc * kBox64, &tm_do, &bar.in_full[st], cc * 64, h, pr.s, c * kChunk,
                    pr.b, within);
        }
        const int64_t srow = q_problem(p, pr.b, h, pr.s, within) * p.seq_pad + (int64_t)c * kChunk;
        bulk_load(sStat + st * 2 * kChunk, p.nlse + srow, kChunk * 4, &bar.in_full[st]);
        bulk_load(sStat + st * 2 * kChunk + kChunk, p.ndelta + srow, kChunk * 4, &bar.in_full[st]);
        issued = it + 1;
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      if (!drain_ring(bar, issued)) report(p.dev_status, kDevTimeout);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRows, kChunk, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kRows, D, true);
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      const uint32_t ring = smem_u32(sRing);
      auto issue_sdp = [&](int it) {
        const int bf = it & 1;
        const uint32_t qb = ring + (it % kStages) * Cfg::kStageBytes;
        const uint32_t ob = qb + Cfg::kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a_off = (kk >> 2) * kBox128 + (kk & 3) * 32;
          const uint32_t b_off = (kk >> 2) * kBox64 + (kk & 3) * 32;
          mma_ss(tmem + Cfg::col_s(bf), smem_desc_sw128(k_base + a_off, 16, 1024),
                 smem_desc_sw128(qb + b_off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a_off = (kk >> 2) * kBox128 + (kk & 3) * 32;
          const uint32_t b_off = (kk >> 2) * kBox64 + (kk & 3) * 32;
          mma_ss(tmem + Cfg::col_dp(bf), smem_desc_sw128(v_base + a_off, 16, 1024),
                 smem_desc_sw128(ob + b_off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.s_full[bf]);
      };
      auto issue_acc = [&](int it) {
        const int bf = it & 1;
        const int st = it % kStages;
        const uint32_t qb = ring + st * Cfg::kStageBytes;
        const uint32_t ob = qb + Cfg::kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          mma_ts(tmem + Cfg::kColAcc0, tmem + Cfg::col_s(bf) + a_col(kk),
                 smem_desc_sw128(ob + kk * 2048, kBox64, 1024), idesc_acc,
                 (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          mma_ts(tmem + Cfg::kColAcc1, tmem + Cfg::col_dp(bf) + a_col(kk),
                 smem_desc_sw128(qb + kk * 2048, kBox64, 1024), idesc_acc,
                 (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar.in_empty[st]);
      };
      bool ok = mbar_wait(bar.res_full, 0);
      for (int it = 0; it < 2 && it < nit && ok; ++it) {
        if (!(ok = mbar_wait(&bar.in_full[it % kStages], (it / kStages) & 1))) break;
        tc_fence_after();
        issue_sdp(it);
      }
      for (int it = 0; it < nit && ok; ++it) {
        if (!(ok = mbar_wait(&bar.p_full[it & 1], (it >> 1) & 1))) break;
        tc_fence_after();
        issue_acc(it);
        const int nx = it + 2;
        if (nx < nit) {
          if (!(ok = mbar_wait(&bar.in_full[nx % kStages], (nx / kStages) & 1))) break;
          tc_fence_after();
          issue_sdp(nx);  // S/dP buffer it&1 is free: issued after the MMAs that read it
        }
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      mma_commit(bar.acc_done);
      if (!mbar_wait(bar.acc_done, 0)) report(p.dev_status, kDevTimeout);
    }
  } else {
    // ------------------------------------------------------------ dS (warps 0-7)
    const int wq = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
    const int row = wq * 32 + lane;             // key row of the tile
    const int kpos = k0 + row;
    const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int it = 0; it < nit; ++it) {
      const int bf = it & 1, st = it % kStages;
      if (!(ok = mbar_wait(&bar.s_full[bf], (it >> 1) & 1) &&
                 mbar_wait(&bar.in_full[st], (it / kStages) & 1)))
        break;
      tc_fence_after();
      const int qc0 = (c_lo + it % nch) * kChunk + half * 32;  // first query of this half
      const uint64_t *nl = reinterpret_cast<const uint64_t *>(sStat + st * 2 * kChunk + half * 32);
      const uint64_t *nd = nl + kChunk / 2;
      // masks only where this half's queries meet the tile's diagonal or window edge
      bool need = qc0 < k0 + kRows - 1;
      if (kWindow) need = need || window_lo(p, qc0 + 31) > k0;
      uint32_t sr[32], dr[32];
      tmem_ld32(tmem + lane_addr + Cfg::col_s(bf) + half * 32, sr);
      tmem_ld32(tmem + lane_addr + Cfg::col_dp(bf) + half * 32, dr);
      tmem_wait_ld();
      uint32_t pp[16], dd[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float p0, p1;
        {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                           sl2, nl[i]),
                    x0, x1);
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        if (need) {
          const int q = qc0 + 2 * i;
          bool a0 = kpos <= q, a1 = kpos <= q + 1;
          if (kWindow) {
            a0 = a0 && kpos >= window_lo(p, q);
            a1 = a1 && kpos >= window_lo(p, q + 1);
          }
          p0 = a0 ? p0 : 0.f;
          p1 = a1 ? p1 : 0.f;
        }
        const uint64_t pv = f2_pack(p0, p1);
        float d0, d1;
        f2_unpack(f2_mul(pv, f2_add(f2_pack(__uint_as_float(dr[2 * i]),
                                            __uint_as_float(dr[2 * i + 1])),
                                    nd[i])),
                  d0, d1);
        pp[i] = pack_bf16x2(p0, p1);
        dd[i] = pack_bf16x2(d0, d1);
      }
      tmem_st16(tmem + lane_addr + Cfg::col_s(bf) + half * 32, pp);
      tmem_st16(tmem + lane_addr + Cfg::col_dp(bf) + half * 32, dd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.p_full[bf]);
    }
    if (ok) ok = mbar_wait(bar.acc_done, 0);
    if (!ok) report(p.dev_status, kDevTimeout);
    // Epilogue: dV and dK (scaled) -> bf16 -> the ring (no longer read) -> TMA.
    uint8_t *stage_dv = sRing;
    uint8_t *stage_dk = sRing + Cfg::kTile;
    if (ok) {
      tc_fence_after();
      stage_rows<D>(tmem + lane_addr + Cfg::kColAcc0, stage_dv, row, 1.f, half);
      stage_rows<D>(tmem + lane_addr + Cfg::kColAcc1, stage_dk, row, p.scale, half);
    }
    tc_fence_before();
    fence_proxy_async_smem();
    named_bar_sync(1, kCompute);
    if (ok && warp == 0 && lane == 0) {
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c) {
        if (within) {
          tma_store_5d(&tm_dv, stage_dv + c * kBox128, c * 64, g, pr.s, k0, pr.b);
          tma_store_5d(&tm_dk, stage_dk + c * kBox128, c * 64, g, pr.s, k0, pr.b);
        } else {
          tma_store_4d(&tm_dv, stage_dv + c * kBox128, c * 64, g, k0, pr.b);
          tma_store_4d(&tm_dk, stage_dk + c * kBox128, c * 64, g, k0, pr.b);
        }
      }
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- dQ

template <int D, bool kWindow>
__global__ void __launch_bounds__(kThreads, 1)
    sfa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,   // 128-row boxes
                      const __grid_constant__ CUtensorMap tm_do,  // 128-row boxes
                      const __grid_constant__ CUtensorMap tm_k,   // 64-row boxes
                      const __grid_constant__ CUtensorMap tm_v,   // 64-row boxes
                      const __grid_constant__ CUtensorMap tm_dq,  // 128-row boxes (store)
                      const BwdParams p) {
  using Cfg = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *smem = smem_raw + pad;
  uint8_t *sQ = smem + Cfg::kSmemRes;
  uint8_t *sDO = sQ + Cfg::kTile;
  uint8_t *sRing = smem + Cfg::kSmemStage;
  const Bars bar = carve_bars(smem + Cfg::kSmemBar);
  uint32_t *tmem_ptr_smem = reinterpret_cast<uint32_t *>(smem + Cfg::kSmemTmemPtr);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool within = (p.mode == 0);

  // Work item: query tile i, last (longest) first.
  const int64_t per = p.problems_q;
  const int i = p.tiles - 1 - (int)(blockIdx.x / per);
  const int64_t qprob = blockIdx.x % per;
  const Problem pr = decode_problem(qprob, p.Hq, p.n, within);
  const int h = pr.head;
  const int g = h / p.G;
  const int q0 = i * kRows;
  const int c_lo = kWindow ? window_lo(p, q0) / kChunk : 0;
  const int nit = min(q0 + kRows - 1, p.seq - 1) / kChunk + 1 - c_lo;

  if (threadIdx.x == 0) init_bars(bar);
  if (warp == kWarpMma) {
    tmem_alloc(tmem_ptr_smem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr_smem;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar.res_full, 2 * Cfg::kTile);
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c) {
        load_rows(sQ + c * kBox128, &tm_q, bar.res_full, c * 64, h, pr.s, q0, pr.b, within);
        load_rows(sDO + c * kBox128, &tm_do, bar.res_full, c * 64, h, pr.s, q0, pr.b, within);
      }
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < nit; ++it) {
        const int st = it % kStages;
        if (!(ok = mbar_wait(&bar.in_empty[st], ((it / kStages) & 1) ^ 1))) break;
        const int c = c_lo + it;
        uint8_t *dk = sRing + st * Cfg::kStageBytes;
        uint8_t *dv = dk + Cfg::kChunkBytes;
        mbar_arrive_expect_tx(&bar.in_full[st], Cfg::kStageBytes);
#pragma unroll
        for (int cc = 0; cc < Cfg::kBoxes; ++cc) {
          load_rows(dk + cc * kBox64, &tm_k, &bar.in_full[st], cc * 64, g, pr.s, c * kChunk,
                    pr.b, within);
          load_rows(dv + cc * kBox64, &tm_v, &bar.in_full[st], cc * 64, g, pr.s, c * kChunk,
                    pr.b, within);
        }
        issued = it + 1;
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      if (!drain_ring(bar, issued)) report(p.dev_status, kDevTimeout);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRows, kChunk, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kRows, D, true);
      const uint32_t ring = smem_u32(sRing);
      // S = Q K_c^T and dP = dO V_c^T with A (Q, dO) in TMEM: only the 64-row
      // chunk is read from shared memory.
      auto issue_sdp = [&](int it) {
        const int bf = it & 1;
        const uint32_t kb = ring + (it % kStages) * Cfg::kStageBytes;
        const uint32_t vb = kb + Cfg::kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t b_off = (kk >> 2) * kBox64 + (kk & 3) * 32;
          mma_ts(tmem + Cfg::col_s(bf), tmem + Cfg::kColQ + kk * 8,
                 smem_desc_sw128(kb + b_off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t b_off = (kk >> 2) * kBox64 + (kk & 3) * 32;
          mma_ts(tmem + Cfg::col_dp(bf), tmem + Cfg::kColDO + kk * 8,
                 smem_desc_sw128(vb + b_off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.s_full[bf]);
      };
      auto issue_acc = [&](int it) {
        const int bf = it & 1;
        const int st = it % kStages;
        const uint32_t kb = ring + st * Cfg::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          mma_ts(tmem + Cfg::kColAcc0, tmem + Cfg::col_s(bf) + a_col(kk),
                 smem_desc_sw128(kb + kk * 2048, kBox64, 1024), idesc_acc,
                 (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar.in_empty[st]);
      };
      bool ok = mbar_wait(bar.res_full, 0) && mbar_wait(bar.a_ready, 0);
      for (int it = 0; it < 2 && it < nit && ok; ++it) {
        if (!(ok = mbar_wait(&bar.in_full[it % kStages], (it / kStages) & 1))) break;
        tc_fence_after();
        issue_sdp(it);
      }
      for (int it = 0; it < nit && ok; ++it) {
        if (!(ok = mbar_wait(&bar.p_full[it & 1], (it >> 1) & 1))) break;
        tc_fence_after();
        issue_acc(it);
        const int nx = it + 2;
        if (nx < nit) {
          if (!(ok = mbar_wait(&bar.in_full[nx % kStages], (nx / kStages) & 1))) break;
          tc_fence_after();
          issue_sdp(nx);
        }
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      mma_commit(bar.acc_done);
      if (!mbar_wait(bar.acc_done, 0)) report(p.dev_status, kDevTimeout);
    }
  } else {
    // ------------------------------------------------------------ dS (warps 0-7)
    const int wq = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
    const int row = wq * 32 + lane;             // query row of the tile
    const int qpos = q0 + row;
    const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    // This row's statistics (padding rows: -LSE2 = -inf, so P = 0).
    const int64_t srow = qprob * p.seq_pad + qpos;
    const float nlse = p.nlse[srow], ndel = p.ndelta[srow];
    const uint64_t nl2 = f2_pack(nlse, nlse), nd2 = f2_pack(ndel, ndel);
    const int lo_row = kWindow ? window_lo(p, qpos) : 0;
    // Stage this thread's half of its Q and dO rows into TMEM (A operands of S
    // and dP): 16-byte chunks of the 128B-swizzled tiles, two bf16 per column.
    bool ok = mbar_wait(bar.res_full, 0);
    if (ok) {
      constexpr int kHalfChunks = D / 16;  // 16-byte chunks in half a row
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint8_t *tile = t ? sDO : sQ;
        uint32_t w[4 * kHalfChunks];  // D/4 packed columns
#pragma unroll
        for (int c = 0; c < kHalfChunks; ++c) {
          const int col = half * (D / 2) + c * 8;  // first element of the chunk
          const uint4 v4 = *reinterpret_cast<const uint4 *>(
              tile + (col >> 6) * kBox128 + sw128_offset(row, (col & 63) >> 3));
          w[4 * c] = v4.x;
          w[4 * c + 1] = v4.y;
          w[4 * c + 2] = v4.z;
          w[4 * c + 3] = v4.w;
        }
        const uint32_t col0 = (t ? Cfg::kColDO : Cfg::kColQ) + half * (D / 4);
        if constexpr (D == 128) {
          tmem_st32(tmem + lane_addr + col0, w);
        } else {
          tmem_st16(tmem + lane_addr + col0, w);
        }
      }
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(bar.a_ready);
    for (int it = 0; it < nit && ok; ++it) {
      const int bf = it & 1;
      if (!(ok = mbar_wait(&bar.s_full[bf], (it >> 1) & 1))) break;
      tc_fence_after();
      const int kc0 = (c_lo + it) * kChunk + half * 32;  // first key of this half
      // masks only where this half's keys meet the tile's diagonal or window edge
      bool need = kc0 + 31 > q0;
      if (kWindow) need = need || kc0 < window_lo(p, q0 + kRows - 1);
      uint32_t sr[32], dr[32];
      tmem_ld32(tmem + lane_addr + Cfg::col_s(bf) + half * 32, sr);
      tmem_ld32(tmem + lane_addr + Cfg::col_dp(bf) + half * 32, dr);
      tmem_wait_ld();
      uint32_t dd[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float p0, p1;
        {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                           sl2, nl2),
                    x0, x1);
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        if (need) {
          const int kp = kc0 + 2 * i;
          bool a0 = kp <= qpos, a1 = kp + 1 <= qpos;
          if (kWindow) {
            a0 = a0 && kp >= lo_row;
            a1 = a1 && kp + 1 >= lo_row;
          }
          p0 = a0 ? p0 : 0.f;
          p1 = a1 ? p1 : 0.f;
        }
        float d0, d1;
        f2_unpack(f2_mul(f2_pack(p0, p1),
                         f2_add(f2_pack(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1])),
                                nd2)),
                  d0, d1);
        dd[i] = pack_bf16x2(d0, d1);
      }
      tmem_st16(tmem + lane_addr + Cfg::col_s(bf) + half * 32, dd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.p_full[bf]);
    }
    if (ok) ok = mbar_wait(bar.acc_done, 0);
    if (!ok) report(p.dev_status, kDevTimeout);
    // Epilogue: dQ (scaled) -> bf16 -> the Q buffer (no longer read) -> TMA.
    if (ok) {
      tc_fence_after();
      stage_rows<D>(tmem + lane_addr + Cfg::kColAcc0, sQ, row, p.scale, half);
    }
    tc_fence_before();
    fence_proxy_async_smem();
    named_bar_sync(1, kCompute);
    if (ok && warp == 0 && lane == 0) {
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c) {
        if (within)
          tma_store_5d(&tm_dq, sQ + c * kBox128, c * 64, h, pr.s, q0, pr.b);
        else
          tma_store_4d(&tm_dq, sQ + c * kBox128, c * 64, h, q0, pr.b);
      }
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D, bool kWindow>
cudaError_t launch_bwd(const CUtensorMap &q_c, const CUtensorMap &do_c, const CUtensorMap &k_t,
                       const CUtensorMap &v_t, const CUtensorMap &dk_t, const CUtensorMap &dv_t,
                       const CUtensorMap &q_t, const CUtensorMap &do_t, const CUtensorMap &k_c,
                       const CUtensorMap &v_c, const CUtensorMap &dq_t, const BwdParams &p,
                       cudaStream_t stream, int num_sms) {
  static int done_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (done_dev != dev) {
    cudaError_t e = set_smem(sfa_bwd_dkdv_kernel<D, kWindow>, BCfg<D>::kDynSmem);
    if (e == cudaSuccess) e = set_smem(sfa_bwd_dq_kernel<D, kWindow>, BCfg<D>::kDynSmem);
    if (e != cudaSuccess) return e;
    done_dev = dev;
  }
  const int64_t rows = p.problems_q * p.seq_pad;
  const int64_t rows_per_block = 8 * (32 / (D / 8));
  int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (blocks > (int64_t)num_sms * 64) blocks = (int64_t)num_sms * 64;
  bwd_rowstat_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sfa_bwd_dkdv_kernel<D, kWindow>
      <<<(unsigned)(p.problems_kv * p.tiles), kThreads, BCfg<D>::kDynSmem, stream>>>(
          q_c, do_c, k_t, v_t, dk_t, dv_t, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sfa_bwd_dq_kernel<D, kWindow>
      <<<(unsigned)(p.problems_q * p.tiles), kThreads, BCfg<D>::kDynSmem, stream>>>(
          q_t, do_t, k_c, v_c, dq_t, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sfa_backward(const CUtensorMap &q_c, const CUtensorMap &do_c,
                                const CUtensorMap &k_t, const CUtensorMap &v_t,
                                const CUtensorMap &dk_t, const CUtensorMap &dv_t,
                                const CUtensorMap &q_t, const CUtensorMap &do_t,
                                const CUtensorMap &k_c, const CUtensorMap &v_c,
                                const CUtensorMap &dq_t, const BwdParams &p, int D,
                                cudaStream_t stream, int num_sms) {
  if (p.problems_q * p.tiles == 0) return cudaSuccess;
  if (p.problems_q * p.tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const bool win = (p.mode == 2);
  if (D == 128)
    return win ? launch_bwd<128, true>(q_c, do_c, k_t, v_t, dk_t, dv_t, q_t, do_t, k_c, v_c, dq_t,
                                       p, stream, num_sms)
               : launch_bwd<128, false>(q_c, do_c, k_t, v_t, dk_t, dv_t, q_t, do_t, k_c, v_c,
                                        dq_t, p, stream, num_sms);
  return win ? launch_bwd<64, true>(q_c, do_c, k_t, v_t, dk_t, dv_t, q_t, do_t, k_c, v_c, dq_t, p,
                                    stream, num_sms)
             : launch_bwd<64, false>(q_c, do_c, k_t, v_t, dk_t, dv_t, q_t, do_t, k_c, v_c, dq_t,
                                     p, stream, num_sms);
}

}  // namespace hd
