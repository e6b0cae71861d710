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
//                 shared memory; the CTA streams every 128-row query chunk
//                 that sees the tile, for each query head of the KV head's
//                 group, and accumulates dV and dK in TMEM.
//   sfa_bwd_dq    one CTA per (query problem, 128-query tile): Q and dO stay in
//                 shared memory; the CTA streams the 128-row key chunks the
//                 tile sees and accumulates dQ in TMEM.
// Each output row is written by exactly one CTA: no atomics, and the result
// does not depend on scheduling.  S and dP are computed in both kernels (7
// tile products per pair of tiles instead of 5); in exchange dQ needs no fp32
// accumulation buffer in HBM and no reduction traffic through L2.
//
// Every tile product is M=128, N=128 (or N=D): narrower products measured at
// about the cost of full-width ones per instruction, so the chunks are 128
// rows wide and TMEM is budgeted around that.
//
// Roles (320 threads), the same in both kernels:
//   warps 0-7  two threads per row of the resident tile (TMEM lane = row;
//              warps w and w+4 share lane quarter w and split the chunk's 128
//              columns in halves): P = 2^(S*scale*log2e - LSE2) and
//              dS = P (dP - Delta) in packed fp32 pairs, written back to TMEM
//              in bf16 inside the half's own columns (the bf16 pairs of
//              columns 64h .. 64h+63 go to columns 64h .. 64h+31), so the two
//              halves never overwrite what the other still reads
//   warp 8     TMA producer: the resident tiles once, then 128-row chunks
//   warp 9     TMEM owner and MMA issuer (one thread)
//
// dK/dV kernel, per query chunk c (TMEM: S^T [0,128), dP^T [128,256),
// dV [256,256+D), dK [256+D,256+2D)):
//   S^T = K Q_c^T, dP^T = V dO_c^T          SS, M=128 (keys), N=128, K=D
//   P phase:  P^T in bf16 over S^T           -> dV += P^T dO_c   TS, K=128
//   dS phase: dS^T in bf16 over dP^T         -> dK += dS^T Q_c   TS, K=128
//   issue order dV(c), S^T(c+1), dK(c), dP^T(c+1): the tensor core computes
//   dV(c) and S^T(c+1) while the dS phase of chunk c runs, and dK(c),
//   dP^T(c+1) while the P phase of chunk c+1 runs.  Q_c/dO_c ring: 2 stages.
// dQ kernel, per key chunk c (TMEM: S in slot 0 or 2 by chunk parity at
// [0,128) / [256,384), dP at [128,256), dQ at [384,384+D)):
//   S = Q K_c^T, dP = dO V_c^T              SS, M=128 (queries), N=128, K=D
//   dS in bf16 over S                       -> dQ += dS K_c      TS, K=128
//   issue order dP(c+1), dQ(c), S(c+2): S of the next two chunks is always
//   ahead of the dS warps.  K ring 3 stages (K_c is read by S(c) and dQ(c)),
//   V ring 2 stages (V_c only by dP(c)).
#include "hd_kernels.cuh"

namespace hd {

namespace {

constexpr int kRows = 128;    // rows of the resident tile (MMA M)
constexpr int kChunk = 128;   // rows of a streamed chunk (MMA N of S / dP)
constexpr int kThreads = 320;
constexpr int kCompute = 256;  // threads of warps 0-7
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr uint32_t kTmemCols = 512;
constexpr int kBox = 128 * 128;  // TMA box: 128 rows x 128 B (64 bf16)
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------ dK/dV layout
constexpr int kKvStages = 2;
template <int D>
struct KvCfg {
  static constexpr int kTile = (D / 64) * kBox;        // one 128-row operand
  static constexpr int kSmemK = 0;
  static constexpr int kSmemV = kTile;
  static constexpr int kSmemRing = 2 * kTile;          // stage: Q_c, dO_c
  static constexpr int kStageBytes = 2 * kTile;
  static constexpr int kSmemStat = kSmemRing + kKvStages * kStageBytes;  // -LSE2[128], -Delta[128]
  static constexpr int kSmemBar = kSmemStat + kKvStages * kChunk * 8;
  static constexpr int kNumBars = 1 + 2 * kKvStages + 5;
  static constexpr int kSmemTmemPtr = kSmemBar + kNumBars * 8;
  static constexpr size_t kDynSmem = 1024 + kSmemTmemPtr + 16;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
};

// ------------------------------------------------------------ dQ layout
constexpr int kKStages = 3;
constexpr int kVStages = 2;
template <int D>
struct QCfg {
  static constexpr int kTile = (D / 64) * kBox;
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemDO = kTile;
  static constexpr int kSmemK = 2 * kTile;                   // K ring
  static constexpr int kSmemV = kSmemK + kKStages * kTile;   // V ring
  static constexpr int kSmemBar = kSmemV + kVStages * kTile;
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 5;
  static constexpr int kSmemTmemPtr = kSmemBar + kNumBars * 8;
  static constexpr size_t kDynSmem = 1024 + kSmemTmemPtr + 16;
  __host__ __device__ static constexpr uint32_t col_s(int c) { return (c & 1) ? 256u : 0u; }
  static constexpr uint32_t kColDP = 128, kColDQ = 384;
};

// TMEM column (relative to the slot) of the bf16 A operand of k-step kk (16
// rows of the chunk): half h of the chunk's columns holds its 64 values packed
// in 32 columns at 64h.
__device__ __forceinline__ uint32_t a_col(int kk) {
  return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8);
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

// The 128-row operand [row0, row0 + 128) of head `head` (stream `stream` in
// the within-stream view): D / 64 boxes of 64 columns.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t *dst, const CUtensorMap *m, uint64_t *bar,
                                          int head, int stream, int row0, int batch,
                                          bool within) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    if (within)
      tma_load_5d(dst + c * kBox, m, bar, c * 64, head, stream, row0, batch);
    else
      tma_load_4d(dst + c * kBox, m, bar, c * 64, head, row0, batch);
  }
}

template <int D>
__device__ __forceinline__ void store_tile(const CUtensorMap *m, const uint8_t *src, int head,
                                           int stream, int row0, int batch, bool within) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    if (within)
      tma_store_5d(m, src + c * kBox, c * 64, head, stream, row0, batch);
    else
      tma_store_4d(m, src + c * kBox, c * 64, head, row0, batch);
  }
}

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

// SS product of two 128-row K-major operands over K = D: D[tmem] = A B^T.
template <int D>
__device__ __forceinline__ void mma_rows(uint32_t d_tmem, uint32_t a, uint32_t b, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
    mma_ss(d_tmem, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), idesc,
           kk > 0 ? 1u : 0u);
  }
}

// TS product over K = 128 chunk rows: D[tmem] (+)= A[tmem slot] B, B a
// 128-row operand used MN-major (its D columns are N).
__device__ __forceinline__ void mma_acc(uint32_t d_tmem, uint32_t a_slot, uint32_t b,
                                        uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kChunk / 16; ++kk)
    mma_ts(d_tmem, a_slot + a_col(kk), smem_desc_sw128(b + kk * 2048, kBox, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

// Rows of a resident 128-row accumulator in TMEM -> bf16 (times `mul`) into a
// 128B-swizzled staging tile laid out like a TMA box sequence; this thread
// writes columns [half * D/2, (half + 1) * D/2).
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
      uint8_t *dst = stage + (col >> 6) * kBox + sw128_offset(row, (col & 63) >> 3);
      *reinterpret_cast<uint4 *>(dst) =
          make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  }
}

__device__ __forceinline__ uint64_t u2(uint32_t lo, uint32_t hi) {
  return f2_pack(__uint_as_float(lo), __uint_as_float(hi));
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
    sfa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_dk,  // store
                        const __grid_constant__ CUtensorMap tm_dv,  // store
                        const BwdParams p) {
  using Cfg = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *smem = smem_raw + pad;
  uint8_t *sK = smem + Cfg::kSmemK;
  uint8_t *sV = smem + Cfg::kSmemV;
  uint8_t *sRing = smem + Cfg::kSmemRing;
  float *sStat = reinterpret_cast<float *>(smem + Cfg::kSmemStat);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kSmemBar);
  uint64_t *res_full = bars;
  uint64_t *in_full = bars + 1;                // [kKvStages]
  uint64_t *in_empty = in_full + kKvStages;    // [kKvStages]
  uint64_t *s_full = in_empty + kKvStages;     // S^T(c) computed
  uint64_t *dp_full = s_full + 1;              // dP^T(c) computed
  uint64_t *pp_full = dp_full + 1;             // P^T(c) written (kCompute arrivals)
  uint64_t *ds_full = pp_full + 1;             // dS^T(c) written (kCompute arrivals)
  uint64_t *acc_done = ds_full + 1;
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

  if (threadIdx.x == 0) {
    mbar_init(res_full, 1);
    for (int i = 0; i < kKvStages; ++i) {
      mbar_init(&in_full[i], 1);
      mbar_init(&in_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(pp_full, kCompute);
    mbar_init(ds_full, kCompute);
    mbar_init(acc_done, 1);
    fence_barrier_init();
  }
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
      mbar_arrive_expect_tx(res_full, 2 * Cfg::kTile);
      load_tile<D>(sK, &tm_k, res_full, g, pr.s, k0, pr.b, within);
      load_tile<D>(sV, &tm_v, res_full, g, pr.s, k0, pr.b, within);
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < nit; ++it) {
        const int st = it % kKvStages;
        if (!(ok = mbar_wait(&in_empty[st], ((it / kKvStages) & 1) ^ 1))) break;
        const int h = g * p.G + it / nch;
        const int c = c_lo + it % nch;
        uint8_t *dst = sRing + st * Cfg::kStageBytes;
        mbar_arrive_expect_tx(&in_full[st], Cfg::kStageBytes + kChunk * 8);
        load_tile<D>(dst, &tm_q, &in_full[st], h, pr.s, c * kChunk, pr.b, within);
        load_tile<D>(dst + Cfg::kTile, &tm_do, &in_full[st], h, pr.s, c * kChunk, pr.b, within);
        const int64_t srow = q_problem(p, pr.b, h, pr.s, within) * p.seq_pad + (int64_t)c * kChunk;
        float *sd = sStat + st * 2 * kChunk;
        bulk_load(sd, p.nlse + srow, kChunk * 4, &in_full[st]);
        bulk_load(sd + kChunk, p.ndelta + srow, kChunk * 4, &in_full[st]);
        issued = it + 1;
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      // every copy issued must land before the CTA exits
      bool drained = mbar_wait(res_full, 0);
      for (int it = max(0, issued - kKvStages); it < issued && drained; ++it)
        drained = mbar_wait(&in_full[it % kKvStages], (it / kKvStages) & 1);
      if (!drained) report(p.dev_status, kDevTimeout);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRows, kChunk, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kRows, D, true);
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      const uint32_t ring = smem_u32(sRing);
      auto q_of = [&](int it) { return ring + (it % kKvStages) * Cfg::kStageBytes; };
      bool ok = mbar_wait(res_full, 0) && mbar_wait(&in_full[0], 0);
      if (ok) {
        tc_fence_after();
        mma_rows<D>(tmem + Cfg::kColS, k_base, q_of(0), idesc_s);
        mma_commit(s_full);
        mma_rows<D>(tmem + Cfg::kColDP, v_base, q_of(0) + Cfg::kTile, idesc_s);
        mma_commit(dp_full);
      }
      for (int it = 0; it < nit && ok; ++it) {
        const uint32_t qb = q_of(it), ob = qb + Cfg::kTile;
        if (!(ok = mbar_wait(pp_full, it & 1))) break;
        tc_fence_after();
        mma_acc(tmem + Cfg::kColDV, tmem + Cfg::kColS, ob, idesc_acc, it > 0);  // dV += P^T dO_c
        const int nx = it + 1;
        if (nx < nit) {
          if (!(ok = mbar_wait(&in_full[nx % kKvStages], (nx / kKvStages) & 1))) break;
          tc_fence_after();
          mma_rows<D>(tmem + Cfg::kColS, k_base, q_of(nx), idesc_s);  // after dV(it) read P^T
          mma_commit(s_full);
        }
        if (!(ok = mbar_wait(ds_full, it & 1))) break;
        tc_fence_after();
        mma_acc(tmem + Cfg::kColDK, tmem + Cfg::kColDP, qb, idesc_acc, it > 0);  // dK += dS^T Q_c
        mma_commit(&in_empty[it % kKvStages]);  // Q_c, dO_c no longer read
        if (nx < nit) {
          mma_rows<D>(tmem + Cfg::kColDP, v_base, q_of(nx) + Cfg::kTile, idesc_s);
          mma_commit(dp_full);
        }
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      mma_commit(acc_done);
      if (!mbar_wait(acc_done, 0)) report(p.dev_status, kDevTimeout);
    }
  } else {
    // ------------------------------------------------------------ P, dS (warps 0-7)
    const int wq = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
    const int row = wq * 32 + lane;             // key row of the tile
    const int kpos = k0 + row;
    const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_addr + Cfg::kColS + half * 64;
    const uint32_t t_dp = tmem + lane_addr + Cfg::kColDP + half * 64;
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int it = 0; it < nit; ++it) {
      const int st = it % kKvStages;
      if (!(ok = mbar_wait(s_full, it & 1) && mbar_wait(&in_full[st], (it / kKvStages) & 1)))
        break;
      tc_fence_after();
      const int qc0 = (c_lo + it % nch) * kChunk + half * 64;  // first query of this half
      const uint64_t *nl = reinterpret_cast<const uint64_t *>(sStat + st * 2 * kChunk + half * 64);
      const uint64_t *nd = nl + kChunk / 2;
      // masks only where this half's queries meet the tile's diagonal or window edge
      bool need = qc0 < k0 + kRows - 1;
      if (kWindow) need = need || window_lo(p, qc0 + 63) > k0;
      // P phase: P^T = 2^(S^T * scale * log2e - LSE2) for 64 queries, kept in
      // registers for the dS phase and written to TMEM in bf16 over S^T.
      float pv[64];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(t_s, r0);
        tmem_ld32(t_s + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t lo = i < 16 ? r0[2 * i] : r1[2 * i - 32];
          const uint32_t hi = i < 16 ? r0[2 * i + 1] : r1[2 * i - 31];
          float x0, x1;
          f2_unpack(f2_fma(u2(lo, hi), sl2, nl[i]), x0, x1);
          pv[2 * i] = ex2_approx(x0);
          pv[2 * i + 1] = ex2_approx(x1);
        }
      }
      if (need) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int q = qc0 + i;
          bool a = kpos <= q;
          if (kWindow) a = a && kpos >= window_lo(p, q);
          pv[i] = a ? pv[i] : 0.f;
        }
      }
      {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pv[2 * i], pv[2 * i + 1]);
        tmem_st16(t_s, pk);
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pv[32 + 2 * i], pv[33 + 2 * i]);
        tmem_st16(t_s + 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(pp_full);
      // dS phase: dS^T = P^T (dP^T - Delta), in bf16 over dP^T.
      if (!(ok = mbar_wait(dp_full, it & 1))) break;
      tc_fence_after();
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        uint32_t r[32];
        tmem_ld32(t_dp + pass * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = pass * 32 + 2 * i;
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(pv[c], pv[c + 1]), f2_add(u2(r[2 * i], r[2 * i + 1]), nd[c / 2])),
                    d0, d1);
          pk[i] = pack_bf16x2(d0, d1);
        }
        tmem_st16(t_dp + pass * 16, pk);  // columns already read by pass 0
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok) ok = mbar_wait(acc_done, 0);
    if (!ok) report(p.dev_status, kDevTimeout);
    // Epilogue: dV and dK (scaled) -> bf16 -> ring stage 0 (no longer read) -> TMA.
    uint8_t *stage_dv = sRing;
    uint8_t *stage_dk = sRing + Cfg::kTile;
    if (ok) {
      tc_fence_after();
      stage_rows<D>(tmem + lane_addr + Cfg::kColDV, stage_dv, row, 1.f, half);
      stage_rows<D>(tmem + lane_addr + Cfg::kColDK, stage_dk, row, p.scale, half);
    }
    tc_fence_before();
    fence_proxy_async_smem();
    named_bar_sync(1, kCompute);
    if (ok && warp == 0 && lane == 0) {
      store_tile<D>(&tm_dv, stage_dv, g, pr.s, k0, pr.b, within);
      store_tile<D>(&tm_dk, stage_dk, g, pr.s, k0, pr.b, within);
      tma_store_commit();
      tma_store_wait_read();  // shared memory read; the writes finish on their own
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
    sfa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_dq,  // store
                      const BwdParams p) {
  using Cfg = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t *smem = smem_raw + pad;
  uint8_t *sQ = smem + Cfg::kSmemQ;
  uint8_t *sDO = smem + Cfg::kSmemDO;
  uint8_t *sK = smem + Cfg::kSmemK;
  uint8_t *sV = smem + Cfg::kSmemV;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kSmemBar);
  uint64_t *res_full = bars;
  uint64_t *k_full = bars + 1;              // [kKStages]
  uint64_t *k_empty = k_full + kKStages;    // [kKStages]
  uint64_t *v_full = k_empty + kKStages;    // [kVStages]
  uint64_t *v_empty = v_full + kVStages;    // [kVStages]
  uint64_t *s_full = v_empty + kVStages;    // [2] S(c) computed, by chunk parity
  uint64_t *dp_full = s_full + 2;           // dP(c) computed
  uint64_t *p_full = dp_full + 1;           // dS(c) written (kCompute arrivals)
  uint64_t *acc_done = p_full + 1;
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

  if (threadIdx.x == 0) {
    mbar_init(res_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, kCompute);
    mbar_init(acc_done, 1);
    fence_barrier_init();
  }
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
      mbar_arrive_expect_tx(res_full, 2 * Cfg::kTile);
      load_tile<D>(sQ, &tm_q, res_full, h, pr.s, q0, pr.b, within);
      load_tile<D>(sDO, &tm_do, res_full, h, pr.s, q0, pr.b, within);
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int it = 0; it < nit; ++it) {
        const int c = c_lo + it;
        const int ks = it % kKStages, vs = it % kVStages;
        if (!(ok = mbar_wait(&k_empty[ks], ((it / kKStages) & 1) ^ 1))) break;
        mbar_arrive_expect_tx(&k_full[ks], Cfg::kTile);
        load_tile<D>(sK + ks * Cfg::kTile, &tm_k, &k_full[ks], g, pr.s, c * kChunk, pr.b, within);
        k_issued = it + 1;
        if (!(ok = mbar_wait(&v_empty[vs], ((it / kVStages) & 1) ^ 1))) break;
        mbar_arrive_expect_tx(&v_full[vs], Cfg::kTile);
        load_tile<D>(sV + vs * Cfg::kTile, &tm_v, &v_full[vs], g, pr.s, c * kChunk, pr.b, within);
        v_issued = it + 1;
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      bool drained = mbar_wait(res_full, 0);
      for (int it = max(0, k_issued - kKStages); it < k_issued && drained; ++it)
        drained = mbar_wait(&k_full[it % kKStages], (it / kKStages) & 1);
      for (int it = max(0, v_issued - kVStages); it < v_issued && drained; ++it)
        drained = mbar_wait(&v_full[it % kVStages], (it / kVStages) & 1);
      if (!drained) report(p.dev_status, kDevTimeout);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRows, kChunk, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kRows, D, true);
      const uint32_t q_base = smem_u32(sQ), do_base = smem_u32(sDO);
      const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
      auto k_of = [&](int it) { return k_base + (it % kKStages) * Cfg::kTile; };
      auto v_of = [&](int it) { return v_base + (it % kVStages) * Cfg::kTile; };
      auto issue_s = [&](int it) {  // S(it) into its parity's slot
        mma_rows<D>(tmem + Cfg::col_s(it), q_base, k_of(it), idesc_s);
        mma_commit(&s_full[it & 1]);
      };
      auto issue_dp = [&](int it) {  // dP(it); V_it is then free
        mma_rows<D>(tmem + Cfg::kColDP, do_base, v_of(it), idesc_s);
        mma_commit(dp_full);
        mma_commit(&v_empty[it % kVStages]);
      };
      bool ok = mbar_wait(res_full, 0) && mbar_wait(&k_full[0], 0) && mbar_wait(&v_full[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        if (nit > 1) {
          if ((ok = mbar_wait(&k_full[1], 0))) {
            tc_fence_after();
            issue_s(1);
          }
        }
      }
      for (int it = 0; it < nit && ok; ++it) {
        if (!(ok = mbar_wait(p_full, it & 1))) break;
        tc_fence_after();
        const int n1 = it + 1, n2 = it + 2;
        if (n1 < nit) {  // dP(it) has been read: its slot takes dP(it+1)
          if (!(ok = mbar_wait(&v_full[n1 % kVStages], (n1 / kVStages) & 1))) break;
          tc_fence_after();
          issue_dp(n1);
        }
        mma_acc(tmem + Cfg::kColDQ, tmem + Cfg::col_s(it), k_of(it), idesc_acc, it > 0);
        mma_commit(&k_empty[it % kKStages]);  // K_it no longer read
        if (n2 < nit) {  // S(it+2) into S(it)'s slot, after dQ(it) read dS(it) from it
          if (!(ok = mbar_wait(&k_full[n2 % kKStages], (n2 / kKStages) & 1))) break;
          tc_fence_after();
          issue_s(n2);
        }
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      mma_commit(acc_done);
      if (!mbar_wait(acc_done, 0)) report(p.dev_status, kDevTimeout);
    }
  } else {
    // ------------------------------------------------------------ dS (warps 0-7)
    const int wq = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
    const int row = wq * 32 + lane;             // query row of the tile
    const int qpos = q0 + row;
    const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
    const uint32_t t_dp = tmem + lane_addr + Cfg::kColDP + half * 64;
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    // This row's statistics (padding rows: -LSE2 = -inf, so P = 0).
    const int64_t srow = qprob * p.seq_pad + qpos;
    const float nlse = p.nlse[srow], ndel = p.ndelta[srow];
    const uint64_t nl2 = f2_pack(nlse, nlse), nd2 = f2_pack(ndel, ndel);
    const int lo_row = kWindow ? window_lo(p, qpos) : 0;
    bool ok = true;
    for (int it = 0; it < nit; ++it) {
      if (!(ok = mbar_wait(&s_full[it & 1], (it >> 1) & 1) && mbar_wait(dp_full, it & 1))) break;
      tc_fence_after();
      const uint32_t t_s = tmem + lane_addr + Cfg::col_s(it) + half * 64;
      const int kc0 = (c_lo + it) * kChunk + half * 64;  // first key of this half
      // masks only where this half's keys meet the tile's diagonal or window edge
      bool need = kc0 + 63 > q0;
      if (kWindow) need = need || kc0 < window_lo(p, q0 + kRows - 1);
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        uint32_t sr[32], dr[32];
        tmem_ld32(t_s + pass * 32, sr);
        tmem_ld32(t_dp + pass * 32, dr);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) {
          float p0, p1;
          {
            float x0, x1;
            f2_unpack(f2_fma(u2(sr[2 * i2], sr[2 * i2 + 1]), sl2, nl2), x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          if (need) {
            const int kp = kc0 + pass * 32 + 2 * i2;
            bool a0 = kp <= qpos, a1 = kp + 1 <= qpos;
            if (kWindow) {
              a0 = a0 && kp >= lo_row;
              a1 = a1 && kp + 1 >= lo_row;
            }
            p0 = a0 ? p0 : 0.f;
            p1 = a1 ? p1 : 0.f;
          }
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(p0, p1), f2_add(u2(dr[2 * i2], dr[2 * i2 + 1]), nd2)), d0, d1);
          pk[i2] = pack_bf16x2(d0, d1);
        }
        tmem_st16(t_s + pass * 16, pk);  // columns already read by pass 0
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok) ok = mbar_wait(acc_done, 0);
    if (!ok) report(p.dev_status, kDevTimeout);
    // Epilogue: dQ (scaled) -> bf16 -> the Q buffer (no longer read) -> TMA.
    if (ok) {
      tc_fence_after();
      stage_rows<D>(tmem + lane_addr + Cfg::kColDQ, sQ, row, p.scale, half);
    }
    tc_fence_before();
    fence_proxy_async_smem();
    named_bar_sync(1, kCompute);
    if (ok && warp == 0 && lane == 0) {
      store_tile<D>(&tm_dq, sQ, h, pr.s, q0, pr.b, within);
      tma_store_commit();
      tma_store_wait_read();  // shared memory read; the writes finish on their own
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
cudaError_t launch_bwd(const CUtensorMap &q_t, const CUtensorMap &do_t, const CUtensorMap &k_t,
                       const CUtensorMap &v_t, const CUtensorMap &dq_t, const CUtensorMap &dk_t,
                       const CUtensorMap &dv_t, const BwdParams &p, cudaStream_t stream,
                       int num_sms) {
  static int done_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (done_dev != dev) {
    cudaError_t e = set_smem(sfa_bwd_dkdv_kernel<D, kWindow>, KvCfg<D>::kDynSmem);
    if (e == cudaSuccess) e = set_smem(sfa_bwd_dq_kernel<D, kWindow>, QCfg<D>::kDynSmem);
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
      <<<(unsigned)(p.problems_kv * p.tiles), kThreads, KvCfg<D>::kDynSmem, stream>>>(
          q_t, do_t, k_t, v_t, dk_t, dv_t, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sfa_bwd_dq_kernel<D, kWindow>
      <<<(unsigned)(p.problems_q * p.tiles), kThreads, QCfg<D>::kDynSmem, stream>>>(
          q_t, do_t, k_t, v_t, dq_t, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sfa_backward(const CUtensorMap &q_t, const CUtensorMap &do_t,
                                const CUtensorMap &k_t, const CUtensorMap &v_t,
                                const CUtensorMap &dq_t, const CUtensorMap &dk_t,
                                const CUtensorMap &dv_t, const BwdParams &p, int D,
                                cudaStream_t stream, int num_sms) {
  if (p.problems_q * p.tiles == 0) return cudaSuccess;
  if (p.problems_q * p.tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const bool win = (p.mode == 2);
  if (D == 128)
    return win ? launch_bwd<128, true>(q_t, do_t, k_t, v_t, dq_t, dk_t, dv_t, p, stream, num_sms)
               : launch_bwd<128, false>(q_t, do_t, k_t, v_t, dq_t, dk_t, dv_t, p, stream, num_sms);
  return win ? launch_bwd<64, true>(q_t, do_t, k_t, v_t, dq_t, dk_t, dv_t, p, stream, num_sms)
             : launch_bwd<64, false>(q_t, do_t, k_t, v_t, dq_t, dk_t, dv_t, p, stream, num_sms);
}

}  // namespace hd
