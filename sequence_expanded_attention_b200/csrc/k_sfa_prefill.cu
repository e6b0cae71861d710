// k_sfa_prefill.cu -- Stream-Factorized Attention forward on tcgen05 tensor
// cores ("Hidden Decoding at Scale" review, "Method": most layers attend only
// within their own stream, O(nL^2); a few mix streams over the whole expanded
// sequence following the base model's pattern, full or sliding-window,
// O(n^2 L^2) at most; README "Key Idea").
//
// One CTA computes two adjacent 128-row query tiles (A and B) of one attention
// problem, so every K/V tile brought into shared memory serves 256 rows:
//   within-stream: problem = (batch, query head, stream s); its sequence is
//     the L tokens of stream s, read through a 5-D TMA view
//     [B][L][n][H][D] of the token-major expanded tensor, so no copy or
//     transpose is made and each stream is a plain causal problem of length L
//     (the n-fold cost the pages give, not n^2);
//   cross-stream: problem = (batch, query head); its sequence is all N = nL
//     expanded positions, read through a 4-D view [B][N][H][D];
//   cross-stream sliding window (mode 2): as cross-stream, but a query of
//     token t sees only the last `window` tokens; each query tile starts at
//     the KV tile holding its first row's window start;
//   transient intermediate streams (mode 3): as within-stream, but every
//     stream's queries read the final stream's keys of earlier tokens; each
//     row starts from the state the own-token pre-pass (k_sfa_transient.cu)
//     left in o and lse.
// Only unmasked or partly masked KV tiles are visited; the grid is ordered
// longest-first inside chunks of problems whose K/V fit in L2 together, so
// the hardware scheduler balances the triangle and K/V come from DRAM about
// once.
//
// Roles (320 threads):
//   warps 0-3   softmax of tile A, one thread per query row (TMEM lane = row)
//   warps 4-7   softmax of tile B
//   warp 8      TMA producer: Q_A, Q_B once, then K_j / V_j into a ring of
//               shared-memory stages (128B swizzle), completion on mbarriers
//   warp 9      TMEM owner and MMA issuer (one thread; it shares a scheduler
//               with two softmax warps, so its instruction count matters):
//                 S_x(j) = Q_x K_j^T  tcgen05.mma SS, M=128 N=128 K=D -> TMEM
//                 O_x   += P_x(j) V_j tcgen05.mma TS, A = P_x(j) in TMEM (bf16,
//                                     written over S_x(j)), B = V_j MN-major
//               issue order per KV tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1),
//               so the tensor core works on one tile while the other tile's
//               softmax runs (the two warpgroups ping-pong).
// The softmax scales with one packed FFMA per score pair into the log2
// domain, masks the diagonal tile (and the window's leading edge), keeps the
// running max and two running sums (of the fp32 P, for the log-sum-exp, and
// one that counts P as rounded to bf16 wherever that rounding could reach O,
// for normalising O), evaluates 2^x on MUFU for most
// pairs and on the FMA pipe (ex2_poly) for one pair in kPolyEvery, writes P
// back to TMEM, and rescales O in TMEM only when its running max grew by more
// than 2^60 (then and only then it waits for the previous PV).  The epilogue
// normalises O, stages it in the tile's Q buffer and TMA-stores it.
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [256+D,256+2D).
//
// Persistent variants (one CTA per SM looping over the items, the next item's
// loads and first QK^T overlapping this item's tail) measured slower than
// this one-item-per-CTA form: 3-9% on cross-stream prefill, at most 1% faster
// on the short within-stream problems.
#include <cfloat>

#include "hd_kernels.cuh"

namespace hd {

namespace {

constexpr int kBM = 128;      // query rows per tile (MMA M)
constexpr int kBN = 128;      // keys per KV tile
constexpr int kThreads = 320;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kStages = 2;    // K/V ring depth
constexpr uint32_t kTmemCols = 512;
constexpr int kBoxBytes = 128 * 128;  // 128 rows x 128 B (64 bf16)
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
// Rescale O only when the running row max grows by more than this (log2
// units).  Weights are then at most 2^60, sums of up to 2^15 keys at most
// 2^75 and O at most 2^75 times max |v|: far inside fp32 and bf16 range, with
// the same relative precision as at 2^0.  On keys with outliers the max grows
// by tens of log2 units along a row, so a small threshold would rescale O
// (a TMEM round trip of every O column) several times per row.
constexpr float kRescaleThreshold = 60.0f;
constexpr int kPolyEvery = 4;
// Paged K/V: page-table entries a CTA reads into shared memory before its
// first copy (entries past these are read from global memory when needed).
// Sized so the kernel's shared memory, with the 1 KB the system reserves per
// CTA, stays within the 196 KB carve-out (60 KB of L1 left); at 228 KB the
// transient kind, whose rows start from global-memory state, ran 8% slower.
constexpr int kPageCache = 256;

template <int D>
struct PCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // a Q, K or V tile of 128 rows
  static constexpr int kSmemQ = 0;                       // Q_A, Q_B
  static constexpr int kSmemK = kSmemQ + 2 * kTileBytes;
  static constexpr int kSmemV = kSmemK + kStages * kTileBytes;
  static constexpr int kSmemBar = kSmemV + kStages * kTileBytes;
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 2 + 1 + 1 + 1;
  static constexpr int kSmemTmemPtr = kSmemBar + kNumBars * 8;
  static constexpr int kSmemPages = kSmemTmemPtr + 16;  // paged K/V: this CTA's page ids
  static constexpr int kSmemBytes = kSmemPages + kPageCache * 4;
  static constexpr size_t kDynSmem = 1024 + kSmemBytes;
  __host__ __device__ static constexpr uint32_t col_s(int x) { return (uint32_t)x * 128u; }
  __host__ __device__ static constexpr uint32_t col_o(int x) { return 256u + (uint32_t)x * D; }
};

static_assert(PCfg<128>::kDynSmem + 1024 <= 196 * 1024,
              "prefill shared memory must fit the 196 KB carve-out");

struct Bars {
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_full, *mma_done;
  uint64_t *v_fixed;  // paged K/V: the last V tile's rows past the sequence are zeroed
  uint64_t *q_full_b;  // Q of tile B (q_full: Q of tile A)
};

__device__ __forceinline__ Bars carve_bars(uint8_t *base) {
  uint64_t *b = reinterpret_cast<uint64_t *>(base);
  Bars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = r.k_full + kStages;
  r.v_full = r.k_empty + kStages;
  r.v_empty = r.v_full + kStages;
  r.s_full = r.v_empty + kStages;  // [2] per query tile
  r.p_full = r.s_full + 2;         // [2]
  r.o_full = r.p_full + 2;         // [2]
  r.mma_done = r.o_full + 2;       // [1]
  r.v_fixed = r.mma_done + 1;      // [1]
  r.q_full_b = r.v_fixed + 1;      // [1]
  return r;
}

// First key position a query at position `pos` may attend in the cross-stream
// sliding-window mode: all n streams of the last `window` tokens.
__device__ __forceinline__ int window_lo(const PrefillParams &p, int pos) {
  const int t0 = pos / p.n - p.window + 1;
  return t0 > 0 ? t0 * p.n : 0;
}

// TMA coordinates of row `row0` of the problem's sequence for head `head`.
__device__ __forceinline__ void load_tile(void *dst, const CUtensorMap *m, uint64_t *bar, int dcol,
                                          int head, int stream, int row0, int batch, bool within) {
  if (within)
    tma_load_5d(dst, m, bar, dcol, head, stream, row0, batch);
  else
    tma_load_4d(dst, m, bar, dcol, head, row0, batch);
}

// Work item `it` -> (query-tile pair qp, problem).  Problems are numbered
// (batch, stream, head) with the head fastest, so the heads of one KV group
// are adjacent; the list walks them in chunks of p.chunk_problems (whole KV
// groups whose K/V fit in L2 together), and inside a chunk the heaviest
// pairs (last rows of the causal triangle) come first, all of the chunk's
// problems at one pair before the next lighter pair.  A chunk's K/V is thus
// read from DRAM about once, and the list still ends with light items.
__device__ __forceinline__ void item_coords(const PrefillParams &p, int64_t it, int &qp,
                                            int64_t &prob) {
  const int q_pairs = (p.q_tiles + 1) / 2;
  const int64_t C = p.chunk_problems;
  const int64_t c = it / (C * q_pairs);
  const int64_t rem = it - c * C * q_pairs;
  const int64_t Cc = min(C, p.problems - c * C);  // the last chunk may be short
  qp = q_pairs - 1 - (int)(rem / Cc);
  prob = c * C + rem % Cc;
}

// One softmax step of the query row in this thread's TMEM lane over KV tile
// j: S from TMEM, the causal edge at the row's position qabs (and, with a
// window, its start lo_row), the running max m (log2 units), P = 2^(S*scale -
// max) as bf16 written over S, and the lazy O rescale.  Two running sums: l
// of the fp32 weights, for the log-sum-exp, and lr, by which O is normalised:
// it counts weights as rounded to the bf16 the PV product multiplies V with,
// wherever their rounding could reach O (so when keys dominate a row their
// rounding cancels): the tile's largest weight where it is at least 1/4 of
// the row's sum so far (in any lane of the warp), and the whole tile where
// besides the other weights hold more than 1/8 of it (or the largest
// weight's rounding depends on which exp2 form computed it).  The weights it
// counts as computed are then either each at most 1/4 of the sum (their
// rounding errors, at most 2^-8 of each, average out) or together at most
// 1/8 of it.
// o_live: O holds data a new max must rescale; o_prev: a PV of this row may
// still be in flight, so a rescale first waits for it (o_bar, parity o_par).
// Returns false if that bounded wait gave up.
template <int D, bool kWindow, bool kTransient>
__device__ __forceinline__ bool softmax_step(uint32_t s_tmem, uint32_t o_tmem, int j, int qabs,
                                             int lo_row, float sl2, float &m, float &l, float &lr,
                                             bool o_live, bool o_prev, uint64_t *o_bar,
                                             uint32_t o_par) {
  float sv[kBN];
  {
    uint32_t r0[32], r1[32], r2[32], r3[32];
    tmem_ld32(s_tmem + 0, r0);
    tmem_ld32(s_tmem + 32, r1);
    tmem_ld32(s_tmem + 64, r2);
    tmem_ld32(s_tmem + 96, r3);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      sv[i] = __uint_as_float(r0[i]);
      sv[32 + i] = __uint_as_float(r1[i]);
      sv[64 + i] = __uint_as_float(r2[i]);
      sv[96 + i] = __uint_as_float(r3[i]);
    }
  }
  {  // keys after the query (at or after it, in transient mode) are masked
    const int lim = qabs - j * kBN;
    if (lim < (kTransient ? kBN : kBN - 1)) {
#pragma unroll
      for (int i = 0; i < kBN; ++i)
        if (kTransient ? (i >= lim) : (i > lim)) sv[i] = -INFINITY;
    }
  }
  if (kWindow && lo_row > j * kBN) {  // keys before the window are masked
    const int lo = lo_row - j * kBN;
#pragma unroll
    for (int i = 0; i < kBN; ++i)
      if (i < lo) sv[i] = -INFINITY;
  }
  // row max of the raw scores (scale > 0): eight chains of 3-input max
  float mc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mc[c] = fmaxf(sv[2 * c], sv[2 * c + 1]);
#pragma unroll
  for (int k = 1; k < kBN / 16; ++k)
#pragma unroll
    for (int c = 0; c < 8; ++c) mc[c] = max3(mc[c], sv[16 * k + 2 * c], sv[16 * k + 2 * c + 1]);
  const float mx = fmaxf(max3(mc[0], mc[1], mc[2]),
                         fmaxf(max3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7])));
  const float m_cand = fmaxf(m, mx * sl2);
  const bool need = m_cand > m + kRescaleThreshold;
  const float m_new = need ? m_cand : m;
  const float base = (m_new == -INFINITY) ? 0.f : m_new;
  // The tile's largest weight.
  const float xm = fmaf(mx, sl2, -base);
  const float pm = ex2_approx(xm);
  // P = 2^(S*scale*log2e - base) in bf16, written over S: keys 32c .. 32c+31
  // pack into the 16 columns starting at 16c (two keys per column).  One
  // pair in kPolyEvery goes through the FMA-pipe exp2, the rest through MUFU.
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t nbase2 = f2_pack(-base, -base);
  uint64_t acc2 = 0ull;
#pragma unroll
  for (int c = 0; c < kBN / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int q = c * 16 + i;
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(sv[2 * q], sv[2 * q + 1]), scale2, nbase2), x0, x1);
      float p0, p1;
      if (q % kPolyEvery == 0) {
        p0 = ex2_poly(x0);
        p1 = ex2_poly(x1);
      } else {
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      acc2 = f2_add(acc2, f2_pack(p0, p1));
      pk[i] = pack_bf16x2(p0, p1);
    }
    tmem_st16(s_tmem + c * 16, pk);
  }
  float rs;
  {
    float lo, hi;
    f2_unpack(acc2, lo, hi);
    rs = lo + hi;
  }
  const float alpha = ex2_approx(m - base);
  l = l * alpha + rs;
  // Where the tile's largest weight is a sizeable share of the row's sum so
  // far it counts rounded to bf16.  It was computed by one of the two exp2
  // forms, whichever its key's lane uses; where their roundings differ (a
  // rounding midpoint between them), or where the other weights are a
  // sizeable share too, the whole tile's rounded sum is read back from TMEM
  // instead.
  float rsr = rs;
  if (__any_sync(0xffffffffu, pm > 0.25f * l)) {
    const uint32_t pmb = pack_bf16x2(pm, ex2_poly(xm));
    rsr = rs + (__uint_as_float(pmb << 16) - pm);
    if (__any_sync(0xffffffffu, pm > 0.25f * l &&
                                    (rs - pm > 0.125f * l || (pmb >> 16) != (pmb & 0xffffu)))) {
      tmem_wait_st();
      uint32_t r0[32], r1[32];
      tmem_ld32(s_tmem + 0, r0);
      tmem_ld32(s_tmem + 32, r1);
      tmem_wait_ld();
      uint64_t accr2 = 0ull;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        // bf16 pairs back to fp32: low half-word shifted up, high half-word masked
        accr2 = f2_add(accr2, f2_pack(__uint_as_float(r0[i] << 16),
                                      __uint_as_float(r0[i] & 0xffff0000u)));
        accr2 = f2_add(accr2, f2_pack(__uint_as_float(r1[i] << 16),
                                      __uint_as_float(r1[i] & 0xffff0000u)));
      }
      float lo, hi;
      f2_unpack(accr2, lo, hi);
      rsr = lo + hi;
    }
  }
  lr = lr * alpha + rsr;
  if (o_live && __any_sync(0xffffffffu, need)) {
    // (uniform over the warp, like every wait of the softmax loop: its lanes
    // leave the loop together or not at all)
    if (!__all_sync(0xffffffffu, !o_prev || mbar_wait(o_bar, o_par))) return false;
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(o_tmem + c * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
      tmem_st32(o_tmem + c * 32, r);
    }
  }
  tmem_wait_st();
  m = m_new;
  return true;
}

// kKind selects the masks compiled in: 0 within / cross (by p.mode), 1 the
// cross-stream sliding window (mode 2), 2 transient intermediate streams
// (mode 3).  Each kind is its own instantiation, so the within / cross
// kernels carry none of the other masks' code.
template <int D, int kKind>
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
  int32_t *page_ids = reinterpret_cast<int32_t *>(smem + Cfg::kSmemPages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool kWindow = (kKind == 1);
  constexpr bool kTransient = (kKind == 2);
  // Transient mode runs on the within-stream decomposition: query stream s,
  // keys from the final stream n-1 of strictly earlier tokens (its own
  // token's streams come from a pre-pass, the state each row starts from).
  const bool within = (p.mode == 0 || kTransient);

  int qp;
  int64_t prob;
  item_coords(p, blockIdx.x, qp, prob);
  const int h = (int)(prob % p.Hq);
  prob /= p.Hq;
  const int s = within ? (int)(prob % p.n) : 0;
  const int b = within ? (int)(prob / p.n) : (int)prob;
  const int g = h / p.G;
  const int kv_s = kTransient ? p.n - 1 : s;  // stream coordinate of the K/V views
  const int q0 = qp * 2 * kBM;               // first row of tile A
  // Rows of this problem: p.seq, or this sequence's own chunk length in a
  // variable-length chunk batch (o rows past it in its last tile hold
  // unspecified values; their lse is not written).
  int seq = p.seq;
  if (p.chunk_len) {
    const int cb = p.chunk_len[b];
    if (cb < 0 || cb > (within ? p.seq : p.seq / p.n)) {
      if (threadIdx.x == 0) report(p.dev_status, kDevBadLength);
      return;  // uniform over the CTA, before any barrier or TMEM allocation
    }
    seq = within ? cb : cb * p.n;
    if (q0 >= seq) return;  // no row of this CTA belongs to the sequence
  }
  // Queries' offset among the keys: the cached prefix of a chunk (per sequence
  // for a paged cache, whose prefix must fit the sequence's page table).
  int q_off = p.q_off;
  if (p.prefix) {
    const int pre = p.prefix[b];
    const int64_t tokens = (int64_t)pre + (within ? seq : seq / p.n);
    if (pre < 0 || tokens > (int64_t)p.max_pages * p.page_tokens) {
      if (threadIdx.x == 0) report(p.dev_status, kDevBadLength);
      return;  // uniform over the CTA, before any barrier or TMEM allocation
    }
    q_off = within ? pre : pre * p.n;
  }
  // Keys of the sequence (rows of its view): a V row at or past this is stale.
  const int key_end = q_off + seq;
  const bool hasB = q0 + kBM < seq;          // tile B holds at least one real row
  // KV tiles each query tile needs: up to the tile of its last real row's
  // absolute position (queries start q_off positions into the keys when a
  // chunk follows a cached prefix; q_off = 0 otherwise).
  const int ntA = (int)((q_off + min(q0 + kBM - 1, seq - 1)) / kBN) + 1;
  const int ntB = hasB ? (int)((q_off + min(q0 + 2 * kBM - 1, seq - 1)) / kBN) + 1 : ntA;
  const int nt = hasB ? ntB : ntA;
  // First KV tile each query tile needs: 0, or the tile holding its first
  // row's window start in the sliding-window mode.  K/V tiles jbeg .. nt-1
  // stream through the ring; ring slot of tile j is (j - jbeg) % kStages.
  const int j0A = kWindow ? (int)(window_lo(p, q_off + q0) / kBN) : 0;
  const int j0B = (kWindow && hasB) ? (int)(window_lo(p, q_off + q0 + kBM) / kBN) : j0A;
  // Paged K/V: the last tile's V rows past the sequence come from a stale page
  // and are zeroed before their product (a zero probability times NaN is NaN).
  const bool fix_last = p.page_table && (nt * kBN > key_end);
  const int jbeg = j0A;

  // The producer thread sets up the barriers and, over a contiguous K/V
  // view, issues the Q tiles and the first K/V tile before the CTA-wide
  // barrier, so the copies are in flight while TMEM is allocated.
  const bool early = !p.page_table;
  if (threadIdx.x == kWarpTma * 32) {
    mbar_init(bar.q_full, 1);
    mbar_init(bar.q_full_b, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar.k_full[i], 1);
      mbar_init(&bar.k_empty[i], 1);
      mbar_init(&bar.v_full[i], 1);
      mbar_init(&bar.v_empty[i], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar.s_full[x], 1);
      mbar_init(&bar.p_full[x], 4);  // one arrival per softmax warp
      mbar_init(&bar.o_full[x], 1);
    }
    mbar_init(bar.mma_done, 1);
    mbar_init(bar.v_fixed, 1);
    fence_barrier_init();
    if (early) {
      fence_proxy_async_smem();  // the initialised barriers, before the copies signal them
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // In the order the first products need them: Q_A and K of the first tile
      // (S_A), then Q_B (S_B), then V (the first PV); ring slot 0 is free.
      mbar_arrive_expect_tx(bar.q_full, Cfg::kTileBytes);
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c)
        load_tile(sQ + c * kBoxBytes, &tm_q, bar.q_full, c * 64, h, s, q0, b, within);
      mbar_arrive_expect_tx(&bar.k_full[0], Cfg::kTileBytes);
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c)
        load_tile(sK + c * kBoxBytes, &tm_k, &bar.k_full[0], c * 64, g, kv_s, jbeg * kBN, b,
                  within);
      if (hasB) {
        mbar_arrive_expect_tx(bar.q_full_b, Cfg::kTileBytes);
#pragma unroll
        for (int c = 0; c < Cfg::kBoxes; ++c)
          load_tile(sQ + Cfg::kTileBytes + c * kBoxBytes, &tm_q, bar.q_full_b, c * 64, h, s,
                    q0 + kBM, b, within);
      }
      mbar_arrive_expect_tx(&bar.v_full[0], Cfg::kTileBytes);
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c)
        load_tile(sV + c * kBoxBytes, &tm_v, &bar.v_full[0], c * 64, g, kv_s, jbeg * kBN, b,
                  within);
    }
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
    // Paged K/V: the page ids of this CTA's tiles, read by the whole warp at
    // once, so that no copy waits on a page-table load.
    const int per_page = within ? p.page_tokens : p.page_rows;
    const int pi0 = p.page_table ? (jbeg * kBN) / per_page : 0;
    if (p.page_table) {
      const int32_t *tab = p.page_table + (int64_t)b * p.max_pages;
      const int cnt = min((nt * kBN - 1) / per_page - pi0 + 1, kPageCache);
      for (int i = lane; i < cnt; i += 32) {
        const int pi = pi0 + i;
        page_ids[i] = pi < p.max_pages ? __ldg(tab + pi) : -1;
      }
      __syncwarp();
    }
    if (lane == 0) {
      tma_prefetch_desc(&tm_o);
      if (!early) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        mbar_arrive_expect_tx(bar.q_full, Cfg::kTileBytes);
        if (hasB) mbar_arrive_expect_tx(bar.q_full_b, Cfg::kTileBytes);
#pragma unroll
        for (int c = 0; c < Cfg::kBoxes; ++c) {
          load_tile(sQ + c * kBoxBytes, &tm_q, bar.q_full, c * 64, h, s, q0, b, within);
          if (hasB)
            load_tile(sQ + Cfg::kTileBytes + c * kBoxBytes, &tm_q, bar.q_full_b, c * 64, h, s,
                      q0 + kBM, b, within);
        }
      }
      // K or V tile j: one view of a contiguous tensor, or rows of the page pool
      // (cross-stream: one box, a page holds whole tiles; within-stream: boxes
      // of box_tokens tokens of stream kv_s, one page each).
      auto load_kv = [&](uint8_t *dst, const CUtensorMap *m, uint64_t *bar_, int j) {
        if (!p.page_table) {
#pragma unroll
          for (int c = 0; c < Cfg::kBoxes; ++c)
            load_tile(dst + c * kBoxBytes, m, bar_, c * 64, g, kv_s, j * kBN, b, within);
          return;
        }
        const int32_t *tab = p.page_table + (int64_t)b * p.max_pages;
        const int rows = within ? p.box_tokens : kBN;
        for (int sub = 0; sub < kBN / rows; ++sub) {
          const int r0 = j * kBN + sub * rows;  // token (within) or position (cross)
          const int pi = r0 / per_page;
          int page = pi - pi0 < kPageCache ? page_ids[pi - pi0]
                     : pi < p.max_pages   ? __ldg(tab + pi)
                                          : -1;
          if (page < 0 || page >= p.num_pages) {
            if (r0 < key_end) report(p.dev_status, kDevPageRange);
            page = p.num_pages;  // past the pool: the box reads as zeros
          }
#pragma unroll
          for (int c = 0; c < Cfg::kBoxes; ++c) {
            uint8_t *d = dst + c * kBoxBytes + sub * rows * 128;
            if (within)
              tma_load_5d(d, m, bar_, c * 64, g, kv_s, r0 % per_page, page);
            else
              tma_load_4d(d, m, bar_, c * 64, g, r0 % per_page, page);
          }
        }
      };
      // the first tile went out before the CTA-wide barrier (contiguous K/V)
      int k_issued = early ? 1 : 0, v_issued = early ? 1 : 0;
      bool ok = true;
      for (int j = jbeg + (early ? 1 : 0); j < nt; ++j) {
        const int r = j - jbeg;
        const int st = r % kStages;
        const uint32_t ph = ((r / kStages) & 1) ^ 1;
        uint8_t *kd = sK + st * Cfg::kTileBytes;
        uint8_t *vd = sV + st * Cfg::kTileBytes;
        if (!(ok = mbar_wait(&bar.k_empty[st], ph))) break;
        mbar_arrive_expect_tx(&bar.k_full[st], Cfg::kTileBytes);
        load_kv(kd, &tm_k, &bar.k_full[st], j);
        k_issued = r + 1;
        if (!(ok = mbar_wait(&bar.v_empty[st], ph))) break;
        mbar_arrive_expect_tx(&bar.v_full[st], Cfg::kTileBytes);
        load_kv(vd, &tm_v, &bar.v_full[st], j);
        v_issued = r + 1;
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      // Every copy issued must land before the CTA can exit (in the normal
      // path the consumers have already waited for all of them).
      bool drained = mbar_wait(bar.q_full, 0) && (!hasB || mbar_wait(bar.q_full_b, 0));
      for (int j = max(0, k_issued - kStages); j < k_issued && drained; ++j)
        drained = mbar_wait(&bar.k_full[j % kStages], (j / kStages) & 1);
      for (int j = max(0, v_issued - kStages); j < v_issued && drained; ++j)
        drained = mbar_wait(&bar.v_full[j % kStages], (j / kStages) & 1);
      if (!drained) report(p.dev_status, kDevTimeout);
    }
    // Lane 0 has issued every copy and waited for the last ones, so the
    // last V stage's barrier is at its final phase for the other lanes too.
    __syncwarp();
    if (fix_last) {
      // Paged K/V: once the last V tile has landed, the whole warp zeroes its
      // rows past the sequence, then releases it to the MMA thread.
      const int jl = nt - 1, rl = jl - jbeg, stl = rl % kStages;
      const bool okw = mbar_wait(&bar.v_full[stl], (rl / kStages) & 1);
      if (okw) {
        const int first = max(0, key_end - jl * kBN);  // first stale row of the tile
        uint8_t *vd = sV + stl * Cfg::kTileBytes;
        for (int idx = lane; idx < (kBN - first) * Cfg::kBoxes * 8; idx += 32) {
          const int rr = first + idx / (Cfg::kBoxes * 8), rem = idx % (Cfg::kBoxes * 8);
          *reinterpret_cast<uint4 *>(vd + (rem >> 3) * kBoxBytes + sw128_offset(rr, rem & 7)) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();  // generic writes, read next by the tensor core
      }
      __syncwarp();
      if (lane == 0) {
        if (!okw) report(p.dev_status, kDevTimeout);
        mbar_arrive(bar.v_fixed);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t k_base = smem_u32(sK);
      const uint32_t v_base = smem_u32(sV);
      // Shared-memory descriptors of the operand buffers, built once: the start
      // address field is address / 16 in bits 0-13, so the descriptor of
      // base + off is the base's plus off / 16 (shared memory ends below 2^18
      // bytes: no carry out of the field).  The issuing thread then spends one
      // add per operand per product.
      constexpr uint64_t kTileDesc = Cfg::kTileBytes >> 4;
      const uint64_t dq0 = smem_desc_sw128(q_base, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(k_base, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(v_base, kBoxBytes, 1024);
      auto issue_s = [&](int x, int j) {
        const uint64_t dq = dq0 + (uint64_t)x * kTileDesc;
        const uint64_t dk = dk0 + (uint64_t)((j - jbeg) % kStages) * kTileDesc;
        const uint32_t dt = tmem + Cfg::col_s(x);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4);
          mma_ss(dt, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {
        const uint64_t dv = dv0 + (uint64_t)((j - jbeg) % kStages) * kTileDesc;
        const uint32_t dt = tmem + Cfg::col_o(x), at = tmem + Cfg::col_s(x);
        const uint32_t acc0 = (kTransient || j > (x ? j0B : j0A)) ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(dt, at + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
        mma_commit(&bar.o_full[x]);
      };
      // Q of tile B has its own barrier: S_A(0) need not wait for it.
      bool qb_ready = false;
      auto wait_qb = [&]() -> bool {
        if (!qb_ready) qb_ready = mbar_wait(bar.q_full_b, 0);
        if (qb_ready) tc_fence_after();
        return qb_ready;
      };
      bool ok = mbar_wait(bar.q_full, 0) && mbar_wait(&bar.k_full[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, jbeg);
        if (hasB && j0B == jbeg) {
          if ((ok = wait_qb())) issue_s(1, jbeg);
        }
        mma_commit(&bar.k_empty[0]);
      }
      for (int j = jbeg; j < nt && ok; ++j) {
        const int r = j - jbeg;
        const int st = r % kStages;
        const uint32_t vph = (r / kStages) & 1;
        bool v_ready = false;
        const bool wait_fix = fix_last && j == nt - 1;
        if (j < ntA) {
          if (!(ok = mbar_wait(&bar.p_full[0], (j - j0A) & 1) && mbar_wait(&bar.v_full[st], vph) &&
                     (!wait_fix || mbar_wait(bar.v_fixed, 0))))
            break;
          v_ready = true;
          tc_fence_after();
          issue_pv(0, j);
        }
        const int jn = j + 1;
        const int rn = r + 1;
        if (jn < nt) {
          if (!(ok = mbar_wait(&bar.k_full[rn % kStages], (rn / kStages) & 1))) break;
          tc_fence_after();
          if (jn < ntA) issue_s(0, jn);
        }
        if (hasB && j >= j0B) {
          if (!(ok = mbar_wait(&bar.p_full[1], (j - j0B) & 1) &&
                     (v_ready || (mbar_wait(&bar.v_full[st], vph) &&
                                  (!wait_fix || mbar_wait(bar.v_fixed, 0))))))
            break;
          tc_fence_after();
          issue_pv(1, j);
        }
        mma_commit(&bar.v_empty[st]);
        if (jn < nt) {
          if (hasB && jn >= j0B) {
            if (!(ok = wait_qb())) break;
            issue_s(1, jn);
          }
          mma_commit(&bar.k_empty[rn % kStages]);
        }
      }
      if (!ok) report(p.dev_status, kDevTimeout);
      // All MMAs this thread issued must finish before TMEM is released.
      mma_commit(bar.mma_done);
      if (!mbar_wait(bar.mma_done, 0)) report(p.dev_status, kDevTimeout);
    }
  } else if (warp < 8 && (warp < 4 || hasB)) {
    // ------------------------------------------------------------ softmax
    const int x = warp >> 2;              // query tile: 0 = A, 1 = B
    const int wq = warp & 3;              // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;       // query row inside the tile
    const int qpos = q0 + x * kBM + row;      // query row inside the problem's sequence
    const int qabs = q_off + qpos;            // its position among the keys (< 2^30)
    const int ntx = x ? ntB : ntA;
    const int j0x = x ? j0B : j0A;
    const int lo_row = kWindow ? window_lo(p, qabs) : 0;
    const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
    const uint32_t s_tmem = tmem + lane_addr + Cfg::col_s(x);
    const uint32_t o_tmem = tmem + lane_addr + Cfg::col_o(x);
    const float sl2 = p.scale_log2;
    // running max (log2 units) and sums of 2^(x - m): fp32 (l) and as rounded
    // to the bf16 P of the PV products (lr)
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    if constexpr (kTransient) {
      // The current token's streams 0..s are keys the final-stream view does
      // not hold.  A pre-pass has left their part of the row in o (normalised)
      // and lse: the row starts from that state (max = its log-sum-exp, sum 1,
      // O = its output) and every PV accumulates onto it (the order of keys
      // does not change the result).  Rows past the sequence start from zero.
      uint4 ov[D / 8];
      if (qpos < seq) {
        const int64_t pos = (int64_t)qpos * p.n + s;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            p.o_own + (((int64_t)b * p.N + pos) * p.Hq + h) * D);
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) ov[c8] = src[c8];
        m = p.lse[((int64_t)b * p.Hq + h) * p.N + pos] * kLog2e;
        l = 1.f;
        lr = 1.f;
      } else {
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) ov[c8] = make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t w[4] = {ov[c * 4 + q4].x, ov[c * 4 + q4].y, ov[c * 4 + q4].z,
                                 ov[c * 4 + q4].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            r[q4 * 8 + 2 * e] = w[e] << 16;               // bf16 -> fp32, low element
            r[q4 * 8 + 2 * e + 1] = w[e] & 0xffff0000u;   // high element
          }
        }
        tmem_st32(o_tmem + c * 32, r);
      }
      tmem_wait_st();  // the first PV (which accumulates) follows this row's p_full arrive
    }
    for (int j = j0x; j < ntx; ++j) {
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bar.s_full[x], (j - j0x) & 1)))) break;
      tc_fence_after();
      // O holds PV_x(j-1) (and, in the transient mode, the current token's
      // streams from the start) and is rescaled for the new max.
      if (!(ok = softmax_step<D, kWindow, kTransient>(s_tmem, o_tmem, j, qabs, lo_row, sl2, m, l,
                                                      lr, kTransient || j > j0x, j > j0x,
                                                      &bar.o_full[x], (j - 1 - j0x) & 1)))
        break;
      // Each lane's P stores are complete (tcgen05.wait::st in the step) and
      // fenced; the warp's lanes meet, then one arrival stands for all 32.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[x]);
    }
    // uniform over the warp: the epilogue's TMEM loads are warp-collective
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.o_full[x], (ntx - 1 - j0x) & 1));
    if (!ok) report(p.dev_status, kDevTimeout);
    uint8_t *stage = sQ + x * Cfg::kTileBytes;  // Q_x is no longer read by any MMA
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / lr;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(o_tmem + c * 32, r);
        tmem_wait_ld();
        // 32 fp32 -> 16 packed bf16x2 = four 16-byte chunks of this row.
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = c * 32 + q * 8;  // first element of the chunk
          uint8_t *dst = stage + (col >> 6) * kBoxBytes + sw128_offset(row, (col & 63) >> 3);
          *reinterpret_cast<uint4 *>(dst) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                                                       pk[4 * q + 3]);
        }
      }
      if (p.lse && qpos < seq) {
        const int64_t pos = within ? (int64_t)qpos * p.n + s : (int64_t)qpos;
        p.lse[((int64_t)b * p.Hq + h) * p.N + pos] = (m + __log2f(l)) * kLn2;
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    named_bar_sync(1 + x, 128);
    if (ok && wq == 0 && lane == 0) {
      const int r0 = q0 + x * kBM;
#pragma unroll
      for (int c = 0; c < Cfg::kBoxes; ++c) {
        if (within)
          tma_store_5d(&tm_o, stage + c * kBoxBytes, c * 64, h, s, r0, b);
        else
          tma_store_4d(&tm_o, stage + c * kBoxBytes, c * 64, h, r0, b);
      }
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

template <int D, int kKind>
cudaError_t prepare_prefill() {
  static int done_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (done_dev == dev) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(sfa_prefill_kernel<D, kKind>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PCfg<D>::kDynSmem);
  if (e == cudaSuccess) done_dev = dev;
  return e;
}

template <int D, int kKind>
cudaError_t launch_one(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                       const CUtensorMap &tm_o, const PrefillParams &p, int64_t ctas,
                       cudaStream_t stream) {
  cudaError_t e = prepare_prefill<D, kKind>();
  if (e != cudaSuccess) return e;
  sfa_prefill_kernel<D, kKind><<<(unsigned)ctas, kThreads, PCfg<D>::kDynSmem, stream>>>(
      tm_q, tm_k, tm_v, tm_o, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sfa_prefill(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                               const CUtensorMap &tm_v, const CUtensorMap &tm_o,
                               const PrefillParams &p, int D, cudaStream_t stream) {
  const int64_t ctas = p.problems * ((p.q_tiles + 1) / 2);
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int kind = (p.mode == 2) ? 1 : (p.mode == 3) ? 2 : 0;
  if (D == 128) {
    if (kind == 1) return launch_one<128, 1>(tm_q, tm_k, tm_v, tm_o, p, ctas, stream);
    if (kind == 2) return launch_one<128, 2>(tm_q, tm_k, tm_v, tm_o, p, ctas, stream);
    return launch_one<128, 0>(tm_q, tm_k, tm_v, tm_o, p, ctas, stream);
  }
  if (kind == 1) return launch_one<64, 1>(tm_q, tm_k, tm_v, tm_o, p, ctas, stream);
  if (kind == 2) return launch_one<64, 2>(tm_q, tm_k, tm_v, tm_o, p, ctas, stream);
  return launch_one<64, 0>(tm_q, tm_k, tm_v, tm_o, p, ctas, stream);
}

}  // namespace hd
