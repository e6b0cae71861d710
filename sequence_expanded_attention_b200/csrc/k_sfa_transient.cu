// Transient intermediate streams (the PHD-style control mask): the pre-pass
// over each row's own token.
//
// Under this mask query (t, s) sees the final stream n-1 of every earlier
// token and streams 0..s of its own token t ("Hidden Decoding at Scale"
// review, "Prior limitations": the PHD-style control whose intermediate
// streams serve their own token and are not kept as context).  The earlier
// tokens' part is a within-stream causal problem on the tensor cores (the
// prefill kernel's transient kind); the own-token part, at most n keys per
// row, is this pre-pass: it leaves each row's normalised output in o and its
// log-sum-exp in lse, and the prefill kernel starts the row from that state.
// Memory-bound: q and the token's K/V rows read once, o written once (about
// 3.7 TB/s on the Qwen3-8B shapes, set by the loads its registers keep in
// flight).
#include <cstdint>
#include <type_traits>

#include "hd_kernels.cuh"

namespace hd {
namespace {
constexpr float kLn2 = 0.6931471805599453f;
}  // namespace

// Transient mode, current token: row (b, t, s, h) attends to streams 0..s of
// its own token t.  One warp per (b, t, KV group): the token's n K and V rows
// are loaded once (D/32 elements per lane) and serve the group's Hq/Hkv heads.
// For each head the n query rows are loaded together, the n(n+1)/2 scores are
// lane partials summed across the warp in one pass (independent shuffles), and
// each row's softmax over its s+1 keys gives its output.  Writes the
// normalised output into o and the natural-log sum-exp into lse, the state
// the main kernel starts each row from.  kNMax bounds n (4 or 8).
template <int D, int kNMax>
__global__ void __launch_bounds__(128)
    transient_own_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                         const __nv_bfloat16 *__restrict__ v, __nv_bfloat16 *__restrict__ o,
                         float *__restrict__ lse, int64_t B, int64_t L, int n, int Hq, int Hkv,
                         float scale_log2) {
  constexpr int E = D / 32;  // elements per lane: 4 (8 bytes) or 2 (4 bytes)
  using Vec = typename std::conditional<E == 4, uint2, uint32_t>::type;
  const int64_t wid = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= B * L * Hkv) return;
  const int g = (int)(wid % Hkv);
  const int64_t t = (wid / Hkv) % L, b = wid / Hkv / L;
  const int64_t N = (int64_t)n * L;
  const int64_t row0 = b * N + t * n;  // stream 0 of token t
  auto unpack = [](Vec w, float *f) {
    if constexpr (E == 4) {
      f[0] = __uint_as_float(w.x << 16);
      f[1] = __uint_as_float(w.x & 0xffff0000u);
      f[2] = __uint_as_float(w.y << 16);
      f[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
      f[0] = __uint_as_float(w << 16);
      f[1] = __uint_as_float(w & 0xffff0000u);
    }
  };
  Vec kw[kNMax], vw[kNMax];
#pragma unroll
  for (int sp = 0; sp < kNMax; ++sp) {
    if (sp < n) {
      const int64_t off = ((row0 + sp) * Hkv + g) * D + lane * E;
      kw[sp] = *reinterpret_cast<const Vec *>(k + off);
      vw[sp] = *reinterpret_cast<const Vec *>(v + off);
    }
  }
  const int G = Hq / Hkv;
  // the query rows of head hh + 1 are loaded while head hh is computed
  Vec qw[kNMax], qn[kNMax];
#pragma unroll
  for (int s = 0; s < kNMax; ++s)
    if (s < n) qn[s] = *reinterpret_cast<const Vec *>(q + ((row0 + s) * Hq + g * G) * D + lane * E);
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
#pragma unroll
    for (int s = 0; s < kNMax; ++s) {
      qw[s] = qn[s];
      if (s < n && hh + 1 < G)
        qn[s] = *reinterpret_cast<const Vec *>(q + ((row0 + s) * Hq + h + 1) * D + lane * E);
    }
    // x[s][sp], sp <= s: this lane's part of q_s . k_sp, then the warp sum
    float x[kNMax][kNMax];
#pragma unroll
    for (int s = 0; s < kNMax; ++s) {
      if (s < n) {
        float qf[E];
        unpack(qw[s], qf);
#pragma unroll
        for (int sp = 0; sp <= s; ++sp) {
          float kf[E];
          unpack(kw[sp], kf);
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) d = fmaf(qf[e], kf[e], d);
          x[s][sp] = d;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int s = 0; s < kNMax; ++s)
        if (s < n) {
#pragma unroll
          for (int sp = 0; sp <= s; ++sp) x[s][sp] += __shfl_xor_sync(0xffffffffu, x[s][sp], off);
        }
    }
#pragma unroll
    for (int s = 0; s < kNMax; ++s) {
      if (s < n) {
        float m = -INFINITY;
#pragma unroll
        for (int sp = 0; sp <= s; ++sp) {
          x[s][sp] *= scale_log2;
          m = fmaxf(m, x[s][sp]);
        }
        float l = 0.f, acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
        for (int sp = 0; sp <= s; ++sp) {
          const float pe = ex2_approx(x[s][sp] - m);
          float vf[E];
          unpack(vw[sp], vf);
          l += pe;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(pe, vf[e], acc[e]);
        }
        const float inv = 1.f / l;
        Vec out;
        if constexpr (E == 4) {
          out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
          out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        } else {
          out = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        }
        *reinterpret_cast<Vec *>(o + ((row0 + s) * Hq + h) * D + lane * E) = out;
        if (lane == 0) lse[(b * Hq + h) * N + t * n + s] = (m + __log2f(l)) * kLn2;
      }
    }
  }
}

// The same for n > 8 streams, one row at a time (the scores of a row in
// sequence), which keeps the registers of 16 streams bounded.
template <int D>
__global__ void __launch_bounds__(128)
    transient_own_serial_kernel(const __nv_bfloat16 *__restrict__ q,
                                const __nv_bfloat16 *__restrict__ k,
                                const __nv_bfloat16 *__restrict__ v, __nv_bfloat16 *__restrict__ o,
                                float *__restrict__ lse, int64_t B, int64_t L, int n, int Hq,
                                int Hkv, float scale_log2) {
  constexpr int E = D / 32;
  using Vec = typename std::conditional<E == 4, uint2, uint32_t>::type;
  const int64_t wid = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= B * L * Hkv) return;
  const int g = (int)(wid % Hkv);
  const int64_t t = (wid / Hkv) % L, b = wid / Hkv / L;
  const int64_t N = (int64_t)n * L;
  const int64_t row0 = b * N + t * n;
  auto unpack = [](Vec w, float *f) {
    if constexpr (E == 4) {
      f[0] = __uint_as_float(w.x << 16);
      f[1] = __uint_as_float(w.x & 0xffff0000u);
      f[2] = __uint_as_float(w.y << 16);
      f[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
      f[0] = __uint_as_float(w << 16);
      f[1] = __uint_as_float(w & 0xffff0000u);
    }
  };
  Vec kw[kMaxStreams], vw[kMaxStreams];
#pragma unroll
  for (int sp = 0; sp < kMaxStreams; ++sp) {
    if (sp < n) {
      const int64_t off = ((row0 + sp) * Hkv + g) * D + lane * E;
      kw[sp] = *reinterpret_cast<const Vec *>(k + off);
      vw[sp] = *reinterpret_cast<const Vec *>(v + off);
    }
  }
  const int G = Hq / Hkv;
  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    for (int s = 0; s < n; ++s) {
      const int64_t qoff = ((row0 + s) * Hq + h) * D + lane * E;
      float qf[E];
      unpack(*reinterpret_cast<const Vec *>(q + qoff), qf);
      float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
      for (int sp = 0; sp < kMaxStreams; ++sp) {
        if (sp <= s) {  // online softmax over the row's keys
          float kf[E], vf[E];
          unpack(kw[sp], kf);
          unpack(vw[sp], vf);
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) d = fmaf(qf[e], kf[e], d);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
          const float xs = d * scale_log2;
          const float m_new = fmaxf(m, xs);
          const float a = ex2_approx(m - m_new), pe = ex2_approx(xs - m_new);
          l = l * a + pe;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(pe, vf[e], acc[e] * a);
          m = m_new;
        }
      }
      const float inv = 1.f / l;
      Vec out;
      if constexpr (E == 4) {
        out.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        out.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      } else {
        out = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      }
      *reinterpret_cast<Vec *>(o + qoff) = out;
      if (lane == 0) lse[(b * Hq + h) * N + t * n + s] = (m + __log2f(l)) * kLn2;
    }
  }
}

template <int D>
cudaError_t launch_transient_own_d(const PrefillParams &p, __nv_bfloat16 *o, unsigned blocks,
                                   cudaStream_t stream) {
  const float sl2 = p.scale_log2;
  if (p.n <= 4)
    transient_own_kernel<D, 4><<<blocks, 128, 0, stream>>>(p.q, p.k, p.v, o, p.lse, p.B, p.L, p.n,
                                                          p.Hq, p.Hkv, sl2);
  else if (p.n <= 8)
    transient_own_kernel<D, 8><<<blocks, 128, 0, stream>>>(p.q, p.k, p.v, o, p.lse, p.B, p.L, p.n,
                                                          p.Hq, p.Hkv, sl2);
  else
    transient_own_serial_kernel<D><<<blocks, 128, 0, stream>>>(p.q, p.k, p.v, o, p.lse, p.B, p.L,
                                                               p.n, p.Hq, p.Hkv, sl2);
  return cudaGetLastError();
}

cudaError_t launch_transient_own(const PrefillParams &p, __nv_bfloat16 *o, int D,
                                 cudaStream_t stream) {
  const int64_t warps = p.B * p.L * p.Hkv;
  const int64_t blocks = (warps + 3) / 4;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  return D == 128 ? launch_transient_own_d<128>(p, o, (unsigned)blocks, stream)
                  : launch_transient_own_d<64>(p, o, (unsigned)blocks, stream);
}

}  // namespace hd
