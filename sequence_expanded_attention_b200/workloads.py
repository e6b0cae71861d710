"""Seeded synthetic workloads for the Hidden Decoding hot path.

This module holds the five workload shapes and the seeded input generators
that both the CUDA library's tests/benchmark and the fp64 oracle consume.  It
contains none of the method's arithmetic (no gather, no attention): only
shapes, random draws and unit accounting.

Shapes follow the pages' workloads: a Qwen3-8B backbone (the released
Hidden-Decoding-8B-n2/n4/n8 checkpoints, Tencent/Sequential-Hidden-Decoding
README "Released Demonstration Models") with 32 query / 8 KV heads of width
128 and a 151936-token vocabulary of width 4096; expansion factors n in
{2, 4, 8} (review "Method": progressive 1 -> 2 -> 4 -> 8); a MoE-shaped long
prefill; and a small-batch decode over the retained expanded KV cache (review
"Limitations": serving cost is the retained per-stream KV).

Value distributions: Q/K/V ~ N(0, 1), embedding tables ~ N(0, 0.02), token
ids uniform or Zipf(1.1) over the vocabulary (rank k -> id k-1), and for the
MoE-shaped case 1% of key rows scaled by 8 (exact in bf16).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

# Stream ids: each tensor of a workload draws from its own seeded sub-stream.
S_Q, S_K, S_V, S_IDS, S_TABLES, S_OUTLIER, S_DECODE_Q, S_CACHE_K, S_CACHE_V, S_DOUT = range(10)

_CHUNK = 1 << 26  # elements per draw when filling large tensors


def _seed(seed: int, stream: int) -> int:
    return (int(seed) * 1_000_003 + int(stream) * 7919 + 12345) & 0x7FFF_FFFF_FFFF_FFFF


def normal_bf16(shape, seed: int, stream: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    """bf16 tensor of N(0, std^2) draws (fp32 draw, round-to-nearest-even to bf16)."""
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, stream))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    for lo in range(0, flat.numel(), _CHUNK):
        hi = min(lo + _CHUNK, flat.numel())
        x = torch.randn(hi - lo, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        flat[lo:hi].copy_(x)
    return out


def uniform_ids(B: int, L: int, V: int, seed: int, stream: int = S_IDS) -> torch.Tensor:
    """int64 [B, L] ids uniform over [0, V)."""
    rng = np.random.Generator(np.random.PCG64(_seed(seed, stream)))
    return torch.from_numpy(rng.integers(0, V, size=(B, L), dtype=np.int64))


def zipf_ids(B: int, L: int, V: int, a: float, seed: int, stream: int = S_IDS) -> torch.Tensor:
    """int64 [B, L] ids with P(rank k) proportional to k^-a over ranks 1..V, id = k-1.

    Drawn by inverse CDF in fp64 from seeded uniforms.
    """
    rng = np.random.Generator(np.random.PCG64(_seed(seed, stream)))
    w = np.arange(1, V + 1, dtype=np.float64) ** (-a)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(size=(B, L))
    ids = np.searchsorted(cdf, u, side="right")
    return torch.from_numpy(np.minimum(ids, V - 1).astype(np.int64))


def outlier_rows_(k: torch.Tensor, frac: float, factor: float, seed: int,
                  stream: int = S_OUTLIER) -> torch.Tensor:
    """Scale an independent Bernoulli(frac) subset of key rows k[b, p, g, :] by factor, in place.

    Returns the bool mask [B, N, Hkv] of scaled rows.
    """
    g = torch.Generator(device=k.device)
    g.manual_seed(_seed(seed, stream))
    mask = torch.rand(k.shape[:3], generator=g, device=k.device) < frac
    k[mask] = (k[mask].float() * factor).to(k.dtype)
    return mask


@dataclasses.dataclass(frozen=True)
class Workload:
    """One seeded workload: SFA prefill shapes, the embedding expansion and/or a decode step."""

    name: str
    index: int               # 1-based position in the workload list; seed = 1000 + index
    n: int                   # streams per token
    L: int                   # tokens per sequence (prefill) / tokens in cache (decode: T)
    B: int
    Hq: int
    Hkv: int
    D: int
    modes: tuple = ("within", "cross")
    vocab: int = 0           # embedding expansion: vocabulary (0 = no embedding step)
    d_model: int = 0
    table_std: float = 0.02
    ids: str = "uniform"     # "uniform" | "zipf"
    zipf_a: float = 1.1
    outlier_frac: float = 0.0
    outlier_factor: float = 8.0
    schedule: tuple = ()     # per-layer modes for a layer-schedule measurement
    decode: bool = False     # True: a decode step over a cache of L tokens
    window: int = 0          # sliding window (tokens) of "cross_window" layers
    page_rows: int = 0       # decode over a paged cache with variable lengths (0: contiguous)
    backward: bool = False   # each prefill layer also runs its backward (training step)
    prefix: int = 0          # chunked prefill: L new tokens after a cached prefix of this many

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def N(self) -> int:
        return self.n * self.L


WORKLOADS = {
    "tiny": Workload("tiny", 1, n=2, L=64, B=1, Hq=2, Hkv=2, D=64, vocab=1000, d_model=128,
                     ids="uniform"),
    "qwen3_8b_prefill": Workload("qwen3_8b_prefill", 2, n=4, L=2048, B=4, Hq=32, Hkv=8, D=128,
                                 vocab=151936, d_model=4096, ids="zipf"),
    "large_expansion": Workload("large_expansion", 3, n=8, L=4096, B=1, Hq=32, Hkv=8, D=128,
                                schedule=("within",) * 3 + ("cross",) + ("within",) * 3
                                + ("cross",)),
    "moe_long_prefill": Workload("moe_long_prefill", 4, n=4, L=8192, B=2, Hq=64, Hkv=4, D=128,
                                 outlier_frac=0.01),
    "decode": Workload("decode", 5, n=4, L=8192, B=64, Hq=32, Hkv=8, D=128, decode=True),
    # Cross-stream layers of a sliding-window base layer (review "Method": 23 of
    # the 80B model's 49 layers); the pages give no window size, 512 tokens here.
    # Serving-style decode: lengths uniform over 1 .. 8192 tokens, 256-row pages
    # (64 tokens x 4 streams) in a shuffled pool.
    "decode_paged": Workload("decode_paged", 7, n=4, L=8192, B=64, Hq=32, Hkv=8, D=128,
                             decode=True, page_rows=256),
    # Training-side ends of the Qwen3-8B-shaped path: the final-stream rows that
    # feed the loss, and the expansion's gradient into the 4 tables.
    "qwen3_8b_embed_train": Workload("qwen3_8b_embed_train", 8, n=4, L=2048, B=4, Hq=32,
                                     Hkv=8, D=128, modes=(), vocab=151936, d_model=4096,
                                     ids="zipf"),
    # The PHD-style control of the shared-KV ablation (intermediate streams
    # transient) on the Qwen3-8B shapes.
    "qwen3_8b_transient": Workload("qwen3_8b_transient", 9, n=4, L=2048, B=4, Hq=32, Hkv=8,
                                   D=128, modes=("transient",)),
    "qwen3_8b_window": Workload("qwen3_8b_window", 6, n=4, L=2048, B=4, Hq=32, Hkv=8, D=128,
                                modes=("cross_window",), window=512),
    # Training through the SFA layers of the Qwen3-8B-shaped path: a within-stream
    # and a cross-stream layer, each forward (with LSE) then backward.
    "qwen3_8b_train_sfa": Workload("qwen3_8b_train_sfa", 10, n=4, L=2048, B=4, Hq=32, Hkv=8,
                                   D=128, backward=True),
    # Serving: a 512-token chunk after a 1536-token cached prefix at the Qwen3-8B
    # shapes, K/V in a shuffled pool of 256-row pages.
    "qwen3_8b_chunk_paged": Workload("qwen3_8b_chunk_paged", 11, n=4, L=512, B=4, Hq=32, Hkv=8,
                                     D=128, prefix=1536, page_rows=256),
}


def make_qkv(w: Workload, device="cpu", B=None, L=None):
    """Seeded q [B, nL, Hq, D], k, v [B, nL, Hkv, D] bf16 for a prefill workload.

    B and L may be overridden for reduced parity cases of the same structure.
    """
    B = w.B if B is None else B
    L = w.L if L is None else L
    N = w.n * L
    q = normal_bf16((B, N, w.Hq, w.D), w.seed, S_Q, device=device)
    k = normal_bf16((B, N, w.Hkv, w.D), w.seed, S_K, device=device)
    v = normal_bf16((B, N, w.Hkv, w.D), w.seed, S_V, device=device)
    if w.outlier_frac > 0:
        outlier_rows_(k, w.outlier_frac, w.outlier_factor, w.seed)
    return q, k, v


def make_embedding(w: Workload, device="cpu", B=None, L=None):
    """Seeded (ids int64 [B, L] on `device`, list of n bf16 tables [V, d])."""
    B = w.B if B is None else B
    L = w.L if L is None else L
    if w.ids == "zipf":
        ids = zipf_ids(B, L, w.vocab, w.zipf_a, w.seed)
    else:
        ids = uniform_ids(B, L, w.vocab, w.seed)
    tables = [normal_bf16((w.vocab, w.d_model), w.seed, S_TABLES * 64 + s, std=w.table_std,
                          device=device) for s in range(w.n)]
    return ids.to(device), tables


def make_decode(w: Workload, device="cpu", B=None, T=None, T_max=None):
    """Seeded decode inputs: q [B, n, Hq, D], k/v cache [B, n*T_max, Hkv, D].

    The first n*T cache rows are valid; rows beyond are filled too (with the
    same distribution) so that reading past the valid prefix would show.
    """
    B = w.B if B is None else B
    T = w.L if T is None else T
    T_max = T if T_max is None else T_max
    q = normal_bf16((B, w.n, w.Hq, w.D), w.seed, S_DECODE_Q, device=device)
    kc = normal_bf16((B, w.n * T_max, w.Hkv, w.D), w.seed, S_CACHE_K, device=device)
    vc = normal_bf16((B, w.n * T_max, w.Hkv, w.D), w.seed, S_CACHE_V, device=device)
    return q, kc, vc


# ---------------------------------------------------------------------------
# Unit accounting (what the benchmark counts; no masked or padded work).

def unmasked_pairs(mode: str, n: int, L: int, window: int = 0) -> int:
    """(query, key) pairs the SFA mask allows in one (batch, head) of a length-nL sequence.

    within-stream: n independent causal problems of length L -> n L (L+1) / 2.
    cross-stream:  one causal problem of length N = nL      -> N (N+1) / 2.
    cross-stream, sliding window of W tokens: query (t, s) sees the n streams of
      tokens max(0, t-W+1) .. t-1 and streams 0..s of token t ->
      n^2 sum_t min(t, W-1) + L n (n+1) / 2.
    plain causal (n = 1) is L (L+1) / 2 either way.
    """
    if mode == "within":
        return n * L * (L + 1) // 2
    if mode == "cross":
        N = n * L
        return N * (N + 1) // 2
    if mode == "cross_window":
        if window < 1:
            raise ValueError("window must be >= 1")
        W = window
        if L <= W:
            full = L * (L - 1) // 2
        else:
            full = (W - 1) * W // 2 + (L - W) * (W - 1)
        return n * n * full + L * n * (n + 1) // 2
    if mode == "transient":
        # query (t, s): the final streams of tokens 0..t-1 plus streams 0..s of token t
        return n * L * (L - 1) // 2 + L * n * (n + 1) // 2
    raise ValueError(mode)


def chunk_pairs(mode: str, n: int, P: int, C: int) -> int:
    """(query, key) pairs the mask allows for the C chunk tokens after a prefix of
    P tokens, in one (batch, head): the rows of tokens P .. P+C-1 of a prefill
    over P + C tokens.
    within-stream: n * sum_{t=P}^{P+C-1} (t + 1).
    cross-stream:  sum over positions p = nP .. n(P+C)-1 of (p + 1)."""
    if mode == "within":
        return n * (C * P + C * (C + 1) // 2)
    if mode == "cross":
        n1, n2 = n * P, n * (P + C)
        return n2 * (n2 + 1) // 2 - n1 * (n1 + 1) // 2
    raise ValueError(mode)


def make_chunk_paged(w: Workload, device="cpu"):
    """Seeded chunked-prefill inputs over a page pool: (q [B, n*L, Hq, D],
    k_pages, v_pages [pages, page_rows, Hkv, D], page_table int32 [B, max_pages],
    prefix int32 [B]).  Every sequence holds w.prefix + w.L tokens; its pages are
    drawn from a seeded shuffle of the pool."""
    g = torch.Generator().manual_seed(_seed(w.seed, S_IDS))
    tokens = w.prefix + w.L
    per_seq = (w.n * tokens + w.page_rows - 1) // w.page_rows
    P = per_seq * w.B
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = perm.reshape(w.B, per_seq).contiguous()
    q = normal_bf16((w.B, w.n * w.L, w.Hq, w.D), w.seed, S_Q, device=device)
    kp = normal_bf16((P, w.page_rows, w.Hkv, w.D), w.seed, S_CACHE_K, device=device)
    vp = normal_bf16((P, w.page_rows, w.Hkv, w.D), w.seed, S_CACHE_V, device=device)
    prefix = torch.full((w.B,), w.prefix, dtype=torch.int32)
    return q, kp, vp, table.to(device), prefix.to(device)


def prefill_flops(mode: str, n: int, L: int, B: int, Hq: int, D: int, window: int = 0) -> int:
    """Unmasked FLOPs of one SFA prefill: 2*D for QK^T plus 2*D for PV per allowed pair."""
    return 4 * D * B * Hq * unmasked_pairs(mode, n, L, window)


def decode_pairs(mode: str, n: int, T: int, window: int = 0) -> int:
    """Allowed pairs of the n new positions of token T (p = n(T-1)+s) over n*T cache rows."""
    if mode == "within":
        return n * T
    if mode == "cross":
        return sum(n * (T - 1) + s + 1 for s in range(n))
    if mode == "cross_window":
        return sum(n * min(T - 1, window - 1) + s + 1 for s in range(n))
    if mode == "transient":
        return sum((T - 1) + s + 1 for s in range(n))
    raise ValueError(mode)


def decode_flops(mode: str, n: int, T: int, B: int, Hq: int, D: int, window: int = 0) -> int:
    return 4 * D * B * Hq * decode_pairs(mode, n, T, window)


def decode_bytes(n: int, T: int, B: int, Hq: int, Hkv: int, D: int) -> int:
    """Algorithmic HBM bytes of one decode call: the n*T valid K and V cache rows once,
    plus q in and o out (bf16).  Both modes read the same rows (within-stream reads
    each row for exactly one of the n queries of its stream)."""
    return 2 * (2 * B * n * T * Hkv * D) + 2 * (2 * B * n * Hq * D)


def gather_bytes(n: int, B: int, L: int, d: int) -> int:
    """Algorithmic HBM bytes of one expansion: each of the B*L*n rows read once and
    written once (bf16), plus the int64 ids."""
    return 2 * (2 * B * L * n * d) + 8 * B * L


def make_paged_decode(w: Workload, device="cpu"):
    """Seeded paged decode inputs: (q [B, n, Hq, D], k_pages, v_pages
    [P, page_rows, Hkv, D], page_table int32 [B, max_pages], seq_tokens int32 [B]).

    Lengths are uniform over 1 .. L tokens; each sequence's row blocks sit in
    pages drawn from a seeded shuffle of the pool."""
    g = torch.Generator().manual_seed(_seed(w.seed, S_IDS))
    Tb = torch.randint(1, w.L + 1, (w.B,), generator=g)
    need = (w.n * Tb + w.page_rows - 1) // w.page_rows
    P = int(need.sum())
    max_pages = (w.n * w.L + w.page_rows - 1) // w.page_rows
    perm = torch.randperm(P, generator=g)
    table = torch.full((w.B, max_pages), -1, dtype=torch.int32)
    start = 0
    for b in range(w.B):
        k = int(need[b])
        table[b, :k] = perm[start:start + k].to(torch.int32)
        start += k
    q = normal_bf16((w.B, w.n, w.Hq, w.D), w.seed, S_DECODE_Q, device=device)
    kp = normal_bf16((P, w.page_rows, w.Hkv, w.D), w.seed, S_CACHE_K, device=device)
    vp = normal_bf16((P, w.page_rows, w.Hkv, w.D), w.seed, S_CACHE_V, device=device)
    return q, kp, vp, table.to(device), Tb.to(torch.int32).to(device)

