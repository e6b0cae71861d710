"""Shared helpers for the GPU parity tests: tolerances and row sampling.

Tolerances are the ones the task states for attention against the fp64
oracle on the same bf16 inputs: max-abs <= 2e-2 and relative-L2 <= 5e-3.
The embedding expansion is compared bit for bit.
"""
import numpy as np
import torch

import oracle

MAX_ABS = 2e-2
REL_L2 = 5e-3
# LSE is fp32 from fp32 logits: absolute error well below the output bound.
LSE_ABS = 2e-3


def assert_close_attention(got: torch.Tensor, ref: torch.Tensor, what: str = ""):
    got = got.double().cpu()
    ref = ref.double().cpu()
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got - ref)
    max_abs = err.abs().max().item()
    rel = (err.norm() / ref.norm().clamp_min(1e-30)).item()
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def assert_close_lse(got: torch.Tensor, ref: torch.Tensor, what: str = ""):
    got = got.double().cpu()
    ref = ref.double().cpu()
    d = (got - ref).abs().max().item()
    assert d <= LSE_ABS, f"{what}: lse max_abs={d:.3e}"


def sample_rows(B: int, seq: int, n: int, Hq: int, within: bool, count: int, seed: int,
                extra_positions=(), every_head: bool = False):
    """Seeded (b, p, h) rows covering every stream, the first/last rows of
    128-row tiles, the last rows of the sequence and random rows.

    With `every_head`, each tile-edge row is taken for every batch and every
    query head, and each extra position for every head of batch 0 (extra
    positions come from batch 0's keys); otherwise each of those rows gets a
    random batch and head.  Random rows fill up to `count`.

    seq is the per-problem sequence length (L within-stream, N cross-stream);
    positions returned are expanded positions p in [0, n*L).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    N = seq * n if within else seq
    L = N // n
    edges = set()
    # tile edges of the problem sequence, mapped to expanded positions
    for t0 in range(0, seq, 128):
        for r in (t0, min(t0 + 127, seq - 1)):
            for s in range(n):
                edges.add((r * n + s) if within else r)
    for p in (0, N - 1, N - 2, n * (L - 1)):
        if 0 <= p < N:
            edges.add(p)
    extras = sorted({int(p) for p in extra_positions if 0 <= p < N} - edges)
    edges = sorted(edges)
    rows = []
    if every_head:
        rows += [(b, p, h) for p in edges for b in range(B) for h in range(Hq)]
        rows += [(0, p, h) for p in extras for h in range(Hq)]
    else:
        for p in edges + extras:
            rows.append((int(rng.integers(0, B)), p, int(rng.integers(0, Hq))))
    while len(rows) < count:
        rows.append((int(rng.integers(0, B)), int(rng.integers(0, N)), int(rng.integers(0, Hq))))
    rb = np.array([r[0] for r in rows], dtype=np.int64)
    rp = np.array([r[1] for r in rows], dtype=np.int64)
    rh = np.array([r[2] for r in rows], dtype=np.int64)
    return rb, rp, rh


# Gradients of attention (SFA backward).  P and dS are rounded to bf16 before
# their tensor-core products (relative 2^-9 each), Delta = <dO, O> uses the
# forward pass's bf16 O, and the outputs are bf16: the error relative to the
# gradient's own scale is a few times 2^-9.  Bound: relative L2 <= 1e-2 and
# max-abs <= 2e-2 of the reference's largest magnitude.
GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2


def assert_close_grad(got: torch.Tensor, ref: torch.Tensor, what: str = ""):
    got = got.double().cpu()
    ref = ref.double().cpu()
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert torch.isfinite(got).all(), f"{what}: non-finite gradient"
    err = got - ref
    scale = ref.abs().max().clamp_min(1e-30).item()
    max_rel = err.abs().max().item() / scale
    rel = (err.norm() / ref.norm().clamp_min(1e-30)).item()
    assert rel <= GRAD_REL_L2 and max_rel <= GRAD_MAX_REL, \
        f"{what}: rel_l2={rel:.3e} max_abs/max|ref|={max_rel:.3e}"
    return rel, max_rel


def check_full_by_batch(o, lse, q, k, v, n, mode, window: int = 0, what: str = ""):
    """Every output row and log-sum-exp of a prefill against the oracle,
    element by element, one batch at a time (bounded host memory)."""
    for b in range(q.shape[0]):
        ref_o, ref_lse = oracle.sfa_prefill(q[b:b + 1].cpu(), k[b:b + 1].cpu(),
                                            v[b:b + 1].cpu(), n, mode, window=window)
        assert_close_attention(o[b:b + 1], ref_o, f"{what} batch {b}")
        assert_close_lse(lse[b:b + 1], ref_lse, f"{what} batch {b}")
        del ref_o, ref_lse
