"""GPU parity of chunked prefill (a chunk of C new tokens after a cached
prefix of P tokens) against the fp64 oracle, plus its two limits: P = 0 is
the plain prefill, bit for bit, and C = 1 is a decode step."""
import numpy as np
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_attention, assert_close_lse

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cache(B, n, T_max, Hkv, D, seed, filled):
    """K/V caches whose rows past `filled` tokens are NaN: reading one shows."""
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 2, device=DEV)
    kc[:, n * filled:] = float("nan")
    vc[:, n * filled:] = float("nan")
    return kc, vc


def _chunk(q, kc, vc, P, n, mode, W=0):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_chunk_fwd(q, kc, vc, P, n, mode, window=W, return_lse=True,
                                      dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


def _oracle_chunk(q, kc, vc, P, n, mode, W=0):
    """Every row of the chunk through the oracle: query i of the chunk is
    expanded position n*P + i among n*(P+C) valid keys."""
    B, NC, Hq, D = q.shape
    b, i, h = np.meshgrid(np.arange(B), np.arange(NC), np.arange(Hq), indexing="ij")
    rb, ri, rh = b.ravel(), i.ravel(), h.ravel()
    rp = n * P + ri
    q_rows = q.cpu()[torch.as_tensor(rb), torch.as_tensor(ri), torch.as_tensor(rh)]
    nk = n * P + NC
    o, lse = oracle.attend_rows(q_rows, rb, rp, rh, kc.cpu(), vc.cpu(), nk, n, Hq, mode,
                                window=W)
    return o.reshape(B, NC, Hq, D), lse.reshape(B, NC, Hq).permute(0, 2, 1)


@pytest.mark.parametrize("mode,B,n,P,C,T_max,Hq,Hkv,D,W", [
    ("cross", 2, 4, 200, 100, 320, 8, 2, 128, 0),     # ragged prefix and chunk
    ("cross", 1, 4, 64, 64, 128, 32, 8, 128, 0),      # prefix = one full KV tile of positions
    ("cross", 1, 3, 37, 250, 300, 4, 2, 64, 0),       # odd n, chunk over several q tiles
    ("within", 2, 4, 200, 100, 320, 8, 2, 128, 0),
    ("within", 1, 2, 300, 40, 350, 4, 1, 64, 0),       # short chunk after a long prefix
    ("cross_window", 1, 4, 300, 90, 400, 8, 2, 128, 50),
    ("cross_window", 2, 2, 100, 70, 200, 4, 4, 128, 1),
    ("cross", 1, 1, 500, 300, 900, 2, 2, 128, 0),     # n = 1: plain chunked causal prefill
])
def test_chunk_matches_oracle(mode, B, n, P, C, T_max, Hq, Hkv, D, W):
    seed = 4100 + P + C + n
    q = wl.normal_bf16((B, n * C, Hq, D), seed, 0, device=DEV)
    kc, vc = _cache(B, n, T_max, Hkv, D, seed, P + C)
    o, lse = _chunk(q, kc, vc, P, n, mode, W)
    ref, ref_lse = _oracle_chunk(q, kc, vc, P, n, mode, W)
    what = f"chunk {mode} n={n} P={P} C={C}"
    assert_close_attention(o, ref, what)
    assert_close_lse(lse, ref_lse, what)


@pytest.mark.parametrize("mode", ["within", "cross", "cross_window"])
def test_chunk_without_prefix_is_the_plain_prefill(mode):
    B, n, L, Hq, Hkv, D, W = 2, 4, 190, 8, 2, 128, 33
    q = wl.normal_bf16((B, n * L, Hq, D), 71, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), 71, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), 71, 2, device=DEV)
    o_c, lse_c = _chunk(q, k, v, 0, n, mode, W)
    if mode == "cross_window":
        o_p, lse_p = hd.sfa_prefill_window_fwd(q, k, v, n, W, return_lse=True)
    else:
        o_p, lse_p = hd.sfa_prefill_fwd(q, k, v, n, mode, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o_c, o_p) and torch.equal(lse_c, lse_p)


def test_successive_chunks_rebuild_the_full_prefill():
    """Prefill in three chunks of an n=4 sequence equals one prefill over it."""
    B, n, L, Hq, Hkv, D = 1, 4, 400, 8, 2, 128
    q = wl.normal_bf16((B, n * L, Hq, D), 72, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), 72, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), 72, 2, device=DEV)
    full = hd.sfa_prefill_fwd(q, k, v, n, "cross")
    kc = torch.full_like(k, float("nan"))
    vc = torch.full_like(v, float("nan"))
    parts = []
    for t0, t1 in ((0, 150), (150, 151), (151, 400)):
        kc[:, n * t0:n * t1] = k[:, n * t0:n * t1]   # append the chunk, then attend
        vc[:, n * t0:n * t1] = v[:, n * t0:n * t1]
        parts.append(_chunk(q[:, n * t0:n * t1].contiguous(), kc, vc, t0, n, "cross")[0])
    assert_close_attention(torch.cat(parts, 1), full.double(), "three chunks vs one prefill")
    ref, _ = oracle.sfa_prefill(q.cpu(), k.cpu(), v.cpu(), n, "cross")
    assert_close_attention(torch.cat(parts, 1), ref, "three chunks vs oracle")


@pytest.mark.parametrize("mode", ["within", "cross"])
def test_one_token_chunk_is_a_decode_step(mode):
    B, n, T, T_max, Hq, Hkv, D = 2, 4, 333, 340, 32, 8, 128
    q = wl.normal_bf16((B, n, Hq, D), 73, 0, device=DEV)
    kc, vc = _cache(B, n, T_max, Hkv, D, 73, T)
    o_c, lse_c = _chunk(q, kc, vc, T - 1, n, mode)
    o_d, lse_d = hd.sfa_decode_fwd(q, kc, vc, T, mode, return_lse=True)
    torch.cuda.synchronize()
    assert_close_attention(o_c, o_d.double(), f"C=1 chunk vs decode ({mode})")
    assert_close_lse(lse_c, lse_d, f"C=1 chunk vs decode ({mode})")


@pytest.mark.parametrize("mode", ["within", "cross"])
def test_chunk_qwen3_shapes_full_oracle(mode):
    """A 512-token chunk after a 1536-token prefix at the Qwen3-8B shapes (n=4,
    B=4, 32/8 heads, D=128): every output row and log-sum-exp against the
    oracle, one sequence at a time."""
    B, n, P, C, Hq, Hkv, D = 4, 4, 1536, 512, 32, 8, 128
    q = wl.normal_bf16((B, n * C, Hq, D), 74, 0, device=DEV)
    kc, vc = _cache(B, n, P + C, Hkv, D, 74, P + C)
    o, lse = _chunk(q, kc, vc, P, n, mode)
    for b in range(B):
        sl = slice(b, b + 1)
        ref, ref_lse = _oracle_chunk(q[sl], kc[sl], vc[sl], P, n, mode)
        assert_close_attention(o[sl], ref, f"qwen3 chunk {mode} b={b}")
        assert_close_lse(lse[sl], ref_lse, f"qwen3 chunk {mode} b={b}")


def test_chunk_argument_checks():
    q = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(1, 16, 2, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_chunk_fwd(q, kc, kc, 5, 2, "cross")          # P + C > T_max
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_chunk_fwd(q, kc, kc, 0, 2, "transient")
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_chunk_fwd(q, kc, kc, 0, 2, "cross_window", window=0)
    o = hd.sfa_prefill_chunk_fwd(q[:, :0], kc, kc, 4, 2, "cross")  # empty chunk
    assert o.shape[1] == 0


# ------------------------------------------------------------ paged pool

def _pool(kc, vc, n, tokens, page_rows, seed, spare=3):
    """Page pool of the first n*tokens[b] rows of each sequence of kc / vc, pages
    in a seeded shuffled order; every other pool row (and every unused table
    entry's target) holds NaN."""
    B, _, Hkv, D = kc.shape
    pages_b = [(n * t + page_rows - 1) // page_rows for t in tokens]
    num_pages = sum(pages_b) + spare
    max_pages = max(pages_b) + 1
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g).tolist()
    kp = torch.full((num_pages, page_rows, Hkv, D), float("nan"), dtype=kc.dtype, device=DEV)
    vp = torch.full_like(kp, float("nan"))
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        rows = n * tokens[b]
        for i in range(pages_b[b]):
            pid = perm[nxt]
            nxt += 1
            table[b, i] = pid
            r0, r1 = i * page_rows, min(rows, (i + 1) * page_rows)
            kp[pid, :r1 - r0] = kc[b, r0:r1]
            vp[pid, :r1 - r0] = vc[b, r0:r1]
    return kp, vp, table.to(DEV)


@pytest.mark.parametrize("mode,n,C,prefixes,page_rows,Hq,Hkv,D,W", [
    ("cross", 4, 100, (0, 130, 257), 256, 8, 2, 128, 0),
    ("within", 4, 100, (0, 130, 257), 256, 8, 2, 128, 0),     # 64 tokens per page
    ("within", 2, 150, (5, 300), 512, 4, 1, 128, 0),          # 256 tokens per page
    ("within", 2, 70, (64, 9), 128, 4, 2, 64, 0),             # D = 64
    ("cross_window", 4, 90, (40, 200), 384, 8, 2, 128, 33),
])
def test_paged_chunk_equals_contiguous_chunk(mode, n, C, prefixes, page_rows, Hq, Hkv, D, W):
    """Each sequence's rows, bit for bit, as the contiguous chunked prefill of
    that sequence alone (same tiles, same arithmetic), with stale NaN rows in
    the pages and shuffled page order."""
    B = len(prefixes)
    T_max = max(prefixes) + C + 8
    seed = 5100 + C + page_rows
    q = wl.normal_bf16((B, n * C, Hq, D), seed, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 2, device=DEV)
    kp, vp, table = _pool(kc, vc, n, [P + C for P in prefixes], page_rows, seed)
    pre = torch.tensor(prefixes, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_chunk_paged_fwd(q, kp, vp, table, pre, n, mode, window=W,
                                            return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(o.float()).all()
    for b, P in enumerate(prefixes):
        kb, vb = kc[b:b + 1].clone(), vc[b:b + 1].clone()
        kb[:, n * (P + C):] = float("nan")
        vb[:, n * (P + C):] = float("nan")
        ob, lb = _chunk(q[b:b + 1].contiguous(), kb, vb, P, n, mode, W)
        assert torch.equal(o[b:b + 1], ob), (mode, b)
        assert torch.equal(lse[b:b + 1], lb), (mode, b)


def test_paged_chunk_matches_oracle():
    B, n, C, Hq, Hkv, D, page_rows = 2, 4, 96, 8, 2, 128, 256
    prefixes = (37, 180)
    T_max = max(prefixes) + C
    q = wl.normal_bf16((B, n * C, Hq, D), 5200, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), 5200, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), 5200, 2, device=DEV)
    kp, vp, table = _pool(kc, vc, n, [P + C for P in prefixes], page_rows, 5200)
    pre = torch.tensor(prefixes, dtype=torch.int32, device=DEV)
    for mode in ("within", "cross"):
        o, lse = hd.sfa_prefill_chunk_paged_fwd(q, kp, vp, table, pre, n, mode, return_lse=True)
        torch.cuda.synchronize()
        for b, P in enumerate(prefixes):
            ref, ref_lse = _oracle_chunk(q[b:b + 1], kc[b:b + 1], vc[b:b + 1], P, n, mode)
            assert_close_attention(o[b:b + 1], ref, f"paged {mode} b={b}")
            assert_close_lse(lse[b:b + 1], ref_lse, f"paged {mode} b={b}")


@pytest.mark.parametrize("mode,n,C,prefixes,chunks,page_rows", [
    ("cross", 4, 200, (0, 130, 257, 40), (200, 37, 129, 0), 256),
    ("within", 4, 200, (0, 130, 257, 40), (200, 37, 129, 0), 256),
    ("within", 2, 300, (5, 300, 17), (1, 300, 128), 512),
])
def test_paged_chunk_variable_lengths(mode, n, C, prefixes, chunks, page_rows):
    """A batch of chunks of different lengths padded to C: each sequence's first
    chunk_tokens[b] tokens, bit for bit, as the contiguous chunked prefill of
    that sequence's own chunk alone; the padding rows of q are NaN."""
    B, Hq, Hkv, D = len(prefixes), 8, 2, 128
    T_max = max(P + c for P, c in zip(prefixes, chunks)) + 8
    seed = 5400 + C + page_rows
    q = wl.normal_bf16((B, n * C, Hq, D), seed, 0, device=DEV)
    for b, c in enumerate(chunks):
        q[b, n * c:] = float("nan")
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 2, device=DEV)
    kp, vp, table = _pool(kc, vc, n, [P + c for P, c in zip(prefixes, chunks)], page_rows, seed)
    pre = torch.tensor(prefixes, dtype=torch.int32, device=DEV)
    ct = torch.tensor(chunks, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_chunk_paged_fwd(q, kp, vp, table, pre, n, mode, return_lse=True,
                                            chunk_tokens=ct, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for b, (P, c) in enumerate(zip(prefixes, chunks)):
        if c == 0:
            continue
        kb, vb = kc[b:b + 1].clone(), vc[b:b + 1].clone()
        kb[:, n * (P + c):] = float("nan")
        vb[:, n * (P + c):] = float("nan")
        ob, lb = _chunk(q[b:b + 1, :n * c].contiguous(), kb, vb, P, n, mode, 0)
        assert torch.isfinite(ob.float()).all()
        assert torch.equal(o[b:b + 1, :n * c], ob), (mode, b)
        assert torch.equal(lse[b:b + 1, :, :n * c], lb), (mode, b)


def test_paged_chunk_variable_length_out_of_range():
    B, n, C, Hq, Hkv, D, page_rows = 2, 4, 64, 4, 2, 128, 256
    q = wl.normal_bf16((B, n * C, Hq, D), 5500, 0, device=DEV)
    kc = wl.normal_bf16((B, n * 200, Hkv, D), 5500, 1, device=DEV)
    vc = wl.normal_bf16((B, n * 200, Hkv, D), 5500, 2, device=DEV)
    kp, vp, table = _pool(kc, vc, n, [100 + C, 10 + C], page_rows, 5500)
    pre = torch.tensor([100, 10], dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ct = torch.tensor([C, C + 1], dtype=torch.int32, device=DEV)
    o = hd.sfa_prefill_chunk_paged_fwd(q, kp, vp, table, pre, n, "cross", chunk_tokens=ct,
                                       dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & hd.binding.HD_DEV_BAD_LENGTH
    assert torch.isfinite(o[0].float()).all()


def test_paged_chunk_status_bits():
    B, n, C, Hq, Hkv, D, page_rows = 2, 4, 64, 4, 2, 128, 256
    q = wl.normal_bf16((B, n * C, Hq, D), 5300, 0, device=DEV)
    kc = wl.normal_bf16((B, n * 300, Hkv, D), 5300, 1, device=DEV)
    vc = wl.normal_bf16((B, n * 300, Hkv, D), 5300, 2, device=DEV)
    kp, vp, table = _pool(kc, vc, n, [100 + C, 10 + C], page_rows, 5300)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    # a prefix larger than the table holds: that sequence is skipped, the bit is set
    too_long = torch.tensor([100, 10_000], dtype=torch.int32, device=DEV)
    hd.sfa_prefill_chunk_paged_fwd(q, kp, vp, table, too_long, n, "cross", dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & hd.binding.HD_DEV_BAD_LENGTH
    # a page id outside the pool within the sequence's rows
    bad = table.clone()
    bad[0, 0] = kp.shape[0] + 5
    status.zero_()
    o = hd.sfa_prefill_chunk_paged_fwd(q, kp, vp, bad, torch.tensor([100, 10], dtype=torch.int32,
                                       device=DEV), n, "within", dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & hd.binding.HD_DEV_PAGE_RANGE
    assert torch.isfinite(o.float()).all()
