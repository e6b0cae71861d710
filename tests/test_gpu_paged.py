"""GPU parity of the paged, variable-length decode against the fp64 oracle.

Each test builds ordinary per-sequence caches, scatters their rows into a
shuffled pool of pages (every row not owned by a sequence's valid range is
NaN), and checks the paged decode against the oracle's decode over the
logical caches with per-sequence token counts."""
import math

import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import binding
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_attention, assert_close_lse

pytestmark = pytest.mark.gpu
DEV = "cuda"


def paginate(kc, vc, Tb, n, page_rows, seed, spare_pages=3):
    """Scatter logical caches [B, rows, Hkv, D] into a shuffled page pool.

    Returns (k_pages, v_pages, page_table int32 [B, max_pages]); rows past a
    sequence's n*T_b and spare pages are NaN."""
    B, rows, Hkv, D = kc.shape
    need = [math.ceil(n * t / page_rows) for t in Tb]
    max_pages = math.ceil(rows / page_rows)
    P = sum(need) + spare_pages
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(P, generator=g).tolist()
    kp = torch.full((P, page_rows, Hkv, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    vp = torch.full_like(kp, float("nan"))
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    i = 0
    for b in range(B):
        valid = n * Tb[b]
        for blk in range(need[b]):
            pg = perm[i]
            i += 1
            table[b, blk] = pg
            lo, hi = blk * page_rows, min((blk + 1) * page_rows, valid)
            kp[pg, : hi - lo] = kc[b, lo:hi]
            vp[pg, : hi - lo] = vc[b, lo:hi]
    return kp, vp, table.to(DEV)


def _oracle(q, kc, vc, Tb, mode, window):
    return oracle.sfa_decode(q.cpu(), kc.cpu(), vc.cpu(), Tb, mode, window=window)


def _run(q, kp, vp, table, Tb, T_bound, mode, window=0):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    seq = torch.tensor(Tb, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_decode_paged_fwd(q, kp, vp, table, seq, T_bound, mode, window=window,
                                     return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    return o, lse, int(status.item())


@pytest.mark.parametrize("mode,window", [("within", 0), ("cross", 0), ("cross_window", 50),
                                         ("cross_window", 1)])
@pytest.mark.parametrize("page_rows", [64, 256])
def test_paged_variable_lengths(mode, window, page_rows):
    B, n, T_bound, Hq, Hkv, D = 4, 4, 300, 32, 8, 128
    Tb = [300, 1, 157, 64]
    seed = 70 + page_rows + window
    q = wl.normal_bf16((B, n, Hq, D), seed, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_bound, Hkv, D), seed, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_bound, Hkv, D), seed, 2, device=DEV)
    kp, vp, table = paginate(kc, vc, Tb, n, page_rows, seed)
    o, lse, st = _run(q, kp, vp, table, Tb, T_bound, mode, window)
    assert st == 0
    ref, ref_lse = _oracle(q, kc, vc, Tb, mode, window)
    assert_close_attention(o, ref, f"paged {mode} W={window} rows={page_rows}")
    assert_close_lse(lse, ref_lse, f"paged {mode}")


@pytest.mark.parametrize("mode", ["within", "cross"])
def test_contiguous_variable_lengths_without_page_table(mode):
    # page_table None: page b is sequence b, rows past n*T_b are NaN
    B, n, T_bound, Hq, Hkv, D = 3, 3, 77, 6, 2, 64
    Tb = [77, 5, 40]
    q = wl.normal_bf16((B, n, Hq, D), 4, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_bound, Hkv, D), 4, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_bound, Hkv, D), 4, 2, device=DEV)
    kpool, vpool = kc.clone(), vc.clone()
    for b, t in enumerate(Tb):
        kpool[b, n * t:] = float("nan")
        vpool[b, n * t:] = float("nan")
    o, lse, st = _run(q, kpool, vpool, None, Tb, T_bound, mode)
    assert st == 0
    ref, ref_lse = _oracle(q, kc, vc, Tb, mode, 0)
    assert_close_attention(o, ref, f"contiguous varlen {mode}")
    assert_close_lse(lse, ref_lse, f"contiguous varlen {mode}")


def test_bad_lengths_and_pages_are_reported_not_fatal():
    B, n, T_bound, Hq, Hkv, D = 3, 4, 100, 8, 2, 128
    q = wl.normal_bf16((B, n, Hq, D), 6, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_bound, Hkv, D), 6, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_bound, Hkv, D), 6, 2, device=DEV)
    Tb = [100, 50, 20]
    kp, vp, table = paginate(kc, vc, Tb, n, 64, 6)
    # a length out of range: that sequence gives zeros, the others stay right
    o, _, st = _run(q, kp, vp, table, [100, 0, 20], T_bound, "cross")
    assert st & binding.HD_DEV_BAD_LENGTH
    assert torch.equal(o[1].float(), torch.zeros_like(o[1].float()))
    ref, _ = _oracle(q[[0, 2]], kc[[0, 2]], vc[[0, 2]], [100, 20], "cross", 0)
    assert_close_attention(o[[0, 2]], ref, "good sequences beside a bad length")
    # a page id out of range reads as zeros and is reported
    bad = table.clone()
    bad[2, 0] = 10_000
    _, _, st = _run(q, kp, vp, bad, Tb, T_bound, "cross")
    assert st & binding.HD_DEV_PAGE_RANGE


def test_decode_workload_paged_full_oracle():
    """Decode workload shapes (batch 64, n = 4, up to 8192 tokens, 32/8 heads) with
    lengths spread over 1 .. 8192 and 256-row pages; every sequence checked."""
    w = wl.WORKLOADS["decode"]
    B, n, T_bound = w.B, w.n, w.L
    g = torch.Generator().manual_seed(w.seed)
    Tb = torch.randint(1, T_bound + 1, (B,), generator=g).tolist()
    Tb[0], Tb[-1] = T_bound, 1
    q, kc, vc = wl.make_decode(w, device=DEV)
    kp, vp, table = paginate(kc, vc, Tb, n, 256, w.seed)
    del kc, vc
    for mode in ("within", "cross"):
        o, lse, st = _run(q, kp, vp, table, Tb, T_bound, mode)
        assert st == 0
        for b in range(B):
            rows = n * Tb[b]
            kb = torch.cat([kp[table[b, i]] for i in range(math.ceil(rows / 256))])[:rows]
            vb = torch.cat([vp[table[b, i]] for i in range(math.ceil(rows / 256))])[:rows]
            ref, ref_lse = oracle.sfa_decode(q[b:b + 1].cpu(), kb[None].cpu(), vb[None].cpu(),
                                             Tb[b], mode)
            assert_close_attention(o[b:b + 1], ref, f"paged workload b={b} {mode}")
            assert_close_lse(lse[b:b + 1], ref_lse, f"paged workload b={b} {mode}")
