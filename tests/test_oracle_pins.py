"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test ties the oracle to what the pages and mathematics fix:

* brute-force enumeration of the SFA masks in (token, stream) coordinates
  (review "Method"; README "Key Idea"), observed through the closed form
  O = mean of V over the allowed set when Q = 0;
* library routines: plain causal attention (torch SDPA in fp64) for n = 1,
  for the cross-stream mode (causal over the whole expanded sequence) and for
  each de-interleaved stream of the within-stream mode; F.embedding for the
  per-stream gather;
* invariants: a cross-stream row ignores later positions, constant V gives
  constant O, decode equals the last n prefill rows, and the LSE closed forms.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from sequence_expanded_attention_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, std=1.0):
    return wl.normal_bf16(shape, seed, 0, std=std)


def _sdpa_causal(q, k, v, scale=None):
    """Library causal attention in fp64: q [B, N, Hq, D], k/v [B, N, Hkv, D] -> [B, N, Hq, D].

    GQA by consecutive groups: query head h reads KV head h // (Hq / Hkv).
    """
    Hq, Hkv = q.shape[2], k.shape[2]
    qf = q.double().permute(0, 2, 1, 3)
    kf = k.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    vf = v.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(qf, kf, vf, is_causal=True, scale=scale)
    return o.permute(0, 2, 1, 3)


# ---------------------------------------------------------------- mask pins

def _allowed_bruteforce(n, L, mode, W=None):
    """Allowed (query, key) expanded-position pairs, enumerated from the pages' wording.

    Position p holds token t = p // n of stream s = p % n (token-major layout).
    within-stream: query (t, s) sees key (t', s') iff s' == s and t' <= t.
    cross-stream:  query p sees key p' iff p' <= p (causal over the expanded sequence).
    cross-stream with a sliding window of W tokens: as cross-stream, and the key's
      token is one of the last W tokens: t - W < t' (t' < t, or t' == t and s' <= s).
    """
    allowed = set()
    for t, s, t2, s2 in itertools.product(range(L), range(n), range(L), range(n)):
        p, p2 = t * n + s, t2 * n + s2
        if mode == "within" and s2 == s and t2 <= t:
            allowed.add((p, p2))
        if mode == "cross" and p2 <= p:
            allowed.add((p, p2))
        if mode == "cross_window" and t - W < t2 and (t2 < t or (t2 == t and s2 <= s)):
            allowed.add((p, p2))
        # transient intermediate streams (PHD-style control): earlier tokens only
        # through their final stream, the current token's streams up to s
        if mode == "transient" and ((t2 < t and s2 == n - 1) or (t2 == t and s2 <= s)):
            allowed.add((p, p2))
    return allowed


@pytest.mark.parametrize("mode", ["within", "cross"])
@pytest.mark.parametrize("n,L", [(1, 6), (3, 5), (4, 4)])
def test_mask_by_enumeration(mode, n, L):
    N = n * L
    D = 32
    assert D >= N
    q = torch.zeros(1, N, 1, D, dtype=torch.bfloat16)
    k = _rand((1, N, 1, D), 11)
    v = torch.zeros(1, N, 1, D, dtype=torch.bfloat16)
    v[0, torch.arange(N), 0, torch.arange(N)] = 1.0  # one-hot rows: O reveals the weights
    o, lse = oracle.sfa_prefill(q, k, v, n, mode)
    allowed = _allowed_bruteforce(n, L, mode)
    for p in range(N):
        keys = sorted(p2 for (pp, p2) in allowed if pp == p)
        want = torch.zeros(D, dtype=torch.float64)
        want[keys] = 1.0 / len(keys)
        assert torch.equal(o[0, p, 0], want), (p, keys)
        # Q = 0: all logits are 0, so LSE = log |A(p)|
        assert abs(lse[0, 0, p].item() - np.log(len(keys))) < 1e-14


def test_lse_constant_logits():
    # identical key rows give every allowed key the same logit c, so LSE = c + log|A(p)|
    n, L, D = 2, 5, 16
    N = n * L
    q = _rand((1, N, 1, D), 3)
    k = _rand((1, 1, 1, D), 4).expand(1, N, 1, D).contiguous()
    v = _rand((1, N, 1, D), 5)
    scale = 0.37
    for mode in ("within", "cross"):
        _, lse = oracle.sfa_prefill(q, k, v, n, mode, scale=scale)
        for p in range(N):
            c = scale * float((q[0, p, 0].double() * k[0, 0, 0].double()).sum())
            size = (p // n + 1) if mode == "within" else p + 1
            assert abs(lse[0, 0, p].item() - (c + np.log(size))) < 1e-12


# ------------------------------------------------------ library-routine pins

@pytest.mark.parametrize("mode", ["within", "cross"])
def test_n1_is_plain_causal_attention(mode):
    B, L, Hq, Hkv, D = 2, 23, 4, 2, 32
    q, k, v = _rand((B, L, Hq, D), 21), _rand((B, L, Hkv, D), 22), _rand((B, L, Hkv, D), 23)
    o, _ = oracle.sfa_prefill(q, k, v, 1, mode)
    ref = _sdpa_causal(q, k, v)
    assert torch.allclose(o, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("scale", [None, 0.3])
def test_cross_is_causal_attention_over_expanded_sequence(scale):
    B, n, L, Hq, Hkv, D = 2, 3, 7, 4, 2, 32
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 31), _rand((B, N, Hkv, D), 32), _rand((B, N, Hkv, D), 33)
    o, _ = oracle.sfa_prefill(q, k, v, n, "cross", scale=scale)
    assert torch.allclose(o, _sdpa_causal(q, k, v, scale=scale), rtol=0, atol=1e-12)


def test_within_is_n_independent_causal_attentions():
    B, n, L, Hq, Hkv, D = 2, 4, 9, 4, 1, 64
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 41), _rand((B, N, Hkv, D), 42), _rand((B, N, Hkv, D), 43)
    o, _ = oracle.sfa_prefill(q, k, v, n, "within")
    for s in range(n):
        ref = _sdpa_causal(q[:, s::n], k[:, s::n], v[:, s::n])
        assert torch.allclose(o[:, s::n], ref, rtol=0, atol=1e-12), s


def test_outlier_keys_match_library():
    # keys scaled x8 give logits far above the rest; the max-subtracted softmax must hold
    B, n, L, Hq, Hkv, D = 1, 4, 16, 2, 1, 128
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 51), _rand((B, N, Hkv, D), 52), _rand((B, N, Hkv, D), 53)
    k[:, ::7] = (k[:, ::7].float() * 8).to(torch.bfloat16)
    for mode in ("within", "cross"):
        o, lse = oracle.sfa_prefill(q, k, v, n, mode)
        assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    o, _ = oracle.sfa_prefill(q, k, v, n, "cross")
    assert torch.allclose(o, _sdpa_causal(q, k, v), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- invariants

def test_cross_row_ignores_later_positions():
    B, n, L, Hq, Hkv, D = 1, 3, 8, 2, 2, 32
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 61), _rand((B, N, Hkv, D), 62), _rand((B, N, Hkv, D), 63)
    o, lse = oracle.sfa_prefill(q, k, v, n, "cross")
    for p in (0, 5, 13, N - 2):
        k2, v2 = k.clone(), v.clone()
        k2[:, p + 1:] = _rand((B, N - p - 1, Hkv, D), 100 + p)
        v2[:, p + 1:] = _rand((B, N - p - 1, Hkv, D), 200 + p)
        o2, lse2 = oracle.sfa_prefill(q, k2, v2, n, "cross")
        assert torch.equal(o[:, : p + 1], o2[:, : p + 1])
        assert torch.equal(lse[:, :, : p + 1], lse2[:, :, : p + 1])
        assert not torch.equal(o[:, p + 1:], o2[:, p + 1:])


@pytest.mark.parametrize("mode", ["within", "cross"])
def test_constant_v_gives_constant_o(mode):
    B, n, L, Hq, Hkv, D = 1, 2, 10, 2, 1, 32
    N = n * L
    q, k = _rand((B, N, Hq, D), 71), _rand((B, N, Hkv, D), 72)
    row = _rand((D,), 73)
    v = row.view(1, 1, 1, D).expand(B, N, Hkv, D).contiguous()
    o, _ = oracle.sfa_prefill(q, k, v, n, mode)
    assert torch.allclose(o, row.double().view(1, 1, 1, D).expand_as(o), rtol=0, atol=1e-14)


def test_gqa_group_map():
    # distinct constant V per KV head identifies which KV head each query head reads
    B, n, L, Hq, Hkv, D = 1, 2, 6, 8, 2, 16
    N = n * L
    q, k = _rand((B, N, Hq, D), 81), _rand((B, N, Hkv, D), 82)
    v = torch.empty(B, N, Hkv, D, dtype=torch.bfloat16)
    for g in range(Hkv):
        v[:, :, g] = float(g + 1)
    for mode in ("within", "cross"):
        o, _ = oracle.sfa_prefill(q, k, v, n, mode)
        for h in range(Hq):
            assert torch.allclose(o[:, :, h], torch.full_like(o[:, :, h], h // (Hq // Hkv) + 1),
                                  rtol=0, atol=1e-14)


@pytest.mark.parametrize("mode", ["within", "cross"])
def test_decode_is_last_n_prefill_rows(mode):
    B, n, Hq, Hkv, D = 3, 4, 4, 2, 32
    Tb = [5, 1, 9]
    T_max = 11
    kc = _rand((B, n * T_max, Hkv, D), 91)
    vc = _rand((B, n * T_max, Hkv, D), 92)
    qfull = _rand((B, n * T_max, Hq, D), 93)
    q = torch.stack([qfull[b, n * (Tb[b] - 1): n * Tb[b]] for b in range(B)])
    o, lse = oracle.sfa_decode(q, kc, vc, Tb, mode)
    for b in range(B):
        N = n * Tb[b]
        ref, ref_lse = oracle.sfa_prefill(qfull[b:b + 1, :N], kc[b:b + 1, :N], vc[b:b + 1, :N],
                                          n, mode)
        assert torch.equal(o[b], ref[0, N - n:])
        assert torch.equal(lse[b], ref_lse[0, :, N - n:])


# ----------------------------------------------------------- gather pins

def test_expand_embed_matches_embedding_per_stream():
    B, L, V, d, n = 3, 17, 50, 24, 4
    ids = torch.randint(0, V, (B, L), generator=torch.Generator().manual_seed(5))
    tables = [_rand((V, d), 300 + s, std=0.02) for s in range(n)]
    out, bad = oracle.expand_embed(ids, tables)
    assert bad == 0 and out.shape == (B, L * n, d)
    for s in range(n):
        ref = F.embedding(ids, tables[s])
        assert torch.equal(out[:, s::n].view(torch.int16), ref.view(torch.int16))


def test_expand_embed_n1_is_embedding():
    ids = torch.randint(0, 40, (2, 9), generator=torch.Generator().manual_seed(6))
    table = _rand((40, 16), 7)
    out, bad = oracle.expand_embed(ids, [table])
    assert bad == 0
    assert torch.equal(out.view(torch.int16), F.embedding(ids, table).view(torch.int16))


def test_expand_embed_out_of_range_ids_give_zero_rows():
    B, L, V, d, n = 1, 6, 10, 8, 2
    ids = torch.tensor([[0, -1, 9, 10, 3, 1 << 40]])
    tables = [_rand((V, d), 400 + s) for s in range(n)]
    out, bad = oracle.expand_embed(ids, tables)
    assert bad == 3
    for t, x in enumerate(ids[0].tolist()):
        for s in range(n):
            row = out[0, t * n + s]
            if 0 <= x < V:
                assert torch.equal(row.view(torch.int16), tables[s][x].view(torch.int16))
            else:
                assert torch.equal(row.view(torch.int16), torch.zeros(d, dtype=torch.int16))


# ------------------------------------------------------ accounting pins

@pytest.mark.parametrize("n,L", [(1, 7), (2, 5), (4, 6), (3, 1)])
def test_pair_counts_match_enumeration(n, L):
    for mode in ("within", "cross"):
        assert wl.unmasked_pairs(mode, n, L) == len(_allowed_bruteforce(n, L, mode))


def test_cost_ratios_against_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "cost_ratios.json")))
    n = g["n"]
    L = 4096
    plain = wl.unmasked_pairs("within", 1, L)
    # within-stream attention is linear in n: exactly n times plain causal
    assert wl.unmasked_pairs("within", n, L) == g["linear_ratio"] * plain
    # dense mixing of all n streams approaches n^2 times plain causal
    ratio = wl.unmasked_pairs("cross", n, L) / plain
    assert abs(ratio - g["dense_ratio"]) / g["dense_ratio"] < 1e-3
    # the layer mixes quoted on the pages add up to the stated depths
    for m in g["layer_mix"]:
        assert sum(m["layers"].values()) == m["depth"]


def test_decode_pair_counts_match_enumeration():
    n, T = 3, 4
    for mode in ("within", "cross"):
        allowed = _allowed_bruteforce(n, T, mode)
        want = sum(1 for (p, _) in allowed if p >= n * (T - 1))
        assert wl.decode_pairs(mode, n, T) == want


# ------------------------------------------------- cross-stream sliding window

@pytest.mark.parametrize("n,L,W", [(1, 7, 3), (3, 6, 2), (2, 5, 1), (4, 4, 9)])
def test_window_mask_by_enumeration(n, L, W):
    N = n * L
    D = 32
    q = torch.zeros(1, N, 1, D, dtype=torch.bfloat16)
    k = _rand((1, N, 1, D), 12)
    v = torch.zeros(1, N, 1, D, dtype=torch.bfloat16)
    v[0, torch.arange(N), 0, torch.arange(N)] = 1.0
    o, lse = oracle.sfa_prefill(q, k, v, n, "cross_window", window=W)
    allowed = _allowed_bruteforce(n, L, "cross_window", W)
    for p in range(N):
        keys = sorted(p2 for (pp, p2) in allowed if pp == p)
        want = torch.zeros(D, dtype=torch.float64)
        want[keys] = 1.0 / len(keys)
        assert torch.equal(o[0, p, 0], want), (p, keys)
        assert abs(lse[0, 0, p].item() - np.log(len(keys))) < 1e-14


def test_window_covering_the_sequence_is_full_cross():
    B, n, L, Hq, Hkv, D = 1, 3, 9, 2, 1, 32
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 13), _rand((B, N, Hkv, D), 14), _rand((B, N, Hkv, D), 15)
    full, full_lse = oracle.sfa_prefill(q, k, v, n, "cross")
    for W in (L, L + 5):
        o, lse = oracle.sfa_prefill(q, k, v, n, "cross_window", window=W)
        assert torch.equal(o, full) and torch.equal(lse, full_lse)


@pytest.mark.parametrize("W", [1, 4, 11])
def test_window_n1_is_banded_causal_attention(W):
    # n = 1: the textbook sliding-window causal attention, a banded mask
    B, L, Hq, Hkv, D = 2, 25, 4, 2, 32
    q, k, v = _rand((B, L, Hq, D), 16), _rand((B, L, Hkv, D), 17), _rand((B, L, Hkv, D), 18)
    o, _ = oracle.sfa_prefill(q, k, v, 1, "cross_window", window=W)
    band = torch.ones(L, L, dtype=torch.bool).tril().triu(-(W - 1))
    qf = q.double().permute(0, 2, 1, 3)
    kf = k.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    vf = v.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    ref = F.scaled_dot_product_attention(qf, kf, vf, attn_mask=band).permute(0, 2, 1, 3)
    assert torch.allclose(o, ref, rtol=0, atol=1e-12)


def test_window_decode_is_last_n_prefill_rows():
    B, n, Hq, Hkv, D, W = 2, 4, 4, 2, 32, 3
    Tb = [7, 2]
    T_max = 8
    kc, vc = _rand((B, n * T_max, Hkv, D), 19), _rand((B, n * T_max, Hkv, D), 20)
    qfull = _rand((B, n * T_max, Hq, D), 21)
    q = torch.stack([qfull[b, n * (Tb[b] - 1): n * Tb[b]] for b in range(B)])
    o, lse = oracle.sfa_decode(q, kc, vc, Tb, "cross_window", window=W)
    for b in range(B):
        N = n * Tb[b]
        ref, ref_lse = oracle.sfa_prefill(qfull[b:b + 1, :N], kc[b:b + 1, :N], vc[b:b + 1, :N],
                                          n, "cross_window", window=W)
        assert torch.equal(o[b], ref[0, N - n:])
        assert torch.equal(lse[b], ref_lse[0, :, N - n:])


@pytest.mark.parametrize("n,L,W", [(1, 7, 3), (3, 6, 2), (2, 5, 1), (4, 4, 9), (2, 9, 4)])
def test_window_pair_counts_match_enumeration(n, L, W):
    assert wl.unmasked_pairs("cross_window", n, L, W) == len(
        _allowed_bruteforce(n, L, "cross_window", W))
    allowed = _allowed_bruteforce(n, L, "cross_window", W)
    assert wl.decode_pairs("cross_window", n, L, W) == sum(1 for (p, _) in allowed
                                                            if p >= n * (L - 1))



# ------------------------------------------------------ training-side pieces

def test_final_stream_rows_is_a_strided_slice():
    B, n, L, d = 2, 4, 9, 24
    x = _rand((B, n * L, d), 80)
    got = oracle.final_stream_rows(x, n)
    assert torch.equal(got.view(torch.int16), x[:, n - 1::n].contiguous().view(torch.int16))


def test_expand_embed_backward_matches_autograd():
    # the library's own gradient of F.embedding, per stream, in fp64
    B, L, V, d, n = 3, 11, 13, 8, 3
    ids = torch.randint(0, V, (B, L), generator=torch.Generator().manual_seed(81))
    ids[0, 0] = V + 2  # out of range: contributes nothing
    g = _rand((B, n * L, d), 82)
    got = oracle.expand_embed_backward(ids, g, n, V)
    valid = (ids >= 0) & (ids < V)
    for s in range(n):
        table = torch.zeros(V, d, dtype=torch.float64, requires_grad=True)
        out = F.embedding(ids.clamp(0, V - 1), table)
        (out * (g[:, s::n].double() * valid[..., None])).sum().backward()
        assert torch.allclose(got[s], table.grad, rtol=0, atol=1e-12), s


# ------------------------------------------- transient intermediate streams (PHD-style)

@pytest.mark.parametrize("n,L", [(1, 6), (3, 5), (4, 4), (2, 7)])
def test_transient_mask_by_enumeration(n, L):
    N = n * L
    D = 32
    q = torch.zeros(1, N, 1, D, dtype=torch.bfloat16)
    k = _rand((1, N, 1, D), 13)
    v = torch.zeros(1, N, 1, D, dtype=torch.bfloat16)
    v[0, torch.arange(N), 0, torch.arange(N)] = 1.0
    o, lse = oracle.sfa_prefill(q, k, v, n, "transient")
    allowed = _allowed_bruteforce(n, L, "transient")
    for p in range(N):
        keys = sorted(p2 for (pp, p2) in allowed if pp == p)
        want = torch.zeros(D, dtype=torch.float64)
        want[keys] = 1.0 / len(keys)
        assert torch.equal(o[0, p, 0], want), (p, keys)
        assert abs(lse[0, 0, p].item() - np.log(len(keys))) < 1e-14


def test_transient_rows_are_attention_over_the_gathered_keys():
    # each row equals unmasked library attention over its key set, gathered by hand:
    # final-stream rows of earlier tokens, then the current token's streams 0..s
    B, n, L, Hq, Hkv, D = 1, 3, 6, 2, 1, 32
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 14), _rand((B, N, Hkv, D), 15), _rand((B, N, Hkv, D), 16)
    o, _ = oracle.sfa_prefill(q, k, v, n, "transient")
    for t in range(L):
        for s in range(n):
            idx = [tt * n + n - 1 for tt in range(t)] + [t * n + ss for ss in range(s + 1)]
            for h in range(Hq):
                qq = q[0, t * n + s, h].double()[None, None, None]
                kk = k[0, idx, h // (Hq // Hkv)].double()[None, None]
                vv = v[0, idx, h // (Hq // Hkv)].double()[None, None]
                ref = F.scaled_dot_product_attention(qq, kk, vv)[0, 0, 0]
                assert torch.allclose(o[0, t * n + s, h], ref, rtol=0, atol=1e-12)


def test_transient_n1_is_plain_causal_attention():
    B, L, Hq, Hkv, D = 2, 19, 4, 2, 32
    q, k, v = _rand((B, L, Hq, D), 17), _rand((B, L, Hkv, D), 18), _rand((B, L, Hkv, D), 19)
    o, _ = oracle.sfa_prefill(q, k, v, 1, "transient")
    assert torch.allclose(o, _sdpa_causal(q, k, v), rtol=0, atol=1e-12)


def test_transient_decode_and_pair_counts():
    B, n, Hq, Hkv, D, T = 1, 4, 2, 1, 32, 6
    kc, vc = _rand((B, n * T, Hkv, D), 20), _rand((B, n * T, Hkv, D), 21)
    qfull = _rand((B, n * T, Hq, D), 22)
    o, lse = oracle.sfa_decode(qfull[:, n * (T - 1):], kc, vc, T, "transient")
    ref, ref_lse = oracle.sfa_prefill(qfull, kc, vc, n, "transient")
    assert torch.equal(o[0], ref[0, n * (T - 1):])
    for nn, LL in [(1, 5), (3, 4), (4, 6)]:
        allowed = _allowed_bruteforce(nn, LL, "transient")
        assert wl.unmasked_pairs("transient", nn, LL) == len(allowed)
        assert wl.decode_pairs("transient", nn, LL) == sum(1 for (p, _) in allowed
                                                           if p >= nn * (LL - 1))



# ------------------------------------------------------------ SFA backward
#
# The backward oracle is written from the derivation of softmax attention's
# gradient.  It is pinned to torch autograd through library attention (fp64)
# under a mask enumerated from the pages' wording, and to two closed forms:
# the key gradients of a row sum to zero (softmax rows sum to one), and the
# value gradients of a KV head sum to the output gradients of its query heads.

def _autograd_sdpa(q, k, v, dout, allowed, N, scale=None):
    """(dq, dk, dv) of sum(O * dout) with O = library attention under an explicit
    boolean mask built from `allowed` pairs; GQA by consecutive groups."""
    Hq, Hkv = q.shape[2], k.shape[2]
    mask = torch.zeros(N, N, dtype=torch.bool)
    for p, p2 in allowed:
        mask[p, p2] = True
    qf = q.double().requires_grad_()
    kf = k.double().requires_grad_()
    vf = v.double().requires_grad_()
    kr = kf.repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    vr = vf.repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(qf.permute(0, 2, 1, 3), kr, vr, attn_mask=mask,
                                       scale=scale).permute(0, 2, 1, 3)
    (o * dout.double()).sum().backward()
    return qf.grad, kf.grad, vf.grad


@pytest.mark.parametrize("mode,n,L,W", [("within", 3, 5, 0), ("cross", 3, 5, 0),
                                        ("within", 1, 9, 0), ("cross", 4, 4, 0),
                                        ("cross_window", 3, 6, 2), ("transient", 3, 5, 0)])
def test_backward_matches_autograd_of_library_attention(mode, n, L, W):
    B, Hq, Hkv, D = 2, 4, 2, 16
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 501), _rand((B, N, Hkv, D), 502), _rand((B, N, Hkv, D), 503)
    dout = _rand((B, N, Hq, D), 504)
    dq, dk, dv = oracle.sfa_prefill_backward(q, k, v, dout, n, mode, window=W)
    rq, rk, rv = _autograd_sdpa(q, k, v, dout, _allowed_bruteforce(n, L, mode, W), N)
    for got, ref, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        assert torch.allclose(got, ref, rtol=0, atol=1e-11), (mode, name,
                                                              (got - ref).abs().max().item())


def test_backward_cross_is_causal_attention_gradient_with_scale():
    B, n, L, Hq, Hkv, D = 1, 2, 8, 2, 1, 32
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 511), _rand((B, N, Hkv, D), 512), _rand((B, N, Hkv, D), 513)
    dout = _rand((B, N, Hq, D), 514)
    dq, dk, dv = oracle.sfa_prefill_backward(q, k, v, dout, n, "cross", scale=0.3)
    qf, kf, vf = (t.double().requires_grad_() for t in (q, k, v))
    o = F.scaled_dot_product_attention(
        qf.permute(0, 2, 1, 3), kf.repeat_interleave(2, 2).permute(0, 2, 1, 3),
        vf.repeat_interleave(2, 2).permute(0, 2, 1, 3), is_causal=True, scale=0.3)
    (o.permute(0, 2, 1, 3) * dout.double()).sum().backward()
    assert torch.allclose(dq, qf.grad, rtol=0, atol=1e-11)
    assert torch.allclose(dk, kf.grad, rtol=0, atol=1e-11)
    assert torch.allclose(dv, vf.grad, rtol=0, atol=1e-11)


@pytest.mark.parametrize("mode", ["within", "cross", "transient"])
def test_backward_closed_forms(mode):
    """sum over keys of dK is zero; sum over keys of dV equals the summed output
    gradients of the KV head's query heads (each softmax row sums to one)."""
    B, n, L, Hq, Hkv, D = 2, 3, 7, 6, 2, 24
    N = n * L
    q, k, v = _rand((B, N, Hq, D), 521), _rand((B, N, Hkv, D), 522), _rand((B, N, Hkv, D), 523)
    dout = _rand((B, N, Hq, D), 524)
    dq, dk, dv = oracle.sfa_prefill_backward(q, k, v, dout, n, mode)
    assert dk.sum(1).abs().max().item() < 1e-11
    G = Hq // Hkv
    want = dout.double().sum(1).reshape(B, Hkv, G, D).sum(2)
    assert torch.allclose(dv.sum(1), want, rtol=0, atol=1e-10)
    # a query whose only allowed key is itself gets no gradient (its output is V[p])
    if mode in ("within", "cross"):
        assert dq[:, 0].abs().max().item() == 0.0


def test_backward_gqa_gradients_sum_over_the_group():
    """With Hq/Hkv = 3, dK/dV of a KV head equal the sums of the per-head
    gradients computed with the KV head repeated for each query head."""
    B, n, L, Hkv, G, D = 1, 2, 5, 2, 3, 16
    Hq, N = Hkv * G, n * L
    q, k, v = _rand((B, N, Hq, D), 531), _rand((B, N, Hkv, D), 532), _rand((B, N, Hkv, D), 533)
    dout = _rand((B, N, Hq, D), 534)
    _, dk, dv = oracle.sfa_prefill_backward(q, k, v, dout, n, "cross")
    k_rep = k.repeat_interleave(G, dim=2).contiguous()
    v_rep = v.repeat_interleave(G, dim=2).contiguous()
    _, dk1, dv1 = oracle.sfa_prefill_backward(q, k_rep, v_rep, dout, n, "cross")
    assert torch.allclose(dk, dk1.reshape(B, N, Hkv, G, D).sum(3), rtol=0, atol=1e-12)
    assert torch.allclose(dv, dv1.reshape(B, N, Hkv, G, D).sum(3), rtol=0, atol=1e-12)


@pytest.mark.parametrize("n,P,C", [(1, 5, 3), (3, 4, 2), (4, 0, 3), (2, 6, 1)])
def test_chunk_pair_counts_match_enumeration(n, P, C):
    """The chunk FLOP counter equals the allowed pairs of the chunk's rows in a
    prefill over P + C tokens, enumerated from the masks."""
    for mode in ("within", "cross"):
        allowed = _allowed_bruteforce(n, P + C, mode)
        rows = {p for p in range(n * P, n * (P + C))}
        want = sum(1 for (p, _) in allowed if p in rows)
        assert wl.chunk_pairs(mode, n, P, C) == want, (mode, n, P, C)
