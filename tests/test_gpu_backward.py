"""GPU parity of the SFA backward (dQ, dK, dV) against the fp64 oracle, which
recomputes the forward pass itself: within-stream, cross-stream and the
sliding-window mode, ragged tiles, GQA groups, D = 64 and 128, n = 1."""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_grad

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fwd_bwd(q, k, v, dout, n, mode, W=0, scale=0.0):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if mode == "cross_window":
        o, lse = hd.sfa_prefill_window_fwd(q, k, v, n, W, softmax_scale=scale, return_lse=True,
                                           dev_status=status)
    else:
        o, lse = hd.sfa_prefill_fwd(q, k, v, n, mode, softmax_scale=scale, return_lse=True,
                                    dev_status=status)
    dq, dk, dv = hd.sfa_prefill_bwd(q, k, v, o, dout, lse, n, mode, window=W,
                                    softmax_scale=scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return dq, dk, dv


def _inputs(B, n, L, Hq, Hkv, D, seed):
    N = n * L
    q = wl.normal_bf16((B, N, Hq, D), seed, 0, device=DEV)
    k = wl.normal_bf16((B, N, Hkv, D), seed, 1, device=DEV)
    v = wl.normal_bf16((B, N, Hkv, D), seed, 2, device=DEV)
    dout = wl.normal_bf16((B, N, Hq, D), seed, 3, device=DEV)
    return q, k, v, dout


@pytest.mark.parametrize("mode,B,n,L,Hq,Hkv,D,W", [
    ("cross", 2, 4, 150, 8, 2, 128, 0),      # N = 600: ragged last tile and chunk
    ("within", 2, 4, 200, 8, 2, 128, 0),     # L = 200 per stream
    ("cross", 1, 3, 100, 4, 4, 64, 0),       # odd n, D = 64, no GQA
    ("within", 1, 2, 300, 4, 1, 64, 0),      # G = 4 query heads per KV head
    ("cross", 1, 1, 333, 4, 2, 128, 0),      # n = 1: plain causal attention
    ("cross_window", 1, 4, 150, 8, 2, 128, 20),
    ("cross_window", 2, 2, 130, 4, 2, 64, 1),
    ("cross", 1, 4, 16, 4, 2, 128, 0),       # a single partial tile
])
def test_backward_matches_oracle(mode, B, n, L, Hq, Hkv, D, W):
    seed = 7000 + n * L + Hq + D + W
    q, k, v, dout = _inputs(B, n, L, Hq, Hkv, D, seed)
    dq, dk, dv = _fwd_bwd(q, k, v, dout, n, mode, W)
    rq, rk, rv = oracle.sfa_prefill_backward(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), n, mode,
                                             window=W)
    what = f"bwd {mode} n={n} L={L} D={D} G={Hq // Hkv}"
    assert_close_grad(dq, rq, what + " dq")
    assert_close_grad(dk, rk, what + " dk")
    assert_close_grad(dv, rv, what + " dv")


def test_backward_with_scale_and_deterministic():
    q, k, v, dout = _inputs(1, 4, 90, 8, 2, 128, 7100)
    a = _fwd_bwd(q, k, v, dout, 4, "cross", scale=0.05)
    b = _fwd_bwd(q, k, v, dout, 4, "cross", scale=0.05)
    for x, y in zip(a, b):
        assert torch.equal(x, y)  # each row has one writer: bitwise repeatable
    rq, rk, rv = oracle.sfa_prefill_backward(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), 4, "cross",
                                             scale=0.05)
    assert_close_grad(a[0], rq, "scale dq")
    assert_close_grad(a[1], rk, "scale dk")
    assert_close_grad(a[2], rv, "scale dv")


def test_backward_closed_forms_at_qwen3_shapes():
    """The Qwen3-8B-shaped cross-stream layer (n=4, L=2048, B=4, 32/8, D=128),
    in the launch the bench times: the value gradients of each KV head sum over
    keys to the output gradients of its query heads, and the key gradients sum
    to zero (softmax rows sum to one, at any size)."""
    w = wl.WORKLOADS["qwen3_8b_prefill"]
    q, k, v = wl.make_qkv(w, device=DEV)
    dout = wl.normal_bf16(q.shape, w.seed, 40, device=DEV)
    dq, dk, dv = _fwd_bwd(q, k, v, dout, w.n, "cross")
    G = w.Hq // w.Hkv
    want = dout.double().sum(1).reshape(w.B, w.Hkv, G, w.D).sum(2)
    got = dv.double().sum(1)
    assert ((got - want).norm() / want.norm()).item() < 1e-2
    # sum over 32768 keys of bf16 rows: compare with the sum of magnitudes
    ksum = dk.double().sum(1).abs()
    kmag = dk.double().abs().sum(1)
    assert (ksum / kmag).max().item() < 1e-2
    assert torch.isfinite(dq.float()).all()


@pytest.mark.parametrize("mode", ["within", "cross"])
def test_backward_full_size_one_kv_group(mode):
    """One KV group of the Qwen3-8B-shaped layer at full length (n=4, L=2048,
    so 8192 expanded positions; 4 query heads on 1 KV head, D=128): dQ, dK and
    dV against the oracle element by element.

    The oracle spreads its work over (batch, KV head) pairs, so the group's
    four query heads go in as four batch entries that share the same K/V; each
    KV head collects the gradients of the query heads that read it, so the
    group's dK and dV are the sums over those entries."""
    B, n, L, Hq, Hkv, D = 1, 4, 2048, 4, 1, 128
    q, k, v, dout = _inputs(B, n, L, Hq, Hkv, D, 7300)
    dq, dk, dv = _fwd_bwd(q, k, v, dout, n, mode)
    qh = q[0].permute(1, 0, 2).unsqueeze(2).cpu()      # [Hq, N, 1, D]: head -> batch entry
    dh = dout[0].permute(1, 0, 2).unsqueeze(2).cpu()
    kh = k.cpu().expand(Hq, -1, -1, -1).contiguous()   # the shared K/V of the group
    vh = v.cpu().expand(Hq, -1, -1, -1).contiguous()
    rq, rk, rv = oracle.sfa_prefill_backward(qh, kh, vh, dh, n, mode)
    rq = rq[:, :, 0].permute(1, 0, 2).unsqueeze(0)     # back to [1, N, Hq, D]
    what = f"bwd full-size {mode} (n=4, L=2048, one KV group)"
    assert_close_grad(dq, rq, what + " dq")
    assert_close_grad(dk, rk.sum(0, keepdim=True), what + " dk")
    assert_close_grad(dv, rv.sum(0, keepdim=True), what + " dv")


def test_backward_argument_checks():
    q = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros(1, 2, 8, dtype=torch.float32, device=DEV)
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_bwd(q, q, q, q, q, lse, 2, "transient")
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_bwd(q, q, q, q, q, lse, 2, "cross_window", window=0)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_bwd(q, q, q, q, q, lse, 2, "cross", workspace=small)
