"""GPU parity of the cross-stream sliding-window entry points against the
fp64 oracle (mode "cross_window"): prefill over several windows, ragged
sequences and GQA layouts, and decode over the last `window` tokens."""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_attention, assert_close_lse, check_full_by_batch

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _prefill(q, k, v, n, W):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_window_fwd(q, k, v, n, W, return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


@pytest.mark.parametrize("n,L,B,Hq,Hkv,D,W", [
    (4, 160, 2, 8, 2, 128, 40),     # window of 160 positions: a few partial tiles
    (4, 300, 1, 4, 1, 128, 1),      # window of one token: own token's earlier streams only
    (3, 100, 1, 4, 2, 64, 33),      # odd n, D = 64
    (1, 700, 1, 2, 2, 128, 200),    # n = 1: plain sliding-window causal attention
    (8, 64, 1, 32, 8, 128, 16),     # Qwen3-8B heads, n = 8
    (2, 90, 2, 2, 1, 128, 1000),    # window longer than the sequence: full cross-stream
])
def test_prefill_window_full(n, L, B, Hq, Hkv, D, W):
    seed = 300 + n + L + W
    q = wl.normal_bf16((B, n * L, Hq, D), seed, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), seed, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), seed, 2, device=DEV)
    o, lse = _prefill(q, k, v, n, W)
    ref, ref_lse = oracle.sfa_prefill(q.cpu(), k.cpu(), v.cpu(), n, "cross_window", window=W)
    assert_close_attention(o, ref, f"window n={n} L={L} W={W}")
    assert_close_lse(lse, ref_lse, f"window n={n} L={L} W={W}")


def test_prefill_window_at_least_sequence_equals_cross():
    B, n, L, Hq, Hkv, D = 1, 4, 200, 8, 2, 128
    q = wl.normal_bf16((B, n * L, Hq, D), 7, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), 7, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), 7, 2, device=DEV)
    o_w, _ = _prefill(q, k, v, n, L)
    o_c = hd.sfa_prefill_fwd(q, k, v, n, "cross")
    assert_close_attention(o_w, o_c.double(), "window = L vs cross")


def test_prefill_window_qwen3_full_oracle():
    """The Qwen3-8B-shaped workload (n=4, L=2048, B=4, 32/8) with a 512-token
    window: every output row and log-sum-exp against the oracle."""
    w = wl.WORKLOADS["qwen3_8b_prefill"]
    W = 512
    q, k, v = wl.make_qkv(w, device=DEV)
    o, lse = _prefill(q, k, v, w.n, W)
    check_full_by_batch(o, lse, q, k, v, w.n, "cross_window", window=W, what="qwen3 window 512")


@pytest.mark.parametrize("B,n,T,T_max,Hq,Hkv,D,W", [
    (2, 4, 300, 310, 32, 8, 128, 50),
    (1, 4, 30, 30, 8, 2, 128, 100),    # window covers the whole cache
    (3, 3, 77, 80, 6, 2, 64, 1),       # window of the new token only
    (1, 8, 500, 500, 32, 8, 128, 17),
])
def test_decode_window(B, n, T, T_max, Hq, Hkv, D, W):
    seed = 900 + T + W
    q = wl.normal_bf16((B, n, Hq, D), seed, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 2, device=DEV)
    if T_max > T:
        kc[:, n * T:] = float("nan")
        vc[:, n * T:] = float("nan")
    # rows before the window must not be read either
    lo = max(0, n * (T - W))
    if lo > 0:
        kc[:, :lo] = float("nan")
        vc[:, :lo] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_decode_window_fwd(q, kc, vc, T, W, return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kc0, vc0 = kc.clone(), vc.clone()
    kc0[:, :lo] = 0
    vc0[:, :lo] = 0
    ref, ref_lse = oracle.sfa_decode(q.cpu(), kc0.cpu(), vc0.cpu(), T, "cross_window", window=W)
    assert_close_attention(o, ref, f"decode window T={T} W={W}")
    assert_close_lse(lse, ref_lse, f"decode window T={T} W={W}")


def test_window_argument_checks():
    q = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_window_fwd(q, q, q, 2, 0)
    with pytest.raises(hd.HdError):
        hd.sfa_decode_window_fwd(q[:, :2].contiguous(), q, q, 4, 0)
