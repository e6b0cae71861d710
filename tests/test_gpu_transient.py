"""GPU parity of the transient-intermediate-streams mode (the PHD-style
control of the shared-KV ablation: earlier tokens are seen only through their
final stream, the current token's streams up to s stay visible) against the
fp64 oracle, for prefill and decode."""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_attention, assert_close_lse, check_full_by_batch

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("n,L,B,Hq,Hkv,D", [
    (4, 160, 2, 8, 2, 128),
    (1, 200, 1, 4, 4, 128),     # n = 1: plain causal attention
    (3, 100, 1, 4, 1, 64),
    (16, 20, 1, 2, 2, 128),     # largest n: the own-token part dominates
    (2, 1, 2, 2, 1, 128),       # a single token: only its own streams
    (8, 300, 1, 32, 8, 128),
    (6, 40, 1, 16, 2, 128),     # 8 heads per group: the own-token pass without staging, n <= 8
    (4, 50, 2, 16, 1, 64),      # 16 heads per group, n <= 4, D = 64
])
def test_prefill_transient(n, L, B, Hq, Hkv, D):
    seed = 600 + n + L
    q = wl.normal_bf16((B, n * L, Hq, D), seed, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), seed, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), seed, 2, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_fwd(q, k, v, n, "transient", return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, ref_lse = oracle.sfa_prefill(q.cpu(), k.cpu(), v.cpu(), n, "transient")
    assert_close_attention(o, ref, f"transient n={n} L={L}")
    assert_close_lse(lse, ref_lse, f"transient n={n} L={L}")


def test_prefill_transient_qwen3_full_oracle():
    """The Qwen3-8B shapes (n=4, L=2048, B=4, 32/8) under the transient mask:
    every output row and log-sum-exp against the oracle."""
    w = wl.WORKLOADS["qwen3_8b_prefill"]
    q, k, v = wl.make_qkv(w, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_fwd(q, k, v, w.n, "transient", return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_full_by_batch(o, lse, q, k, v, w.n, "transient", what="qwen3 transient")


@pytest.mark.parametrize("B,n,T,T_max,Hq,Hkv,D", [(2, 4, 300, 310, 32, 8, 128),
                                                  (3, 3, 1, 4, 6, 2, 64),
                                                  (1, 8, 77, 77, 32, 8, 128)])
def test_decode_transient(B, n, T, T_max, Hq, Hkv, D):
    seed = 700 + T
    q = wl.normal_bf16((B, n, Hq, D), seed, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 2, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_decode_fwd(q, kc, vc, T, "transient", return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, ref_lse = oracle.sfa_decode(q.cpu(), kc.cpu(), vc.cpu(), T, "transient")
    assert_close_attention(o, ref, f"decode transient T={T}")
    assert_close_lse(lse, ref_lse, f"decode transient T={T}")


def test_decode_transient_equals_last_prefill_rows():
    B, n, L, Hq, Hkv, D = 2, 4, 130, 8, 2, 128
    q = wl.normal_bf16((B, n * L, Hq, D), 8, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), 8, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), 8, 2, device=DEV)
    o_pre = hd.sfa_prefill_fwd(q, k, v, n, "transient")
    o_dec = hd.sfa_decode_fwd(q[:, n * (L - 1):].contiguous(), k, v, L, "transient")
    assert_close_attention(o_dec, o_pre[:, n * (L - 1):].double(), "transient decode vs prefill")


def test_prefill_transient_own_token_extremes():
    """Own-token scores far above, and far below, every earlier key's: the
    running max starts from the current token's streams, so both the case where
    no later tile moves it and the case where the first tile rescales the
    starting O are taken."""
    B, n, L, Hq, Hkv, D = 1, 4, 300, 4, 1, 128
    q = wl.normal_bf16((B, n * L, Hq, D), 910, 0, device=DEV).float() * 2.0
    k = wl.normal_bf16((B, n * L, Hkv, D), 910, 1, device=DEV).float()
    v = wl.normal_bf16((B, n * L, Hkv, D), 910, 2, device=DEV)
    qh = q[0, :, 0]  # head 0's query rows (the KV group of every head)
    for t in range(0, L, 3):      # own streams aligned with the final stream's query
        for s in range(n - 1):
            k[0, t * n + s, 0] = qh[t * n + n - 1] * 0.5
    for t in range(1, L, 3):      # the previous token's final stream aligned instead
        k[0, (t - 1) * n + n - 1, 0] = qh[t * n + n - 1] * 0.5
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_fwd(q, k, v, n, "transient", return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, ref_lse = oracle.sfa_prefill(q.cpu(), k.cpu(), v.cpu(), n, "transient")
    assert_close_attention(o, ref, "transient extremes")
    assert_close_lse(lse, ref_lse, "transient extremes")
