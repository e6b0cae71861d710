"""GPU parity of sfa_prefill_fwd (tcgen05 path) against the fp64 oracle.

Small cases and the Qwen3-8B-shaped workload compare every output element;
the larger workloads (n=8, L=4096 and the MoE-shaped n=4, L=8192) compare
seeded sampled rows (the first and last row of each 128-row tile in every
stream for every batch and head, rows at outlier keys, the sequence tail,
random rows), in the launch configuration the benchmark times.
"""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import workloads as wl

from _parity import (assert_close_attention, assert_close_lse, check_full_by_batch,
                     sample_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"
MODES = ["within", "cross"]


def _gpu(q, k, v, n, mode, scale=0.0):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_prefill_fwd(q.to(DEV), k.to(DEV), v.to(DEV), n, mode, softmax_scale=scale,
                                return_lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


def _full_check(q, k, v, n, mode, scale=None, what=""):
    o, lse = _gpu(q, k, v, n, mode, scale or 0.0)
    ref_o, ref_lse = oracle.sfa_prefill(q.cpu(), k.cpu(), v.cpu(), n, mode, scale=scale)
    assert_close_attention(o, ref_o, what)
    assert_close_lse(lse, ref_lse, what)


@pytest.mark.parametrize("mode", MODES)
def test_tiny_workload(mode):
    w = wl.WORKLOADS["tiny"]
    q, k, v = wl.make_qkv(w, device=DEV)
    _full_check(q, k, v, w.n, mode, what=f"tiny/{mode}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("n,L,B,Hq,Hkv,D", [
    (4, 160, 2, 8, 2, 128),    # several tiles, ragged tail in both modes
    (1, 300, 1, 4, 4, 128),    # n = 1: plain causal attention
    (3, 100, 1, 4, 1, 64),     # odd n (128 % n != 0), GQA 4:1, D = 64
    (16, 20, 1, 2, 2, 128),    # largest n; within-stream sequences of 20 tokens
    (2, 1, 2, 2, 1, 128),      # a single token
    (8, 64, 1, 32, 8, 128),    # Qwen3-8B head layout, n = 8
    (2, 300, 1, 6, 2, 128),    # GQA with an odd group size (3)
])
def test_shapes(mode, n, L, B, Hq, Hkv, D):
    seed = 1000 + n * 31 + L
    q = wl.normal_bf16((B, n * L, Hq, D), seed, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), seed, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), seed, 2, device=DEV)
    _full_check(q, k, v, n, mode, what=f"{mode} n={n} L={L}")


@pytest.mark.parametrize("mode", MODES)
def test_explicit_scale(mode):
    q = wl.normal_bf16((1, 2 * 130, 2, 128), 5, 0, device=DEV)
    k = wl.normal_bf16((1, 2 * 130, 2, 128), 5, 1, device=DEV)
    v = wl.normal_bf16((1, 2 * 130, 2, 128), 5, 2, device=DEV)
    _full_check(q, k, v, 2, mode, scale=0.21, what="scale 0.21")


@pytest.mark.parametrize("mode", MODES)
def test_gqa_group_map(mode):
    # a distinct constant V per KV head: query head h must return h // (Hq/Hkv) + 1
    B, n, L, Hq, Hkv, D = 1, 2, 150, 8, 2, 128
    q = wl.normal_bf16((B, n * L, Hq, D), 9, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), 9, 1, device=DEV)
    v = torch.empty(B, n * L, Hkv, D, dtype=torch.bfloat16, device=DEV)
    for g in range(Hkv):
        v[:, :, g] = float(g + 1)
    o, _ = _gpu(q, k, v, n, mode)
    for h in range(Hq):
        want = float(h // (Hq // Hkv) + 1)
        assert torch.allclose(o[:, :, h].float(), torch.full_like(o[:, :, h].float(), want),
                              atol=1e-2, rtol=0)


@pytest.mark.parametrize("mode", MODES)
def test_outlier_keys(mode):
    # the MoE-shaped workload's structure at reduced size: 1% of key rows x8
    w = wl.WORKLOADS["moe_long_prefill"]
    q, k, v = wl.make_qkv(w, device=DEV, B=1, L=300)
    q, k, v = q[:, :, :8].contiguous(), k[:, :, :2].contiguous(), v[:, :, :2].contiguous()
    _full_check(q, k, v, w.n, mode, what=f"outliers/{mode}")


def test_all_equal_logits():
    # Q = 0: every allowed key has the same logit; O is the mean of V over the mask
    B, n, L, Hq, Hkv, D = 1, 4, 70, 2, 1, 128
    q = torch.zeros(B, n * L, Hq, D, dtype=torch.bfloat16, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), 3, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), 3, 2, device=DEV)
    for mode in MODES:
        _full_check(q, k, v, n, mode, what=f"q=0/{mode}")


def test_invalid_arguments_rejected():
    q = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_fwd(q, k, k, 2, 7)
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_fwd(q[..., :96].contiguous(), k[..., :96].contiguous(),
                           k[..., :96].contiguous(), 2, "cross")
    q3 = torch.zeros(1, 8, 3, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(hd.HdError):
        hd.sfa_prefill_fwd(q3, k, k, 2, "cross")


# ------------------------------------------------------------- full size

def _sampled_check(name, mode, count=384, B=None, L=None, every_head=False):
    w = wl.WORKLOADS[name]
    q, k, v = wl.make_qkv(w, device=DEV, B=B, L=L)
    Bx, N = q.shape[0], q.shape[1]
    o, lse = _gpu(q, k, v, w.n, mode)
    seq = N // w.n if mode == "within" else N
    extra = ()
    if w.outlier_frac > 0:
        # rows at and just after outlier keys (their logits dominate the softmax)
        knorm = k[0].float().norm(dim=-1).amax(dim=-1)  # [N], batch 0
        hot = torch.nonzero(knorm > 4 * knorm.median()).flatten()[:128].tolist()
        extra = tuple(sorted({min(N - 1, p + d) for p in hot for d in (0, 1, w.n)}))
    rb, rp, rh = sample_rows(Bx, seq, w.n, w.Hq, mode == "within", count, seed=w.seed,
                             extra_positions=extra, every_head=every_head)
    # the oracle reads the sampled query rows and the whole K/V of the batch
    idx = (torch.as_tensor(rb, device=DEV), torch.as_tensor(rp, device=DEV),
           torch.as_tensor(rh, device=DEV))
    ref_o, ref_lse = oracle.attend_rows(q[idx].cpu(), rb, rp, rh, k.cpu(), v.cpu(), N, w.n,
                                        w.Hq, mode)
    got_o = o[idx].cpu()
    got_lse = lse[idx[0], idx[2], idx[1]].cpu()
    assert_close_attention(got_o, ref_o, f"{name}/{mode}")
    assert_close_lse(got_lse, ref_lse, f"{name}/{mode}")
    if every_head:  # every (batch, head) met a tile edge
        assert len(set(zip(rb.tolist(), rh.tolist()))) == Bx * w.Hq


@pytest.mark.parametrize("mode", MODES)
def test_qwen3_8b_full_oracle(mode):
    """The Qwen3-8B-shaped prefill (n=4, L=2048, B=4, 32/8 heads, D=128) in the
    launch the benchmark times: every output row and every log-sum-exp against
    the oracle, element by element, one batch at a time."""
    w = wl.WORKLOADS["qwen3_8b_prefill"]
    q, k, v = wl.make_qkv(w, device=DEV)
    o, lse = _gpu(q, k, v, w.n, mode)
    check_full_by_batch(o, lse, q, k, v, w.n, mode, what=f"qwen3_8b_prefill/{mode}")


# Configs 3-4: the first and last row of every 128-row tile (every stream) for
# every batch and every query head, rows at outlier keys for every head, and
# random rows up to 4096.
@pytest.mark.parametrize("mode", MODES)
def test_large_expansion_full_size_sampled(mode):
    _sampled_check("large_expansion", mode, count=4096, every_head=True)


@pytest.mark.parametrize("mode", MODES)
def test_moe_long_full_size_sampled(mode):
    _sampled_check("moe_long_prefill", mode, count=4096, every_head=True)
