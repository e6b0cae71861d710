"""Device building blocks on the GPU: the FMA-pipe exp2 against the true 2^x
and the hardware ex2.approx, and the bounded-wait failure path (a wait that
nothing satisfies gives up with HD_DEV_TIMEOUT and the context stays usable)."""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import binding
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_attention

pytestmark = pytest.mark.gpu


def test_poly_exp2_on_device():
    x = torch.cat([torch.linspace(-120.0, 8.0, 1_000_001), torch.tensor([0.0, -0.5, 0.5, 7.999])])
    x = x.float().cuda()
    y_poly, y_mufu = binding.hd_selftest_ex2(x)
    ref = torch.exp2(x.double())
    rel = (y_poly.double() / ref - 1).abs().max().item()
    assert rel < 1e-4, rel
    # the hardware ex2.approx agrees with both to within its own error
    assert (y_mufu.double() / ref - 1).abs().max().item() < 1e-5
    under = binding.hd_selftest_ex2(torch.tensor([-126.0, -300.0, float("-inf")]).cuda())[0]
    assert (under >= 0).all() and (under <= 2.0 ** -124).all()


def test_bounded_wait_gives_up_and_reports():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.hd_selftest_timeout(status, 2_000_000)  # ~1 ms of SM clocks
    torch.cuda.synchronize()
    assert int(status.item()) & binding.HD_DEV_TIMEOUT
    # the context is intact: a normal call still runs and checks out
    q = wl.normal_bf16((1, 2 * 40, 2, 128), 3, 0, device="cuda")
    k = wl.normal_bf16((1, 2 * 40, 2, 128), 3, 1, device="cuda")
    v = wl.normal_bf16((1, 2 * 40, 2, 128), 3, 2, device="cuda")
    o = hd.sfa_prefill_fwd(q, k, v, 2, "cross")
    ref, _ = oracle.sfa_prefill(q.cpu(), k.cpu(), v.cpu(), 2, "cross")
    assert_close_attention(o, ref, "after timeout self-check")
