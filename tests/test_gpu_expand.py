"""GPU parity of hd_expand_embed against the oracle: bit-exact, every shape."""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t):
    return t.view(torch.int16)


def _run(ids, tables):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = hd.hd_expand_embed(ids.to(DEV), [t.to(DEV) for t in tables], dev_status=status)
    torch.cuda.synchronize()
    return out.cpu(), int(status.item())


def test_tiny_workload_bitexact():
    w = wl.WORKLOADS["tiny"]
    ids, tables = wl.make_embedding(w, device=DEV)
    out, st = _run(ids, tables)
    ref, bad = oracle.expand_embed(ids.cpu(), [t.cpu() for t in tables])
    assert st == 0 and bad == 0
    assert torch.equal(_bits(out), _bits(ref))


@pytest.mark.parametrize("n,B,L,V,d", [(1, 1, 1, 7, 8), (3, 2, 33, 50, 24), (16, 1, 5, 9, 264),
                                       (4, 3, 70, 1000, 4096), (2, 1, 129, 5, 136)])
def test_shapes_bitexact(n, B, L, V, d):
    ids = wl.uniform_ids(B, L, V, seed=7 + n)
    tables = [wl.normal_bf16((V, d), 17, 100 + s, std=0.02) for s in range(n)]
    out, st = _run(ids, tables)
    ref, bad = oracle.expand_embed(ids, tables)
    assert st == 0 and bad == 0
    assert torch.equal(_bits(out), _bits(ref))


def test_out_of_range_ids_zero_rows_and_status():
    V, d, n = 10, 16, 3
    ids = torch.tensor([[0, -1, 9, 10, 4, -(1 << 40), 1 << 40, 2]])
    tables = [wl.normal_bf16((V, d), 19, 200 + s) for s in range(n)]
    out, st = _run(ids, tables)
    ref, bad = oracle.expand_embed(ids, tables)
    assert bad == 4
    assert st & hd.binding.HD_DEV_ID_RANGE
    assert torch.equal(_bits(out), _bits(ref))


def test_empty_is_noop():
    tables = [torch.zeros(4, 8, dtype=torch.bfloat16, device=DEV)]
    out = hd.hd_expand_embed(torch.empty(0, 5, dtype=torch.int64, device=DEV), tables)
    assert out.shape == (0, 5, 8)


def test_qwen3_8b_workload_full_size_bitexact():
    """The benchmark's gather: 4 x 2048 Zipf(1.1) ids, 4 tables of 151936 x 4096."""
    w = wl.WORKLOADS["qwen3_8b_prefill"]
    ids, tables = wl.make_embedding(w, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = hd.hd_expand_embed(ids, tables, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # oracle over the whole output (a byte copy: cheap on the host)
    ref, bad = oracle.expand_embed(ids.cpu(), [t.cpu() for t in tables])
    assert bad == 0
    assert torch.equal(_bits(out.cpu()), _bits(ref))
