"""GPU parity of the training-side ends of the path: the final-stream rows
(bit-exact) and the n-table expansion gradient (fp32 atomics vs fp64)."""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import binding
from sequence_expanded_attention_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("B,n,L,d", [(1, 2, 64, 128), (4, 4, 2048, 4096), (2, 3, 17, 24),
                                     (1, 16, 5, 8), (2, 1, 9, 64)])
def test_final_stream_rows_bitexact(B, n, L, d):
    x = wl.normal_bf16((B, n * L, d), 9 + n, 0, device=DEV)
    got = hd.hd_final_stream_rows(x, n)
    torch.cuda.synchronize()
    ref = oracle.final_stream_rows(x.cpu(), n)
    assert torch.equal(got.cpu().view(torch.int16), ref.view(torch.int16))


def _check_grad(ids, g, n, V, tol=1e-5):
    d = g.shape[2]
    tables = [torch.zeros(V, d, dtype=torch.float32, device=DEV) for _ in range(n)]
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    hd.hd_expand_embed_backward(ids.to(DEV), g, tables, dev_status=status)
    torch.cuda.synchronize()
    ref = oracle.expand_embed_backward(ids.cpu(), g.cpu(), n, V)
    for s in range(n):
        err = (tables[s].double().cpu() - ref[s]).abs().max().item()
        scale = ref[s].abs().max().item() + 1e-30
        assert err <= tol * scale, (s, err, scale)
    return int(status.item())


@pytest.mark.parametrize("B,n,L,V,d", [(1, 2, 64, 1000, 128), (3, 4, 70, 50, 24),
                                       (2, 16, 9, 7, 8)])
def test_expand_embed_backward(B, n, L, V, d):
    ids = wl.uniform_ids(B, L, V, seed=31 + n)
    g = wl.normal_bf16((B, n * L, d), 31, 1, device=DEV)
    assert _check_grad(ids, g, n, V) == 0


def test_expand_embed_backward_zipf_workload():
    """The Qwen3-8B-shaped expansion (4 x 2048 Zipf(1.1) ids, 4 streams of
    width 4096): hot ids take thousands of atomic adds into one row."""
    w = wl.WORKLOADS["qwen3_8b_prefill"]
    ids = wl.zipf_ids(w.B, w.L, w.vocab, w.zipf_a, w.seed)
    # a vocabulary slice keeps the oracle's tables small: remap ids into 4096
    V = 4096
    ids = ids % V
    g = wl.normal_bf16((w.B, w.n * w.L, w.d_model), w.seed, 1, std=0.01, device=DEV)
    assert _check_grad(ids, g, w.n, V) == 0


def test_expand_embed_backward_out_of_range_ids():
    ids = torch.tensor([[0, 5, -1, 9]])
    g = wl.normal_bf16((1, 2 * 4, 8), 3, 1, device=DEV)
    st = _check_grad(ids, g, 2, 6)
    assert st & binding.HD_DEV_ID_RANGE
