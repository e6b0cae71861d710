"""GPU parity of sfa_decode_fwd against the fp64 oracle, and against the GPU
prefill (decode of token T equals the last n prefill rows over n*T positions)."""
import pytest
import torch

import oracle
import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_attention, assert_close_lse

pytestmark = pytest.mark.gpu
DEV = "cuda"
MODES = ["within", "cross"]


def _gpu(q, kc, vc, T, mode, scale=0.0):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_decode_fwd(q, kc, vc, T, mode, softmax_scale=scale, return_lse=True,
                               dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("B,n,T,T_max,Hq,Hkv,D", [
    (2, 2, 5, 7, 4, 2, 64),       # tiny, rows beyond n*T must be ignored
    (1, 4, 300, 301, 32, 8, 128),  # Qwen3-8B heads; 1 (batch, head) pair -> many key splits
    (3, 4, 1, 4, 8, 8, 128),       # T = 1: only the new token's own positions
    (2, 3, 77, 77, 6, 2, 128),     # odd n, ragged last tile
    (1, 8, 40, 40, 32, 8, 128),    # 32 query rows per KV head -> two row groups
    (2, 16, 9, 12, 4, 4, 64),      # largest n
    (2, 4, 700, 700, 64, 4, 128),  # MoE-shaped heads: 64 rows per KV head -> four row groups
])
def test_shapes(mode, B, n, T, T_max, Hq, Hkv, D):
    seed = 77 + n + T
    q = wl.normal_bf16((B, n, Hq, D), seed, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 2, device=DEV)
    # poison the rows past the valid prefix: reading them would show
    if T_max > T:
        kc[:, n * T:] = float("nan")
        vc[:, n * T:] = float("nan")
    o, lse = _gpu(q, kc, vc, T, mode)
    ref_o, ref_lse = oracle.sfa_decode(q.cpu(), kc.cpu(), vc.cpu(), T, mode)
    assert_close_attention(o, ref_o, f"decode {mode} n={n} T={T}")
    assert_close_lse(lse, ref_lse, f"decode {mode}")


@pytest.mark.parametrize("mode", MODES + ["transient"])
def test_decode_per_sequence_lengths(mode):
    """seq_tokens: each sequence's own token count, T only bounds them; rows
    past a sequence's length are poisoned with NaN and must not be read."""
    B, n, T, T_max, Hq, Hkv, D = 5, 4, 700, 720, 32, 8, 128
    q = wl.normal_bf16((B, n, Hq, D), 61, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T_max, Hkv, D), 61, 1, device=DEV)
    vc = wl.normal_bf16((B, n * T_max, Hkv, D), 61, 2, device=DEV)
    lengths = [700, 1, 64, 333, 129]
    for b, t in enumerate(lengths):
        kc[b, n * t:] = float("nan")
        vc[b, n * t:] = float("nan")
    seq = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = hd.sfa_decode_fwd(q, kc, vc, T, mode, return_lse=True, dev_status=status,
                               seq_tokens=seq)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_o, ref_lse = oracle.sfa_decode(q.cpu(), kc.cpu(), vc.cpu(), lengths, mode)
    assert_close_attention(o, ref_o, f"decode seq_tokens {mode}")
    assert_close_lse(lse, ref_lse, f"decode seq_tokens {mode}")


def test_decode_bad_sequence_length_is_flagged():
    B, n, T, Hq, Hkv, D = 3, 2, 40, 4, 2, 64
    q = wl.normal_bf16((B, n, Hq, D), 62, 0, device=DEV)
    kc = wl.normal_bf16((B, n * T, Hkv, D), 62, 1, device=DEV)
    seq = torch.tensor([40, 0, 41], dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = hd.sfa_decode_fwd(q, kc, kc, T, "cross", dev_status=status, seq_tokens=seq)
    torch.cuda.synchronize()
    assert int(status.item()) & hd.HD_DEV_BAD_LENGTH
    assert torch.count_nonzero(o[1:].float()) == 0   # invalid sequences: zero output
    ref_o, _ = oracle.sfa_decode(q[:1].cpu(), kc[:1].cpu(), kc[:1].cpu(), T, "cross")
    assert_close_attention(o[:1], ref_o, "valid sequence beside invalid ones")


@pytest.mark.parametrize("mode", MODES)
def test_decode_equals_last_prefill_rows(mode):
    B, n, L, Hq, Hkv, D = 2, 4, 200, 8, 2, 128
    q = wl.normal_bf16((B, n * L, Hq, D), 5, 0, device=DEV)
    k = wl.normal_bf16((B, n * L, Hkv, D), 5, 1, device=DEV)
    v = wl.normal_bf16((B, n * L, Hkv, D), 5, 2, device=DEV)
    o_pre = hd.sfa_prefill_fwd(q, k, v, n, mode)
    o_dec, _ = _gpu(q[:, n * (L - 1):].contiguous(), k, v, L, mode)
    # two different kernels, same definition: both within the oracle tolerance of each other
    assert_close_attention(o_dec, o_pre[:, n * (L - 1):].double(), f"decode vs prefill {mode}")


def test_workspace_too_small_is_rejected():
    q = wl.normal_bf16((1, 4, 32, 128), 1, 0, device=DEV)
    kc = wl.normal_bf16((1, 4 * 4096, 8, 128), 1, 1, device=DEV)
    need = hd.sfa_decode_workspace_bytes(1, 4, 32, 8, 128, 4096)
    assert need > 0
    ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(hd.HdError):
        hd.sfa_decode_fwd(q, kc, kc, 4096, "cross", workspace=ws)


@pytest.mark.parametrize("mode", MODES)
def test_decode_workload_full_oracle(mode):
    """The decode workload in the launch the benchmark times: batch 64, n = 4,
    an 8192-token (32768-position) cache, 32/8 heads.  Every output row and
    log-sum-exp of all 64 sequences against the oracle, 16 sequences at a time."""
    w = wl.WORKLOADS["decode"]
    q, kc, vc = wl.make_decode(w, device=DEV)
    o, lse = _gpu(q, kc, vc, w.L, mode)
    for b0 in range(0, w.B, 16):
        sl = slice(b0, b0 + 16)
        ref_o, ref_lse = oracle.sfa_decode(q[sl].cpu(), kc[sl].cpu(), vc[sl].cpu(), w.L, mode)
        assert_close_attention(o[sl], ref_o, f"decode workload b={b0}.. {mode}")
        assert_close_lse(lse[sl], ref_lse, f"decode workload b={b0}.. {mode}")
