"""sfa_decode_fwd_noalloc: the decode entry point for callers that cannot
allocate device scratch (plugin interfaces that pass only input and output
buffers; runtimes that forbid allocation on the serving path).

Its key-split partial results live in the library's fixed device array
instead of a caller workspace.  The GPU test checks it against the regular
entry point on two calls in a row (different inputs, so a stale array would
show); the CPU test checks the size limit.  This file is collected last.
"""
import ctypes

import pytest
import torch

import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import binding
from sequence_expanded_attention_b200 import workloads as wl

from _parity import assert_close_attention, assert_close_lse

HD_ERR_WORKSPACE = 5


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    dev = "cuda"
    B, n, T, T_max, Hq, Hkv, D = 2, 4, 1500, 1600, 32, 8, 128
    need = hd.sfa_decode_workspace_bytes(B, n, Hq, Hkv, D, T)
    assert 0 < need <= binding.sfa_decode_noalloc_scratch_bytes()  # the shared array is used
    for call, mode in enumerate(("cross", "within")):
        seed = 500 + call
        q = wl.normal_bf16((B, n, Hq, D), seed, 0, device=dev)
        kc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 1, device=dev)
        vc = wl.normal_bf16((B, n * T_max, Hkv, D), seed, 2, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        ref, ref_lse = hd.sfa_decode_fwd(q, kc, vc, T, mode, return_lse=True)
        got, got_lse = binding.sfa_decode_fwd_noalloc(q, kc, vc, T, mode, return_lse=True,
                                                      dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close_attention(got, ref.double(), f"noalloc call {call} ({mode})")
        assert_close_lse(got_lse, ref_lse, f"noalloc call {call} ({mode})")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = binding.load_library()
    limit = lib.sfa_decode_noalloc_scratch_bytes()
    assert limit == 32 << 20
    # 75 sequences x 4 KV heads (300 key-split units, just past one wave of
    # CTAs) over a 64k-token cache split many ways: more partial results than
    # the array holds
    args = (75, 4, 16, 4, 128, 65536)
    assert lib.sfa_decode_workspace_bytes(*args) > limit
    A = 0x10000  # aligned fake pointer: the call must return before touching memory
    st = lib.sfa_decode_fwd_noalloc(A, A, A, A, None, 75, 65536, 65536, 4, 16, 4, 128, 1, 0.0,
                                    None, None)
    assert st == HD_ERR_WORKSPACE
