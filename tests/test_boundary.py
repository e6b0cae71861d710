"""The C-ABI boundary on the host (no GPU needed): libhd.so loads, exports
every function include/hd.h declares, and rejects bad arguments with the
documented status codes before anything is launched."""
import ctypes
import os
import re

import pytest

import sequence_expanded_attention_b200 as hd
from sequence_expanded_attention_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hd.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, CUDA, WORKSPACE = range(6)
A = 0x10000  # a 16-byte aligned fake device address: never dereferenced on these paths


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)
    keywords = {"if", "sizeof", "defined"}
    return sorted({n for n in names if n not in keywords and (n.startswith("hd_")
                                                               or n.startswith("sfa_"))})


@pytest.fixture(scope="module")
def lib():
    return binding.load_library()


def test_library_loads_and_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert {"hd_expand_embed", "sfa_prefill_fwd", "sfa_decode_fwd",
            "sfa_decode_workspace_bytes", "hd_status_str"} <= set(names)
    raw = ctypes.CDLL(binding.library_path())
    for n in names:
        assert hasattr(raw, n), f"libhd.so does not export {n}"


def test_status_strings(lib):
    for code, word in [(OK, "ok"), (INVALID, "invalid"), (UNSUPPORTED, "unsupported"),
                       (MISALIGNED, "aligned"), (CUDA, "CUDA"), (WORKSPACE, "workspace")]:
        assert word in lib.hd_status_str(code).decode()
    assert lib.hd_version() >> 16 == 2  # 2: sfa_decode_fwd takes seq_tokens


def _expand(lib, B=1, L=4, n=2, V=10, d=16, ids=A, out=A, tables=None):
    tabs = (ctypes.c_void_p * max(n, 1))(*([A] * max(n, 1) if tables is None else tables))
    return lib.hd_expand_embed(ids, B, L, tabs, n, V, d, out, None, None)


def test_expand_embed_argument_checks(lib):
    assert _expand(lib, n=0) == INVALID
    assert _expand(lib, n=17) == INVALID
    assert _expand(lib, d=12) == INVALID
    assert _expand(lib, d=0) == INVALID
    assert _expand(lib, V=0) == INVALID
    assert _expand(lib, B=-1) == INVALID
    assert _expand(lib, L=0) == OK          # nothing to do, nothing launched
    assert _expand(lib, out=0) == INVALID
    assert _expand(lib, out=A + 8) == MISALIGNED
    assert _expand(lib, tables=[A, A + 4]) == MISALIGNED
    assert _expand(lib, tables=[A, 0]) == INVALID
    assert _expand(lib, ids=A + 4) == MISALIGNED


def _prefill(lib, q=A, k=A, v=A, o=A, lse=None, B=1, L=8, n=2, Hq=4, Hkv=2, D=128, mode=1):
    return lib.sfa_prefill_fwd(q, k, v, o, lse, B, L, n, Hq, Hkv, D, mode, 0.0, None, None)


def test_prefill_argument_checks(lib):
    assert _prefill(lib, D=96) == UNSUPPORTED
    assert _prefill(lib, D=256) == UNSUPPORTED
    assert _prefill(lib, Hq=6, Hkv=4) == UNSUPPORTED
    assert _prefill(lib, n=17) == UNSUPPORTED
    assert _prefill(lib, n=0) == INVALID
    assert _prefill(lib, mode=2) == INVALID
    assert _prefill(lib, mode=3) == INVALID       # the transient mode needs lse
    assert _prefill(lib, Hkv=0) == INVALID
    assert _prefill(lib, L=0) == OK
    assert _prefill(lib, B=0) == OK
    assert _prefill(lib, q=0) == INVALID
    assert _prefill(lib, k=A + 2) == MISALIGNED
    assert _prefill(lib, o=A + 8) == MISALIGNED
    assert _prefill(lib, lse=A + 2) == MISALIGNED


def _decode(lib, q=A, kc=A, vc=A, o=A, B=1, T=4, T_max=4, n=2, Hq=4, Hkv=2, D=128, mode=0,
            ws=None, wsb=0, seq=None):
    return lib.sfa_decode_fwd(q, kc, vc, seq, o, None, B, T, T_max, n, Hq, Hkv, D, mode, 0.0, ws,
                              wsb, None, None)


def test_decode_argument_checks(lib):
    assert _decode(lib, T=0) == INVALID
    assert _decode(lib, T=5, T_max=4) == INVALID
    assert _decode(lib, D=80) == UNSUPPORTED
    assert _decode(lib, Hq=3, Hkv=2) == UNSUPPORTED
    assert _decode(lib, mode=-1) == INVALID
    assert _decode(lib, B=0) == OK
    assert _decode(lib, vc=A + 8) == MISALIGNED
    # per-sequence token counts: a nullable device int32 [B]; T bounds them
    assert _decode(lib, seq=A + 2) == MISALIGNED
    assert _decode(lib, seq=A, T=5, T_max=4) == INVALID
    assert _decode(lib, seq=A, B=0) == OK
    assert _decode(lib, ws=A + 8) == MISALIGNED
    # a workload that needs key splits cannot run without its workspace
    need = lib.sfa_decode_workspace_bytes(1, 4, 32, 8, 128, 4096)
    assert need > 0
    assert _decode(lib, B=1, n=4, Hq=32, Hkv=8, T=4096, T_max=4096) == WORKSPACE
    assert _decode(lib, B=1, n=4, Hq=32, Hkv=8, T=4096, T_max=4096, ws=A,
                   wsb=need - 16) == WORKSPACE


def test_workspace_size_is_zero_for_invalid_shapes(lib):
    assert lib.sfa_decode_workspace_bytes(0, 4, 32, 8, 128, 10) == 0
    assert lib.sfa_decode_workspace_bytes(1, 4, 32, 8, 96, 10) == 0
    assert lib.sfa_decode_workspace_bytes(1, 4, 30, 8, 128, 10) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "library_path", lambda: str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        binding.load_library()


def test_package_has_no_cpu_path():
    # the binding never imports the oracle or any CPU implementation of the method
    src = open(binding.__file__).read()
    assert "oracle" not in src.replace("# ", "")
    assert hd.sfa_prefill_fwd is binding.sfa_prefill_fwd


def test_window_entry_points_argument_checks(lib):
    assert lib.sfa_prefill_window_fwd(A, A, A, A, None, 1, 8, 2, 4, 2, 128, 0, 0.0, None,
                                      None) == INVALID
    assert lib.sfa_prefill_window_fwd(A, A, A, A, None, 1, 8, 2, 4, 2, 96, 3, 0.0, None,
                                      None) == UNSUPPORTED
    assert lib.sfa_prefill_window_fwd(A, A, A, A, None, 0, 8, 2, 4, 2, 128, 3, 0.0, None,
                                      None) == OK
    assert lib.sfa_decode_window_fwd(A, A, A, A, None, 1, 4, 4, 2, 4, 2, 128, 0, 0.0, None, 0,
                                     None, None) == INVALID
    assert lib.sfa_decode_window_fwd(A, A, A, A, None, 1, 5, 4, 2, 4, 2, 128, 2, 0.0, None, 0,
                                     None, None) == INVALID  # T > T_max
    assert lib.sfa_decode_window_workspace_bytes(1, 4, 32, 8, 128, 100, 0) == 0
    # a window as long as the cache plans exactly like the plain cross-stream decode
    assert (lib.sfa_decode_window_workspace_bytes(4, 4, 32, 8, 128, 8192, 8192)
            == lib.sfa_decode_workspace_bytes(4, 4, 32, 8, 128, 8192))


def _chunk(lib, B=1, P=4, C=4, T_max=8, n=2, Hq=4, Hkv=2, D=128, mode=1, W=0, q=A, k=A):
    return lib.sfa_prefill_chunk_fwd(q, k, A, A, None, B, P, C, T_max, n, Hq, Hkv, D, mode, W,
                                     0.0, None, None)


def test_chunk_entry_point_argument_checks(lib):
    assert _chunk(lib, P=5) == INVALID            # prefix + chunk beyond the cache
    assert _chunk(lib, P=-1) == INVALID
    assert _chunk(lib, mode=3) == INVALID         # transient mode has no chunked form
    assert _chunk(lib, mode=2, W=0) == INVALID
    assert _chunk(lib, D=96) == UNSUPPORTED
    assert _chunk(lib, C=0) == OK                 # empty chunk: nothing launched
    assert _chunk(lib, k=A + 2) == MISALIGNED
    assert _chunk(lib, q=0) == INVALID


def _bwd(lib, B=1, L=8, n=2, Hq=4, Hkv=2, D=128, mode=1, W=0, ws=A, wsb=1 << 20, q=A, lse=A):
    return lib.sfa_prefill_bwd(q, A, A, A, A, lse, A, A, A, B, L, n, Hq, Hkv, D, mode, W, 0.0, ws,
                               wsb, None, None)


def test_backward_entry_point_argument_checks(lib):
    assert _bwd(lib, mode=3) == INVALID
    assert _bwd(lib, mode=2, W=0) == INVALID
    assert _bwd(lib, D=96) == UNSUPPORTED
    assert _bwd(lib, Hq=6, Hkv=4) == UNSUPPORTED
    assert _bwd(lib, L=0) == OK
    assert _bwd(lib, lse=0) == INVALID
    assert _bwd(lib, lse=A + 2) == MISALIGNED
    assert _bwd(lib, ws=A + 8) == MISALIGNED
    assert _bwd(lib, wsb=16) == WORKSPACE
    # rows padded to 128 per problem, 8 bytes each
    assert lib.sfa_prefill_bwd_workspace_bytes(2, 100, 4, 8, 1) == 2 * 8 * 512 * 8
    assert lib.sfa_prefill_bwd_workspace_bytes(2, 100, 4, 8, 0) == 2 * 8 * 4 * 128 * 8
    assert lib.sfa_prefill_bwd_workspace_bytes(2, 100, 4, 8, 3) == 0


def _chunk_paged(lib, B=1, C=4, n=2, Hq=4, Hkv=2, D=128, mode=1, W=0, page_rows=256,
                 table=A, prefix=A, max_pages=4, num_pages=8, chunk=None):
    return lib.sfa_prefill_chunk_paged_fwd(A, A, A, table, max_pages, num_pages, page_rows, prefix,
                                           chunk, A, None, B, C, n, Hq, Hkv, D, mode, W, 0.0, None,
                                           None)


def test_chunk_paged_entry_point_argument_checks(lib):
    assert _chunk_paged(lib, mode=3) == INVALID            # no transient chunks
    assert _chunk_paged(lib, mode=2, W=0) == INVALID
    assert _chunk_paged(lib, page_rows=192) == UNSUPPORTED  # cross needs whole 128-row tiles
    assert _chunk_paged(lib, page_rows=255) == UNSUPPORTED  # not a multiple of n
    assert _chunk_paged(lib, mode=0, n=4, page_rows=96) == UNSUPPORTED  # 24 tokens per page
    assert _chunk_paged(lib, mode=0, n=4, page_rows=256, C=0) == OK
    assert _chunk_paged(lib, table=A + 2) == MISALIGNED
    assert _chunk_paged(lib, prefix=0) == INVALID
    assert _chunk_paged(lib, D=96) == UNSUPPORTED
    assert _chunk_paged(lib, chunk=A + 2) == MISALIGNED


def test_size_limits_are_refused_before_launch(lib):
    """Sizes past the kernels' 32-bit coordinates and grid are refused on the
    host (HD_ERR_UNSUPPORTED), never launched."""
    big = (1 << 30) // 2 + 1                      # n = 2: n * L just above 2^30
    assert _prefill(lib, L=big) == UNSUPPORTED
    assert _prefill(lib, B=(1 << 20) + 1) == UNSUPPORTED
    assert _chunk(lib, T_max=big) == UNSUPPORTED  # the cache view's extent
    assert _bwd(lib, L=big) == UNSUPPORTED
    assert _decode(lib, T_max=(1 << 30) + 1) == UNSUPPORTED
    assert _chunk_paged(lib, max_pages=(1 << 22) + 1) == UNSUPPORTED  # table spans > 2^30 rows
