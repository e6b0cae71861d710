"""ctypes binding over libhd.so (C ABI in include/hd.h).

Argument marshalling only: tensors become device pointers and sizes, the
current torch stream becomes the launch stream.  Every step of the path runs
in libhd's CUDA kernels; there is no fallback.  If the library is missing the
first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

SFA_WITHIN = 0
SFA_CROSS = 1
SFA_CROSS_WINDOW = 2  # mode value of the paged decode's sliding-window layers
SFA_TRANSIENT = 3     # PHD-style control: earlier tokens through their final stream only
_MODES = {"within": SFA_WITHIN, "cross": SFA_CROSS, "cross_window": SFA_CROSS_WINDOW,
          "transient": SFA_TRANSIENT}


def _mode(mode) -> int:
    """'within' / 'cross' or the sfa_mode integer; other integers pass through
    so that the library itself rejects them."""
    if isinstance(mode, str):
        if mode not in _MODES:
            raise ValueError(f"unknown SFA mode {mode!r}")
        return _MODES[mode]
    return int(mode)


HD_DEV_ID_RANGE = 0x1
HD_DEV_TIMEOUT = 0x2
HD_DEV_BAD_LENGTH = 0x4
HD_DEV_PAGE_RANGE = 0x8

_HERE = os.path.dirname(os.path.abspath(__file__))
_lock = threading.Lock()
_lib = None


class HdError(RuntimeError):
    """A libhd call returned a non-zero hd_status."""

    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (hd_status={status})")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libhd.so")


def load_library():
    """Load libhd.so (built in-tree by ``build.py``); raise if it is absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(
                f"libhd.so not found at {path}; build it with "
                "`python -m sequence_expanded_attention_b200.build`")
        lib = ctypes.CDLL(path)
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        lib.hd_status_str.restype = ctypes.c_char_p
        lib.hd_status_str.argtypes = [i32]
        lib.hd_last_cuda_error.restype = ctypes.c_char_p
        lib.hd_last_cuda_error.argtypes = []
        lib.hd_version.restype = i32
        lib.hd_expand_embed.restype = i32
        lib.hd_expand_embed.argtypes = [vp, i64, i64, vp, i32, i64, i64, vp, vp, vp]
        lib.sfa_prefill_fwd.restype = i32
        lib.sfa_prefill_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, i32, i32,
                                        f32, vp, vp]
        lib.sfa_decode_workspace_bytes.restype = ctypes.c_size_t
        lib.sfa_decode_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i64]
        lib.sfa_decode_fwd.restype = i32
        lib.sfa_decode_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32,
                                       i32, i32, f32, vp, ctypes.c_size_t, vp, vp]
        lib.sfa_prefill_window_fwd.restype = i32
        lib.sfa_prefill_window_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i32, i32, i32, i32,
                                               i64, f32, vp, vp]
        lib.sfa_decode_window_workspace_bytes.restype = ctypes.c_size_t
        lib.sfa_decode_window_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i64, i64]
        lib.sfa_decode_window_fwd.restype = i32
        lib.sfa_decode_window_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32,
                                              i32, i64, f32, vp, ctypes.c_size_t, vp, vp]
        lib.sfa_decode_paged_workspace_bytes.restype = ctypes.c_size_t
        lib.sfa_decode_paged_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i64, i32, i64]
        lib.sfa_decode_paged_fwd.restype = i32
        lib.sfa_decode_paged_fwd.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, i64, vp, vp, i64,
                                             i32, i32, i32, i32, i32, i64, f32, vp,
                                             ctypes.c_size_t, vp, vp]
        lib.hd_final_stream_rows.restype = i32
        lib.hd_final_stream_rows.argtypes = [vp, i64, i64, i32, i64, vp, vp]
        lib.hd_expand_embed_backward.restype = i32
        lib.hd_expand_embed_backward.argtypes = [vp, vp, i64, i64, i32, i64, i64, vp, vp, vp]
        lib.sfa_prefill_chunk_fwd.restype = i32
        lib.sfa_prefill_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i32, i32,
                                              i32, i32, i32, i64, f32, vp, vp]
        lib.sfa_prefill_chunk_paged_fwd.restype = i32
        lib.sfa_prefill_chunk_paged_fwd.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp,
                                                    i64, i64, i32, i32, i32, i32, i32, i64, f32,
                                                    vp, vp]
        lib.sfa_prefill_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.sfa_prefill_bwd_workspace_bytes.argtypes = [i64, i64, i32, i32, i32]
        lib.sfa_prefill_bwd.restype = i32
        lib.sfa_prefill_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i32, i32,
                                        i32, i32, i32, i64, f32, vp, ctypes.c_size_t, vp, vp]
        lib.hd_selftest_ex2.restype = i32
        lib.hd_selftest_ex2.argtypes = [vp, vp, vp, i64, vp]
        lib.hd_selftest_timeout.restype = i32
        lib.hd_selftest_timeout.argtypes = [vp, ctypes.c_longlong, vp]
        lib.sfa_decode_noalloc_scratch_bytes.restype = ctypes.c_size_t
        lib.sfa_decode_noalloc_scratch_bytes.argtypes = []
        lib.sfa_decode_fwd_noalloc.restype = i32
        lib.sfa_decode_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32,
                                               i32, i32, f32, vp, vp]
        _lib = lib
        return lib


def _check(fn: str, status: int):
    if status != 0:
        lib = load_library()
        msg = lib.hd_status_str(status).decode()
        if status == 4:
            msg += ": " + lib.hd_last_cuda_error().decode()
        raise HdError(fn, status, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name, dtype, ndim):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def hd_expand_embed(ids: torch.Tensor, tables, out: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """out[b, t*n+s, :] = tables[s][ids[b, t], :]  (bf16, bit-exact).

    ids: int64 [B, L] on the GPU; tables: sequence of n bf16 [V, d] GPU tensors.
    """
    _need(ids, "ids", torch.int64, 2)
    n = len(tables)
    for i, t in enumerate(tables):
        _need(t, f"tables[{i}]", torch.bfloat16, 2)
    B, L = ids.shape
    V, d = tables[0].shape
    if out is None:
        out = torch.empty(B, L * n, d, dtype=torch.bfloat16, device=ids.device)
    _need(out, "out", torch.bfloat16, 3)
    ptrs = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in tables])
    st = load_library().hd_expand_embed(_ptr(ids), B, L, ptrs, n, V, d, _ptr(out),
                                        _ptr(dev_status), _stream(ids.device))
    _check("hd_expand_embed", st)
    return out


def hd_final_stream_rows(x: torch.Tensor, n: int, out: torch.Tensor | None = None):
    """Rows t*n + n-1 of the expanded hidden states x [B, L*n, d] -> [B, L, d]."""
    _need(x, "x", torch.bfloat16, 3)
    B, N, d = x.shape
    if N % n:
        raise ValueError(f"expanded length {N} is not a multiple of n={n}")
    if out is None:
        out = torch.empty(B, N // n, d, dtype=torch.bfloat16, device=x.device)
    _need(out, "out", torch.bfloat16, 3)
    _check("hd_final_stream_rows", load_library().hd_final_stream_rows(
        _ptr(x), B, N // n, n, d, _ptr(out), _stream(x.device)))
    return out


def hd_expand_embed_backward(ids: torch.Tensor, grad_out: torch.Tensor, grad_tables,
                             dev_status: torch.Tensor | None = None):
    """grad_tables[s][ids[b, t]] += grad_out[b, t*n+s] (fp32 tables, accumulated in place)."""
    _need(ids, "ids", torch.int64, 2)
    _need(grad_out, "grad_out", torch.bfloat16, 3)
    n = len(grad_tables)
    for i, t in enumerate(grad_tables):
        _need(t, f"grad_tables[{i}]", torch.float32, 2)
    B, L = ids.shape
    V, d = grad_tables[0].shape
    ptrs = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in grad_tables])
    _check("hd_expand_embed_backward", load_library().hd_expand_embed_backward(
        _ptr(ids), _ptr(grad_out), B, L, n, V, d, ptrs, _ptr(dev_status), _stream(ids.device)))
    return grad_tables


def sfa_prefill_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int, mode,
                    softmax_scale: float = 0.0, o: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, return_lse: bool = False,
                    dev_status: torch.Tensor | None = None):
    """SFA prefill: q [B, n*L, Hq, D], k/v [B, n*L, Hkv, D] bf16 -> o [B, n*L, Hq, D] bf16.

    Returns o, or (o, lse fp32 [B, Hq, n*L]) when return_lse.  The transient
    mode always needs an lse buffer (one is made when none is given).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, 4)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if N % n != 0:
        raise ValueError(f"expanded length {N} is not a multiple of n={n}")
    if o is None:
        o = torch.empty_like(q)
    if (return_lse or _mode(mode) == SFA_TRANSIENT) and lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    st = load_library().sfa_prefill_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B,
                                        N // n, n, Hq, Hkv, D, _mode(mode),
                                        float(softmax_scale), _ptr(dev_status),
                                        _stream(q.device))
    _check("sfa_prefill_fwd", st)
    return (o, lse) if return_lse else o


def sfa_prefill_window_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int,
                           window: int, softmax_scale: float = 0.0,
                           o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                           return_lse: bool = False, dev_status: torch.Tensor | None = None):
    """Cross-stream SFA prefill with a sliding window of `window` tokens (shapes as
    sfa_prefill_fwd)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, 4)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if N % n != 0:
        raise ValueError(f"expanded length {N} is not a multiple of n={n}")
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    st = load_library().sfa_prefill_window_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B,
                                               N // n, n, Hq, Hkv, D, int(window),
                                               float(softmax_scale), _ptr(dev_status),
                                               _stream(q.device))
    _check("sfa_prefill_window_fwd", st)
    return (o, lse) if return_lse else o


def sfa_decode_window_workspace_bytes(B: int, n: int, Hq: int, Hkv: int, D: int, T: int,
                                      window: int) -> int:
    return int(load_library().sfa_decode_window_workspace_bytes(B, n, Hq, Hkv, D, T, window))


def sfa_decode_window_fwd(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                          T: int, window: int, softmax_scale: float = 0.0,
                          o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                          return_lse: bool = False, workspace: torch.Tensor | None = None,
                          dev_status: torch.Tensor | None = None):
    """Cross-stream SFA decode with a sliding window of `window` tokens (shapes as
    sfa_decode_fwd)."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, name, torch.bfloat16, 4)
    B, n, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    if k_cache.shape[1] % n != 0:
        raise ValueError("cache length is not a multiple of n")
    T_max = k_cache.shape[1] // n
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=q.device)
    need = sfa_decode_window_workspace_bytes(B, n, Hq, Hkv, D, T, window)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().sfa_decode_window_fwd(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o),
                                              _ptr(lse), B, T, T_max, n, Hq, Hkv, D, int(window),
                                              float(softmax_scale), _ptr(workspace), wbytes,
                                              _ptr(dev_status), _stream(q.device))
    _check("sfa_decode_window_fwd", st)
    return (o, lse) if return_lse else o


def sfa_decode_paged_workspace_bytes(B: int, n: int, Hq: int, Hkv: int, D: int, T_bound: int,
                                     mode, window: int = 0) -> int:
    return int(load_library().sfa_decode_paged_workspace_bytes(B, n, Hq, Hkv, D, T_bound,
                                                               _mode(mode), window))


def sfa_decode_paged_fwd(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                         page_table: torch.Tensor | None, seq_tokens: torch.Tensor | None,
                         T_bound: int, mode, window: int = 0, softmax_scale: float = 0.0,
                         o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                         return_lse: bool = False, workspace: torch.Tensor | None = None,
                         dev_status: torch.Tensor | None = None):
    """SFA decode over a paged, variable-length cache.

    q: bf16 [B, n, Hq, D]; k_pages/v_pages: bf16 [num_pages, page_rows, Hkv, D];
    page_table: int32 [B, max_pages] or None (page b holds sequence b);
    seq_tokens: int32 [B] or None (T_bound everywhere).
    """
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages)):
        _need(t, name, torch.bfloat16, 4)
    B, n, Hq, D = q.shape
    num_pages, page_rows, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_pages = 0
    if page_table is not None:
        _need(page_table, "page_table", torch.int32, 2)
        max_pages = page_table.shape[1]
    if seq_tokens is not None:
        _need(seq_tokens, "seq_tokens", torch.int32, 1)
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=q.device)
    need = sfa_decode_paged_workspace_bytes(B, n, Hq, Hkv, D, T_bound, mode, window)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().sfa_decode_paged_fwd(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), max_pages, num_pages, page_rows,
        _ptr(seq_tokens), T_bound, _ptr(o), _ptr(lse), B, n, Hq, Hkv, D, _mode(mode), window,
        float(softmax_scale), _ptr(workspace), wbytes, _ptr(dev_status), _stream(q.device))
    _check("sfa_decode_paged_fwd", st)
    return (o, lse) if return_lse else o


def sfa_prefill_chunk_fwd(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, P: int,
                          n: int, mode, window: int = 0, softmax_scale: float = 0.0,
                          o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                          return_lse: bool = False, dev_status: torch.Tensor | None = None):
    """SFA prefill of a chunk q [B, n*C, Hq, D] that follows a cached prefix of P tokens;
    k_cache / v_cache [B, n*T_max, Hkv, D] already hold the prefix and the chunk's rows.
    Returns what rows n*P .. n*(P+C)-1 of sfa_prefill_fwd over P + C tokens would hold."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, name, torch.bfloat16, 4)
    B, NC, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    if NC % n != 0 or k_cache.shape[1] % n != 0:
        raise ValueError(f"expanded lengths {NC}, {k_cache.shape[1]} are not multiples of n={n}")
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache differ in shape")
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, NC, dtype=torch.float32, device=q.device)
    st = load_library().sfa_prefill_chunk_fwd(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o),
                                              _ptr(lse), B, int(P), NC // n,
                                              k_cache.shape[1] // n, n, Hq, Hkv, D, _mode(mode),
                                              int(window), float(softmax_scale),
                                              _ptr(dev_status), _stream(q.device))
    _check("sfa_prefill_chunk_fwd", st)
    return (o, lse) if return_lse else o


def sfa_prefill_chunk_paged_fwd(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                                page_table: torch.Tensor, prefix_tokens: torch.Tensor, n: int,
                                mode, window: int = 0, softmax_scale: float = 0.0,
                                chunk_tokens: torch.Tensor | None = None,
                                o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                                return_lse: bool = False,
                                dev_status: torch.Tensor | None = None):
    """SFA prefill of a chunk q [B, n*C, Hq, D] after per-sequence cached prefixes
    (prefix_tokens int32 [B]) over a page pool k/v_pages [num_pages, page_rows,
    Hkv, D] addressed through page_table int32 [B, max_pages]; chunk_tokens
    int32 [B] (optional) gives each sequence's own chunk length <= C."""
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages)):
        _need(t, name, torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    _need(prefix_tokens, "prefix_tokens", torch.int32, 1)
    if chunk_tokens is not None:
        _need(chunk_tokens, "chunk_tokens", torch.int32, 1)
    B, NC, Hq, D = q.shape
    num_pages, page_rows, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    if NC % n != 0:
        raise ValueError(f"expanded length {NC} is not a multiple of n={n}")
    if v_pages.shape != k_pages.shape:
        raise ValueError("k_pages and v_pages differ in shape")
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, NC, dtype=torch.float32, device=q.device)
    st = load_library().sfa_prefill_chunk_paged_fwd(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), page_table.shape[1], num_pages,
        page_rows, _ptr(prefix_tokens), _ptr(chunk_tokens), _ptr(o), _ptr(lse), B, NC // n, n,
        Hq, Hkv, D,
        _mode(mode), int(window), float(softmax_scale), _ptr(dev_status), _stream(q.device))
    _check("sfa_prefill_chunk_paged_fwd", st)
    return (o, lse) if return_lse else o


def sfa_prefill_bwd_workspace_bytes(B: int, L: int, n: int, Hq: int, mode) -> int:
    return int(load_library().sfa_prefill_bwd_workspace_bytes(B, L, n, Hq, _mode(mode)))


def sfa_prefill_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                    dout: torch.Tensor, lse: torch.Tensor, n: int, mode, window: int = 0,
                    softmax_scale: float = 0.0, dq: torch.Tensor | None = None,
                    dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None):
    """Gradients (dq, dk, dv) of SFA prefill.  q, o, dout [B, N, Hq, D]; k, v
    [B, N, Hkv, D]; lse fp32 [B, Hq, N] from the forward pass."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _need(t, name, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if N % n != 0:
        raise ValueError(f"expanded length {N} is not a multiple of n={n}")
    L = N // n
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = sfa_prefill_bwd_workspace_bytes(B, L, n, Hq, mode)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = load_library().sfa_prefill_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
        B, L, n, Hq, Hkv, D, _mode(mode), int(window), float(softmax_scale), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(q.device))
    _check("sfa_prefill_bwd", st)
    return dq, dk, dv


def sfa_decode_workspace_bytes(B: int, n: int, Hq: int, Hkv: int, D: int, T: int) -> int:
    return int(load_library().sfa_decode_workspace_bytes(B, n, Hq, Hkv, D, T))


def sfa_decode_fwd(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, T: int,
                   mode, softmax_scale: float = 0.0, o: torch.Tensor | None = None,
                   lse: torch.Tensor | None = None, return_lse: bool = False,
                   workspace: torch.Tensor | None = None,
                   dev_status: torch.Tensor | None = None,
                   seq_tokens: torch.Tensor | None = None):
    """SFA decode of the n new positions of token T over k/v cache [B, n*T_max, Hkv, D].

    q: bf16 [B, n, Hq, D].  seq_tokens (int32 [B] on the device, optional): the
    token count of each sequence, 1 .. T (T then only bounds them).  The
    workspace is allocated here (torch) when not given.
    """
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, name, torch.bfloat16, 4)
    if seq_tokens is not None:
        _need(seq_tokens, "seq_tokens", torch.int32, 1)
    B, n, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    if k_cache.shape[1] % n != 0:
        raise ValueError("cache length is not a multiple of n")
    T_max = k_cache.shape[1] // n
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=q.device)
    need = sfa_decode_workspace_bytes(B, n, Hq, Hkv, D, T)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().sfa_decode_fwd(_ptr(q), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(seq_tokens), _ptr(o), _ptr(lse), B, T, T_max, n,
                                       Hq, Hkv, D, _mode(mode),
                                       float(softmax_scale), _ptr(workspace), wbytes,
                                       _ptr(dev_status), _stream(q.device))
    _check("sfa_decode_fwd", st)
    return (o, lse) if return_lse else o


def sfa_decode_noalloc_scratch_bytes() -> int:
    """Size of the library's fixed decode scratch array."""
    return int(load_library().sfa_decode_noalloc_scratch_bytes())


def sfa_decode_fwd_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           T: int, mode, softmax_scale: float = 0.0,
                           o: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                           return_lse: bool = False, dev_status: torch.Tensor | None = None):
    """sfa_decode_fwd for callers that cannot allocate device scratch.

    The library keeps the key-split partial results in its own fixed device
    array (see include/hd.h); calls must not overlap on the GPU.  Outputs are
    allocated here only when the caller does not pass them.
    """
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _need(t, name, torch.bfloat16, 4)
    B, n, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    if k_cache.shape[1] % n != 0:
        raise ValueError("cache length is not a multiple of n")
    T_max = k_cache.shape[1] // n
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(B, Hq, n, dtype=torch.float32, device=q.device)
    st = load_library().sfa_decode_fwd_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o),
                                               _ptr(lse), B, T, T_max, n, Hq, Hkv, D,
                                               _mode(mode), float(softmax_scale),
                                               _ptr(dev_status), _stream(q.device))
    _check("sfa_decode_fwd_noalloc", st)
    return (o, lse) if return_lse else o


def hd_selftest_ex2(x: torch.Tensor):
    """(FMA-pipe exp2, MUFU exp2) of an fp32 CUDA tensor, evaluated by libhd's device code."""
    _need(x, "x", torch.float32, 1)
    y_poly, y_mufu = torch.empty_like(x), torch.empty_like(x)
    _check("hd_selftest_ex2", load_library().hd_selftest_ex2(
        _ptr(x), _ptr(y_poly), _ptr(y_mufu), x.numel(), _stream(x.device)))
    return y_poly, y_mufu


def hd_selftest_timeout(dev_status: torch.Tensor, limit_clocks: int) -> None:
    """Run the bounded-wait self-check; it ORs HD_DEV_TIMEOUT into dev_status."""
    _need(dev_status, "dev_status", torch.int32, 1)
    _check("hd_selftest_timeout", load_library().hd_selftest_timeout(
        _ptr(dev_status), int(limit_clocks), _stream(dev_status.device)))
