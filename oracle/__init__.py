"""fp64 CPU oracle for the Hidden Decoding / Stream-Factorized Attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library never calls it and shares no code with it.

The arithmetic lives in ``sfa_oracle.c`` (plain C, fp64, OpenMP over whole
rows); this module only compiles it with gcc, marshals torch CPU tensors into
it and shapes the results.  Each function names the passage it follows:

* ``expand_embed``  -- "Hidden Decoding at Scale" review, "Method"; README
  "Key Idea" item 1: n independent embedding tables, token-major expanded
  sequence, position p = t*n + s.
* ``sfa_prefill`` / ``sfa_prefill_rows`` -- review "Method" and README "Key
  Idea": Stream-Factorized Attention, within-stream (same stream, t' <= t) and
  cross-stream (every earlier expanded position) masks over the length-nL
  sequence, dense masked softmax attention per row.
* ``final_stream_rows`` / ``expand_embed_backward`` -- review "Method": the
  loss is applied only at final-stream positions; the tables' gradient is the
  scatter-add of each stream's gradient rows by token id.
* ``sfa_prefill_backward`` -- review "Method" (the model trains end to end
  with the loss at the final-stream positions, so gradients flow through the
  SFA layers): dQ, dK, dV of masked softmax attention from its derivation.
* ``sfa_decode`` -- review "Limitations"/"Notes" (decode over the retained
  per-stream KV cache): the n new positions of the last token attend the nT
  retained positions; equal by definition to the last n prefill rows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sfa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

WITHIN = 0
CROSS = 1
CROSS_WINDOW = 2
TRANSIENT = 3
_MODES = {"within": WITHIN, "cross": CROSS, "cross_window": CROSS_WINDOW, "transient": TRANSIENT,
          WITHIN: WITHIN, CROSS: CROSS, CROSS_WINDOW: CROSS_WINDOW, TRANSIENT: TRANSIENT}


def build(force: bool = False) -> str:
    """Compile ``sfa_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64p = ctypes.POINTER(ctypes.c_int64)
            vp = ctypes.c_void_p
            lib.oracle_expand_embed.restype = ctypes.c_int64
            lib.oracle_expand_embed.argtypes = [
                vp, ctypes.c_int64, ctypes.c_int64, vp, ctypes.c_int, ctypes.c_int64,
                ctypes.c_int64, vp]
            lib.oracle_attend_rows.restype = ctypes.c_int
            lib.oracle_attend_rows.argtypes = [
                vp, vp, vp, vp, ctypes.c_int64, vp, vp, ctypes.c_int64, ctypes.c_int64,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, ctypes.c_int,
                ctypes.c_int64, ctypes.c_double, vp, vp]
            lib.oracle_final_stream_rows.restype = None
            lib.oracle_final_stream_rows.argtypes = [vp, ctypes.c_int64, ctypes.c_int64,
                                                     ctypes.c_int, ctypes.c_int64, vp]
            lib.oracle_expand_embed_backward.restype = None
            lib.oracle_expand_embed_backward.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp,
                                                         ctypes.c_int, ctypes.c_int64,
                                                         ctypes.c_int64, vp]
            lib.oracle_attend_backward.restype = ctypes.c_int
            lib.oracle_attend_backward.argtypes = [
                vp, vp, vp, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_double,
                vp, vp, vp]
            lib.oracle_num_threads.restype = ctypes.c_int
            del i64p
            _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (all host cores unless OMP_NUM_THREADS says otherwise)."""
    return int(_load().oracle_num_threads())


def _bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CPU tensor -> contiguous uint16 numpy view of its bits."""
    if t.dtype != torch.bfloat16:
        raise TypeError(f"oracle expects bf16 tensors, got {t.dtype}")
    t = t.detach().to("cpu").contiguous()
    return t.view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def expand_embed(ids: torch.Tensor, tables) -> tuple[torch.Tensor, int]:
    """out[b, t*n+s, :] = tables[s][ids[b, t], :]; out-of-range ids give zero rows.

    Returns (out bf16 [B, L*n, d], number of out-of-range ids).
    """
    ids_np = np.ascontiguousarray(ids.detach().cpu().numpy().astype(np.int64))
    B, L = ids_np.shape
    tabs = [_bits(t) for t in tables]
    n = len(tabs)
    V, d = tabs[0].shape
    for t in tabs:
        if t.shape != (V, d):
            raise ValueError("all tables must have the same [V, d] shape")
    out = np.empty((B, L * n, d), dtype=np.uint16)
    ptrs = (ctypes.c_void_p * n)(*[_ptr(t) for t in tabs])
    bad = _load().oracle_expand_embed(_ptr(ids_np), B, L, ptrs, n, V, d, _ptr(out))
    return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16), int(bad)


def final_stream_rows(x: torch.Tensor, n: int) -> torch.Tensor:
    """Rows t*n + n-1 of the expanded hidden states x [B, L*n, d] -> [B, L, d] (byte copy).

    Review "Method": the loss is applied only at the final-stream positions."""
    xb = _bits(x)
    B, N, d = xb.shape
    if N % n:
        raise ValueError("expanded length must be a multiple of n")
    out = np.empty((B, N // n, d), dtype=np.uint16)
    _load().oracle_final_stream_rows(_ptr(xb), B, N // n, n, d, _ptr(out))
    return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)


def expand_embed_backward(ids: torch.Tensor, grad_out: torch.Tensor, n: int, V: int):
    """Gradient of expand_embed w.r.t. the n tables: list of n fp64 [V, d] tensors.

    grad_tables[s][v] = sum of grad_out[b, t*n+s] over tokens with ids[b, t] == v."""
    ids_np = np.ascontiguousarray(ids.detach().cpu().numpy().astype(np.int64))
    B, L = ids_np.shape
    gb = _bits(grad_out)
    d = gb.shape[2]
    grads = [np.zeros((V, d), dtype=np.float64) for _ in range(n)]
    ptrs = (ctypes.c_void_p * n)(*[_ptr(g) for g in grads])
    _load().oracle_expand_embed_backward(_ptr(ids_np), B, L, _ptr(gb), n, V, d, ptrs)
    return [torch.from_numpy(g) for g in grads]


def _default_scale(D: int, scale):
    return 1.0 / float(np.sqrt(D)) if scale is None or scale <= 0 else float(scale)


def attend_rows(q_rows: torch.Tensor, rb, rp, rh, k: torch.Tensor, v: torch.Tensor,
                nkeys, n: int, Hq: int, mode, scale=None, window: int = 0):
    """Masked softmax attention for an explicit list of query rows.

    q_rows: bf16 [R, D]; rb/rp/rh: batch, expanded position, query head per row;
    k, v: bf16 [B, Nk, Hkv, D]; nkeys: valid key rows per batch (int or [B]).
    Returns (o fp64 [R, D], lse fp64 [R]).
    """
    qb = _bits(q_rows)
    kb, vb = _bits(k), _bits(v)
    B, Nk, Hkv, D = kb.shape
    if vb.shape != kb.shape or qb.ndim != 2 or qb.shape[1] != D:
        raise ValueError("shape mismatch between q_rows, k and v")
    R = qb.shape[0]
    rb = np.ascontiguousarray(np.asarray(rb, dtype=np.int64).reshape(R))
    rp = np.ascontiguousarray(np.asarray(rp, dtype=np.int64).reshape(R))
    rh = np.ascontiguousarray(np.asarray(rh, dtype=np.int64).reshape(R))
    nk = np.ascontiguousarray(np.broadcast_to(np.asarray(nkeys, dtype=np.int64), (B,)).copy())
    o = np.empty((R, D), dtype=np.float64)
    lse = np.empty((R,), dtype=np.float64)
    rc = _load().oracle_attend_rows(
        _ptr(qb), _ptr(rb), _ptr(rp), _ptr(rh), R, _ptr(kb), _ptr(vb), B, Nk, Hq, Hkv, D,
        _ptr(nk), n, _MODES[mode], int(window), _default_scale(D, scale), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_attend_rows rejected its arguments (rc={rc})")
    return torch.from_numpy(o), torch.from_numpy(lse)


def sfa_prefill_rows(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int, mode,
                     rb, rp, rh, scale=None, window: int = 0):
    """Selected rows (b, p, h) of SFA prefill over q [B,N,Hq,D], k/v [B,N,Hkv,D]."""
    B, N, Hq, D = q.shape
    rb_t = torch.as_tensor(np.asarray(rb, dtype=np.int64))
    rp_t = torch.as_tensor(np.asarray(rp, dtype=np.int64))
    rh_t = torch.as_tensor(np.asarray(rh, dtype=np.int64))
    q_rows = q[rb_t, rp_t, rh_t]
    return attend_rows(q_rows, rb_t.numpy(), rp_t.numpy(), rh_t.numpy(), k, v, N, n, Hq,
                       mode, scale, window)


def sfa_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int, mode, scale=None,
                window: int = 0):
    """Full SFA prefill: (o fp64 [B, N, Hq, D], lse fp64 [B, Hq, N]), N = n*L.

    mode "cross_window" is the cross-stream layer with a sliding window of
    `window` tokens (review "Method": mixing layers follow the base model's
    pattern, full or sliding-window); mode "transient" is the PHD-style
    control whose intermediate streams are not retained for later tokens
    (review "Prior limitations": only the final stream of earlier tokens is
    seen; the current token's streams up to s stay visible)."""
    B, N, Hq, D = q.shape
    if N % n != 0:
        raise ValueError("expanded length must be a multiple of n")
    bb, pp, hh = torch.meshgrid(torch.arange(B), torch.arange(N), torch.arange(Hq), indexing="ij")
    o, lse = attend_rows(q.reshape(B * N * Hq, D), bb.reshape(-1).numpy(),
                         pp.reshape(-1).numpy(), hh.reshape(-1).numpy(), k, v, N, n, Hq,
                         mode, scale, window)
    return o.reshape(B, N, Hq, D), lse.reshape(B, N, Hq).permute(0, 2, 1).contiguous()


def sfa_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, T, mode,
               scale=None, window: int = 0):
    """Decode of the n new positions of token T (append-then-attend).

    q: bf16 [B, n, Hq, D], the queries of positions n(T-1)+s; k_cache/v_cache:
    bf16 [B, n*T_max, Hkv, D] whose first n*T rows are valid (the new rows
    included).  T is an int or a per-batch sequence of token counts.
    Returns (o fp64 [B, n, Hq, D], lse fp64 [B, Hq, n]).
    """
    B, n, Hq, D = q.shape
    Tb = np.broadcast_to(np.asarray(T, dtype=np.int64), (B,)).copy()
    if (Tb < 1).any():
        raise ValueError("decode needs at least one token in the cache")
    bb, ss, hh = torch.meshgrid(torch.arange(B), torch.arange(n), torch.arange(Hq), indexing="ij")
    rp = n * (Tb[bb.reshape(-1).numpy()] - 1) + ss.reshape(-1).numpy()
    o, lse = attend_rows(q.reshape(B * n * Hq, D), bb.reshape(-1).numpy(), rp,
                         hh.reshape(-1).numpy(), k_cache, v_cache, n * Tb, n, Hq, mode, scale,
                         window)
    return o.reshape(B, n, Hq, D), lse.reshape(B, n, Hq).permute(0, 2, 1).contiguous()


def sfa_prefill_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dout: torch.Tensor,
                         n: int, mode, scale=None, window: int = 0):
    """Gradients (dq, dk, dv) fp64 of SFA prefill for the output gradient dout.

    q, dout: bf16 [B, N, Hq, D]; k, v: bf16 [B, N, Hkv, D].  O, LSE and the
    row terms <dO, O> are recomputed in fp64 inside the oracle."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, N, Hq, D = qb.shape
    Hkv = kb.shape[2]
    if db.shape != qb.shape or vb.shape != kb.shape:
        raise ValueError("shape mismatch")
    dq = np.empty((B, N, Hq, D), dtype=np.float64)
    dk = np.empty((B, N, Hkv, D), dtype=np.float64)
    dv = np.empty((B, N, Hkv, D), dtype=np.float64)
    rc = _load().oracle_attend_backward(
        _ptr(qb), _ptr(kb), _ptr(vb), _ptr(db), B, N, Hq, Hkv, D, n, _MODES[mode],
        int(window), _default_scale(D, scale), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError(f"oracle_attend_backward rejected its arguments (rc={rc})")
    return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)
