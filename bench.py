"""Benchmark of the Hidden Decoding hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl hd|reference]

One step is one pass of the whole path.  The default step ('headline') is
the largest single-GPU case of each part of the path, launched back to back:
a within-stream and a cross-stream SFA prefill layer of the MoE-shaped long
prefill (n=4, L=8192, batch 2, 64/4 heads, head_dim 128, 1% outlier keys;
separate Q/K/V per layer, as two layers of a model have), a decode step of
the n new positions of the next token in both modes over an 8.59 GB retained
expanded cache (batch 64, n=4, T=8192, 32/8 heads), and the n-table
embedding expansion at the Qwen3-8B shapes (n=4, L=2048, batch 4, vocab
151936 x 4096 tables) with Zipf(1.1) ids and with uniform ids.  Any single
workload can be measured alone with --workload NAME (its step: expansion,
prefill layers and a decode over its own cross-stream cache).

`value` is unmasked attention TFLOP/s over the whole step (every kernel's
time in the denominator); per-kernel times, TFLOP/s or GB/s and roofline
fractions follow in `kernels`.  N > 1 (torchrun) runs independent replicas:
the path has no exchange step, so no collective is on the data path.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sequence_expanded_attention_b200 import workloads as wl  # noqa: E402

METRIC = "SFA prefill TFLOP/s (unmasked) & % bf16 peak; decode/gather GB/s % of HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- utilities

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# A timed region at least this long (back-to-back steps) runs under the power
# cap, so tensor-core kernels in it are judged against the sustained peak.
LONG_RUN_MS = 250.0


def kernel_file_of(op: str) -> str:
    """Source file of the kernel an op name launches."""
    if op.startswith("sfa_prefill_bwd"):
        return "k_sfa_backward.cu"
    if op.startswith("sfa_prefill"):
        return "k_sfa_prefill.cu"
    if op.startswith("sfa_decode"):
        return "k_sfa_decode.cu"
    if op.startswith("hd_expand_embed") and "backward" not in op:
        return "k_expand_embed.cu"
    return "k_train_embed.cu"


def kernel_source_hash(name: str) -> str:
    path = os.path.join(ROOT, "sequence_expanded_attention_b200", "csrc", name)
    h = hashlib.sha256()
    for p in (path, os.path.join(ROOT, "sequence_expanded_attention_b200", "csrc", "hd_ptx.cuh")):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel_file}:{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(kernel_file):
        return None
    # an op of several kernels (the transient prefill's pre-pass) also names
    # the other sources its bytes were measured on
    for other, h in e.get("other_source_hashes", {}).items():
        if kernel_source_hash(other) != h:
            return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings over the process group (every rank
    takes part; the slowest rank sets the job's time)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, units_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms * 1e-3) / 1e12


# ----------------------------------------------------------------- the step

class Step:
    """Device buffers and the launch sequence of one step of a workload."""

    def __init__(self, w: wl.Workload, device, only=None, uniform_gather=False):
        import sequence_expanded_attention_b200 as hd

        self.hd = hd
        self.w = w
        self.dev = device
        self.ops = []  # (name, fn, units dict)
        self.bwd_io = []  # (output gradient, (dq, dk, dv)) of each backward layer
        self.dec_outs = []  # outputs of the decode ops
        n, L, B, Hq, Hkv, D = w.n, w.L, w.B, w.Hq, w.Hkv, w.D

        def wanted(name):
            return only is None or any(name.startswith(o) for o in only)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        if w.prefix:
            # chunked prefill over a page pool: the chunk's K/V rows are in the
            # pages already (written by the layer's projections)
            self.q_chunk, self.kp, self.vp, self.table, self.pre = wl.make_chunk_paged(w, device)
            self.chunk_outs = []
            for mode in w.modes:
                if not wanted(f"sfa_prefill_chunk_paged_fwd[{mode}]"):
                    continue
                o = torch.empty_like(self.q_chunk)
                self.chunk_outs.append(o)
                fn = (lambda mode=mode, o=o:
                      hd.sfa_prefill_chunk_paged_fwd(self.q_chunk, self.kp, self.vp, self.table,
                                                     self.pre, n, mode, o=o,
                                                     dev_status=self.status))
                self.ops.append((f"sfa_prefill_chunk_paged_fwd[{mode}]", fn,
                                 {"flops": 4 * D * B * Hq * wl.chunk_pairs(mode, n, w.prefix, L),
                                  "mode": mode}))
            return
        if w.decode and w.page_rows:
            self.q_dec, self.kc, self.vc, self.table, self.seq = wl.make_paged_decode(w, device)
            self.T = L
            rows_total = int(self.seq.sum()) * n
            for mode in ("within", "cross"):
                if not wanted(f"sfa_decode_fwd[{mode}]"):
                    continue
                ws_bytes = hd.sfa_decode_paged_workspace_bytes(B, n, Hq, Hkv, D, L, mode)
                ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
                o = torch.empty_like(self.q_dec)
                self.dec_outs.append(o)
                fn = (lambda mode=mode, ws=ws, o=o:
                      hd.sfa_decode_paged_fwd(self.q_dec, self.kc, self.vc, self.table,
                                              self.seq, self.T, mode, o=o, workspace=ws,
                                              dev_status=self.status))
                pairs = sum(wl.decode_pairs(mode, n, int(t)) for t in self.seq.tolist())
                self.ops.append((f"sfa_decode_fwd[{mode}]", fn,
                                 {"flops": 4 * D * Hq * pairs,
                                  "bytes": 2 * 2 * rows_total * Hkv * D + 2 * 2 * B * n * Hq * D,
                                  "mode": mode, "ws_bytes": ws_bytes}))
            return
        if w.decode:
            self.q_dec, self.kc, self.vc = wl.make_decode(w, device=device)
            self.T = L
        else:
            if w.vocab and wanted("hd_expand_embed"):
                self.ids, self.tables = wl.make_embedding(w, device=device)
                self.x = torch.empty(B, n * L, w.d_model, dtype=torch.bfloat16, device=device)
                self.ops.append(("hd_expand_embed", self._gather,
                                 {"bytes": wl.gather_bytes(n, B, L, w.d_model), "mode": w.ids}))
                if uniform_gather and w.ids != "uniform":
                    # the same tables read through uniform ids: every row comes
                    # from DRAM (Zipf ids re-read hot rows from L2)
                    self.ids_u = wl.uniform_ids(B, L, w.vocab, w.seed).to(device)
                    self.x_u = torch.empty_like(self.x)
                    self.ops.append(("hd_expand_embed[uniform ids]",
                                     lambda: hd.hd_expand_embed(self.ids_u, self.tables,
                                                                out=self.x_u,
                                                                dev_status=self.status),
                                     {"bytes": wl.gather_bytes(n, B, L, w.d_model),
                                      "mode": "uniform"}))
            if w.name == "qwen3_8b_embed_train":
                self._train_ops(w, device)
                return
            modes = w.schedule if w.schedule else w.modes
            # separate Q/K/V per layer (a different layer has different activations)
            self.layers = []
            for i, mode in enumerate(modes):
                decode_wanted = only is None or any(o.startswith("sfa_decode_fwd") for o in only)
                if not wanted(f"sfa_prefill_fwd[{mode}]") and not (
                        (mode.startswith("cross") or mode == "transient") and decode_wanted):
                    continue
                wi = wl.Workload(**{**w.__dict__, "index": w.index + 100 * (i + 1)})
                q, k, v = wl.make_qkv(wi, device=device)
                o = torch.empty_like(q)
                self.layers.append((mode, q, k, v, o))
                if not wanted(f"sfa_prefill_fwd[{mode}]"):
                    continue
                lse = (torch.empty(B, Hq, n * L, dtype=torch.float32, device=device)
                       if w.backward or mode == "transient" else None)
                if mode == "cross_window":
                    fn = (lambda q=q, k=k, v=v, o=o, lse=lse:
                          hd.sfa_prefill_window_fwd(q, k, v, n, w.window, o=o, lse=lse,
                                                    dev_status=self.status))
                else:
                    fn = (lambda mode=mode, q=q, k=k, v=v, o=o, lse=lse:
                          hd.sfa_prefill_fwd(q, k, v, n, mode, o=o, lse=lse,
                                             dev_status=self.status))
                fl = wl.prefill_flops(mode, n, L, B, Hq, D, w.window)
                info = {"flops": fl, "mode": mode}
                if mode == "transient":
                    info["launches"] = 2  # the current-token pre-pass, then the main kernel
                self.ops.append((f"sfa_prefill_fwd[{mode}]#{i}", fn, info))
                if w.backward:
                    self._backward_op(i, mode, q, k, v, o, lse, fl)
            # decode of the next token over the last cross-stream layer's cache
            cross = ([lay for lay in self.layers if lay[0].startswith("cross")
                      or lay[0] == "transient"] or self.layers)
            if cross:
                _, _, self.kc, self.vc, _ = cross[-1]
            self.q_dec = wl.normal_bf16((B, n, Hq, D), w.seed, wl.S_DECODE_Q, device=device)
            self.T = L
        if w.backward:
            dec_modes = ()
        elif w.window:
            dec_modes = ("cross_window",)
        elif "transient" in w.modes:
            dec_modes = ("transient",)
        else:
            dec_modes = ("within", "cross")
        for mode in dec_modes:
            if not wanted(f"sfa_decode_fwd[{mode}]"):
                continue
            o = torch.empty_like(self.q_dec)
            self.dec_outs.append(o)
            if mode == "cross_window":
                ws_bytes = hd.sfa_decode_window_workspace_bytes(B, n, Hq, Hkv, D, self.T,
                                                                w.window)
                ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
                fn = (lambda ws=ws, o=o:
                      hd.sfa_decode_window_fwd(self.q_dec, self.kc, self.vc, self.T, w.window,
                                               o=o, workspace=ws, dev_status=self.status))
                rows = n * min(self.T, w.window)
            else:
                ws_bytes = hd.sfa_decode_workspace_bytes(B, n, Hq, Hkv, D, self.T)
                ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
                fn = (lambda mode=mode, ws=ws, o=o:
                      hd.sfa_decode_fwd(self.q_dec, self.kc, self.vc, self.T, mode, o=o,
                                        workspace=ws, dev_status=self.status))
                # the transient mask needs only the final-stream rows of earlier
                # tokens and the new token's own rows: those are its algorithmic bytes
                rows = (self.T - 1 + n) if mode == "transient" else n * self.T
            self.ops.append((f"sfa_decode_fwd[{mode}]", fn,
                             {"flops": wl.decode_flops(mode, n, self.T, B, Hq, D, w.window),
                              "bytes": wl.decode_bytes(n, rows // n, B, Hq, Hkv, D),
                              "mode": mode, "ws_bytes": ws_bytes}))

    def _backward_op(self, i, mode, q, k, v, o, lse, fwd_flops):
        """The layer's backward: dQ, dK, dV from a seeded output gradient.  FLOPs are
        counted as 2.5x the forward's (the five products of the standard backward;
        the kernels recompute S and dP once more, which is not counted)."""
        w, hd = self.w, self.hd
        dout = wl.normal_bf16(q.shape, w.seed + 100 * (i + 1), wl.S_DOUT, device=self.dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        self.bwd_io.append((dout, (dq, dk, dv)))
        ws = torch.empty(max(16, hd.sfa_prefill_bwd_workspace_bytes(w.B, w.L, w.n, w.Hq, mode)),
                         dtype=torch.uint8, device=self.dev)
        fn = (lambda: hd.sfa_prefill_bwd(q, k, v, o, dout, lse, w.n, mode, window=w.window,
                                         dq=dq, dk=dk, dv=dv, workspace=ws,
                                         dev_status=self.status))
        self.ops.append((f"sfa_prefill_bwd[{mode}]#{i}", fn,
                         {"flops": int(2.5 * fwd_flops), "mode": mode, "launches": 3}))

    def _train_ops(self, w, device):
        """Final-stream rows of the expanded hidden states and the expansion's
        gradient into n fp32 tables (accumulated every step)."""
        hd, n, L, B, d = self.hd, w.n, w.L, w.B, w.d_model
        self.hx = wl.normal_bf16((B, n * L, d), w.seed, wl.S_Q, device=device)
        self.final = torch.empty(B, L, d, dtype=torch.bfloat16, device=device)
        self.gx = wl.normal_bf16((B, n * L, d), w.seed, wl.S_K, std=0.01, device=device)
        self.ids_t = wl.zipf_ids(B, L, w.vocab, w.zipf_a, w.seed).to(device)
        self.gtables = [torch.zeros(w.vocab, d, dtype=torch.float32, device=device)
                        for _ in range(n)]
        self.ops.append(("hd_final_stream_rows",
                         lambda: hd.hd_final_stream_rows(self.hx, n, out=self.final),
                         {"bytes": 2 * (2 * B * L * d)}))
        self.ops.append(("hd_expand_embed_backward",
                         lambda: hd.hd_expand_embed_backward(self.ids_t, self.gx, self.gtables,
                                                             dev_status=self.status),
                         # bf16 gradient read + fp32 read-modify-write of the table rows
                         {"bytes": 2 * B * L * n * d + 2 * 4 * B * L * n * d + 8 * B * L}))

    def _gather(self):
        self.hd.hd_expand_embed(self.ids, self.tables, out=self.x, dev_status=self.status)

    def launches_per_step(self) -> int:
        count = 0
        for name, _, u in self.ops:
            count += u.get("launches", 1)
            if name.startswith("sfa_decode_fwd") and u.get("ws_bytes", 0) > 0:
                count += 1  # split combine kernel
        return count

    def flops(self) -> int:
        return sum(u.get("flops", 0) for _, _, u in self.ops)

    def bytes(self) -> int:
        return sum(u.get("bytes", 0) for _, _, u in self.ops)

    def units(self):
        """(algorithmic amount per step, scale to the unit, unit): FLOPs in TFLOP/s
        for a step with attention, bytes in GB/s for a step without (the
        training-side gather / scatter-add step)."""
        f = self.flops()
        return (f, 1e12, "TFLOP/s") if f else (self.bytes(), 1e9, "GB/s")

    def run(self, events=None):
        for i, (_, fn, _) in enumerate(self.ops):
            if events is not None:
                events[i].record()
            fn()
        if events is not None:
            events[len(self.ops)].record()

    # --- end to end through the public API with host buffers
    def host_inputs(self):
        """Pinned host copies of the step's per-step inputs (ids, Q/K/V of each
        layer, output gradients, decode queries).  Embedding tables and the
        retained KV cache are resident state: a decode step uploads its n new
        queries and, for a contiguous cache, the n new K/V rows it appends."""
        hostbufs = []
        if hasattr(self, "q_chunk"):
            hostbufs += [self.q_chunk, self.table, self.pre]
        elif hasattr(self, "gx"):
            hostbufs += [self.hx, self.gx, self.ids_t]
        elif self.w.decode:
            hostbufs.append(self.q_dec)
            if self.w.page_rows:
                hostbufs += [self.table, self.seq]
            else:
                n, T = self.w.n, self.T
                hostbufs += [self.kc[:, n * (T - 1):n * T], self.vc[:, n * (T - 1):n * T]]
        else:
            if hasattr(self, "ids"):
                hostbufs.append(self.ids)
            if hasattr(self, "ids_u"):
                hostbufs.append(self.ids_u)
            for (_, q, k, v, _) in self.layers:
                hostbufs += [q, k, v]
            hostbufs += [dout for dout, _ in self.bwd_io]
            if any(nm.startswith("sfa_decode") for nm, _, _ in self.ops):
                hostbufs.append(self.q_dec)
        pairs = []
        for t in hostbufs:
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            h.copy_(t)
            pairs.append((h, t))
        return pairs

    def host_outputs(self):
        outs = []
        if hasattr(self, "chunk_outs"):
            outs += self.chunk_outs
        elif hasattr(self, "final"):
            outs.append(self.final)
        elif not self.w.decode:
            if hasattr(self, "x"):
                outs.append(self.x)
            if hasattr(self, "x_u"):
                outs.append(self.x_u)
            outs += [lay[4] for lay in self.layers]
            for _, grads in self.bwd_io:
                outs += list(grads)
        outs += self.dec_outs
        pairs = [(torch.empty(t.shape, dtype=t.dtype, pin_memory=True), t) for t in outs]
        return pairs


# The default step: the largest single-GPU prefill (MoE-shaped, n=4, L=8192,
# batch 2, 64/4 heads, 1% outlier keys) in both SFA modes, the decode step over
# the 8.59 GB retained cache (batch 64, T=8192) in both modes, and the n-table
# expansion at the Qwen3-8B shapes with Zipf and with uniform ids.
HEADLINE = "headline"
HEADLINE_PARTS = (
    ("moe_long_prefill", ("sfa_prefill_fwd",), False),
    ("decode", None, False),
    ("qwen3_8b_prefill", ("hd_expand_embed",), True),
)


class CompositeStep:
    """Several workloads' steps launched back to back as one step.  Op names
    carry their workload after an '@'; each op's units name the workload."""

    def __init__(self, parts, device):
        self.parts = []
        self.ops = []
        for name, only, uniform in parts:
            st = Step(wl.WORKLOADS[name], device, only, uniform_gather=uniform)
            self.parts.append(st)
            for op, fn, u in st.ops:
                self.ops.append((f"{op}@{name}", fn, {**u, "workload": name}))
        self.w = self.parts[0].w

    def status_value(self) -> int:
        v = 0
        for st in self.parts:
            v |= int(st.status.item())
        return v

    def launches_per_step(self) -> int:
        return sum(st.launches_per_step() for st in self.parts)

    def flops(self) -> int:
        return sum(st.flops() for st in self.parts)

    def bytes(self) -> int:
        return sum(st.bytes() for st in self.parts)

    units = Step.units
    run = Step.run

    def host_inputs(self):
        return [pair for st in self.parts for pair in st.host_inputs()]

    def host_outputs(self):
        return [pair for st in self.parts for pair in st.host_outputs()]


def make_step(workload: str, device, only=None, batch=None):
    """The step of a named workload ('headline' is the composite default)."""
    if workload == HEADLINE:
        return CompositeStep(HEADLINE_PARTS, device)
    w = wl.WORKLOADS[workload]
    if batch is not None:
        w = wl.Workload(**{**w.__dict__, "B": batch})
    st = Step(w, device, only, uniform_gather=True)
    st.ops = [(op, fn, {**u, "workload": w.name}) for op, fn, u in st.ops]
    st.status_value = lambda: int(st.status.item())
    return st


def time_steps(step: Step, steps: int, warmup: int, world, rank):
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    nops = len(step.ops)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nops + 1)] for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        step.run(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(end)
    per_op = [[evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)] for j in range(nops)]
    return total_ms, per_op


def time_e2e(sets, steps: int, warmup: int, world):
    """The step end to end through the public API: every step uploads its inputs
    from pinned host memory and reads its outputs back.  With two buffer sets
    (two Step objects) the uploads of step i+1 and the read-back of step i-1
    run on their own streams while step i computes; set k is reused only after
    its previous outputs were read back.  Returns (ms for `steps` steps, bytes
    up per step, bytes down per step)."""
    ins = [st.host_inputs() for st in sets]
    outs = [st.host_outputs() for st in sets]
    h2d = sum(h.numel() * h.element_size() for h, _ in ins[0])
    d2h = sum(h.numel() * h.element_size() for h, _ in outs[0])
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    uploaded = [torch.cuda.Event() for _ in sets]
    computed = [torch.cuda.Event() for _ in sets]
    fetched = [torch.cuda.Event() for _ in sets]

    def one(i):
        k = i % len(sets)
        with torch.cuda.stream(up):
            up.wait_event(computed[k])  # the previous use of set k has read its inputs
            for h, d in ins[k]:
                d.copy_(h, non_blocking=True)
            uploaded[k].record(up)
        comp.wait_event(uploaded[k])
        comp.wait_event(fetched[k])  # the previous outputs of set k are on the host
        sets[k].run()
        computed[k].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(computed[k])
            for h, d in outs[k]:
                h.copy_(d, non_blocking=True)
            fetched[k].record(down)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(comp)
    up.wait_event(start)
    for i in range(steps):
        one(i)
    for ev in fetched:
        comp.wait_event(ev)
    end.record(comp)
    torch.cuda.synchronize()
    return start.elapsed_time(end), h2d, d2h


def within_vs_plain_ms(w: wl.Workload, device, within_fn, iters: int = 10):
    """The within-stream layer and plain causal attention (n = 1) at the same L,
    batch and heads, timed alternately in one loop so that both run at the same
    clocks and power state: the reference point for the within-stream cost
    target.  Returns (within ms, plain ms), means over `iters`."""
    import sequence_expanded_attention_b200 as hd

    w1 = wl.Workload(**{**w.__dict__, "n": 1, "index": w.index + 999})
    q, k, v = wl.make_qkv(w1, device=device)
    o = torch.empty_like(q)
    for _ in range(3):
        within_fn()
        hd.sfa_prefill_fwd(q, k, v, 1, "cross", o=o)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(iters)]
    for e in ev:
        e[0].record()
        within_fn()
        e[1].record()
        hd.sfa_prefill_fwd(q, k, v, 1, "cross", o=o)
        e[2].record()
    torch.cuda.synchronize()
    t_w = sum(e[0].elapsed_time(e[1]) for e in ev) / iters
    t_p = sum(e[1].elapsed_time(e[2]) for e in ev) / iters
    return t_w, t_p


# ----------------------------------------------------------------- CPU oracle

_CPU_INPUTS = {}


def cpu_baseline(w: wl.Workload, target_s: float = 12.0):
    """The oracle as it stands, on this host's cores, over a bounded sample of the
    workload's dominant op (cross-stream prefill rows; decode rows for a decode
    workload; the expansion gradient for the training-side workload).
    Returns (value, unit, threads, description)."""
    import oracle

    g = torch.Generator().manual_seed(w.seed)
    if w.name == "qwen3_8b_embed_train":
        Ls = 256  # tokens of one sequence per repetition
        Vs = min(w.vocab, 32768)  # fp64 tables of the sampled vocabulary (zero pages until touched)
        ids = wl.zipf_ids(1, Ls, Vs, w.zipf_a, w.seed)
        gx = wl.normal_bf16((1, w.n * Ls, w.d_model), w.seed, wl.S_K, std=0.01)
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < target_s:
            oracle.expand_embed_backward(ids, gx, w.n, Vs)
            reps += 1
        dt = time.perf_counter() - t0
        by = reps * (2 * Ls * w.n * w.d_model + 2 * 4 * Ls * w.n * w.d_model + 8 * Ls)
        desc = (f"{reps} x expansion gradient of {Ls} Zipf tokens into {w.n} fp64 tables "
                f"[{Vs}][{w.d_model}] (bytes counted as the GPU step's)")
        return by / dt / 1e9, "GB/s", oracle.num_threads(), desc
    if w.prefix:
        # random cross-stream rows of the chunk of batch 0 over its P + C tokens
        N = w.n * (w.prefix + w.L)
        q = wl.normal_bf16((1, N, w.Hq, w.D), w.seed, wl.S_Q)
        k = wl.normal_bf16((1, N, w.Hkv, w.D), w.seed, wl.S_K)
        v = wl.normal_bf16((1, N, w.Hkv, w.D), w.seed, wl.S_V)
        rows_done, flops, chunk = 0, 0, 64
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < target_s:
            rp = (w.n * w.prefix + torch.randint(0, w.n * w.L, (chunk,), generator=g)).numpy()
            rh = torch.randint(0, w.Hq, (chunk,), generator=g).numpy()
            oracle.attend_rows(q[0, rp, rh], np.zeros(chunk, dtype=np.int64), rp, rh, k, v, N,
                               w.n, w.Hq, "cross")
            rows_done += chunk
            flops += int(sum(4 * w.D * (p + 1) for p in rp))
            chunk = min(chunk * 2, 4096)
        dt = time.perf_counter() - t0
        desc = (f"{rows_done} random cross-stream chunk rows of batch 0 ({w.L} tokens after "
                f"{w.prefix}, {w.Hq} heads), unmasked flops only")
        return flops / dt / 1e12, "TFLOP/s", oracle.num_threads(), desc
    if w.backward:
        # the cross-stream backward over a causal prefix of the first Np positions
        # of batch 0 (a prefix is a complete causal problem), all heads
        Np = 256
        q = wl.normal_bf16((1, Np, w.Hq, w.D), w.seed, wl.S_Q)
        k = wl.normal_bf16((1, Np, w.Hkv, w.D), w.seed, wl.S_K)
        v = wl.normal_bf16((1, Np, w.Hkv, w.D), w.seed, wl.S_V)
        dout = wl.normal_bf16((1, Np, w.Hq, w.D), w.seed, wl.S_DOUT)
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < target_s:
            oracle.sfa_prefill_backward(q, k, v, dout, w.n, "cross")
            reps += 1
        dt = time.perf_counter() - t0
        fl = reps * 2.5 * wl.prefill_flops("cross", w.n, Np // w.n, 1, w.Hq, w.D)
        desc = (f"{reps} x cross-stream backward of a {Np}-position prefix of batch 0 "
                f"({w.Hq}/{w.Hkv} heads), flops counted as 2.5x the forward's")
        return fl / dt / 1e12, "TFLOP/s", oracle.num_threads(), desc
    if w.decode:
        B1 = 1
        q = wl.normal_bf16((B1, w.n, w.Hq, w.D), w.seed, wl.S_DECODE_Q)
        kc = wl.normal_bf16((B1, w.n * w.L, w.Hkv, w.D), w.seed, wl.S_CACHE_K)
        vc = wl.normal_bf16((B1, w.n * w.L, w.Hkv, w.D), w.seed, wl.S_CACHE_V)
        t0 = time.perf_counter()
        reps = 0
        while True:
            oracle.sfa_decode(q, kc, vc, w.L, "cross")
            reps += 1
            if time.perf_counter() - t0 > target_s:
                break
        dt = time.perf_counter() - t0
        fl = reps * wl.decode_flops("cross", w.n, w.L, B1, w.Hq, w.D)
        desc = f"{reps} x cross-stream decode of 1 sequence ({w.n}x{w.L} cache rows, {w.Hq} heads)"
        return fl / dt / 1e12, "TFLOP/s", oracle.num_threads(), desc
    # rows of the workload's most expensive prefill mask
    mode = ("transient" if "transient" in w.modes else
            "cross_window" if "cross_window" in w.modes else "cross")

    def allowed(p):  # keys of expanded query row p under that mask
        t, s = divmod(int(p), w.n)
        if mode == "transient":
            return t + s + 1
        if mode == "cross_window":
            return w.n * min(t, w.window - 1) + s + 1
        return int(p) + 1

    B1 = 1
    N = w.n * w.L
    key = (w.name, w.n, w.L, w.Hq, w.Hkv, w.D)
    if key not in _CPU_INPUTS:  # batch 0 of the workload, generated once per process
        _CPU_INPUTS.clear()
        _CPU_INPUTS[key] = wl.make_qkv(w, B=B1)
    q, k, v = _CPU_INPUTS[key]
    rows_done = 0
    flops = 0
    t0 = time.perf_counter()
    chunk = 64
    while time.perf_counter() - t0 < target_s:
        rp = torch.randint(0, N, (chunk,), generator=g).numpy()
        rh = torch.randint(0, w.Hq, (chunk,), generator=g).numpy()
        rb = np.zeros(chunk, dtype=np.int64)
        oracle.attend_rows(q[0, rp, rh], rb, rp, rh, k, v, N, w.n, w.Hq, mode,
                           window=w.window if mode == "cross_window" else 0)
        rows_done += chunk
        flops += int(sum(4 * w.D * allowed(p) for p in rp))
        chunk = min(chunk * 2, 4096)
    dt = time.perf_counter() - t0
    desc = (f"{rows_done} random {mode} prefill rows of batch 0 "
            f"(N={N}, {w.Hq} heads), unmasked flops only")
    return flops / dt / 1e12, "TFLOP/s", oracle.num_threads(), desc


# ----------------------------------------------------------------- main

def workload_config(name: str, batch=None) -> dict:
    """The JSON `config` of a workload (the composite lists its parts)."""
    if name == HEADLINE:
        parts = {}
        for wname, only, uniform in HEADLINE_PARTS:
            w = wl.WORKLOADS[wname]
            d = {"n": w.n, "L" if not w.decode else "T": w.L, "B": w.B}
            if only and only[0] == "hd_expand_embed":
                d.update(vocab=w.vocab, d_model=w.d_model,
                         ids=[f"zipf{w.zipf_a}"] + (["uniform"] if uniform else []))
            else:
                d.update(Hq=w.Hq, Hkv=w.Hkv, D=w.D, modes=["within", "cross"])
                if w.outlier_frac:
                    d["outlier_keys"] = f"{w.outlier_frac:g} of K rows x{w.outlier_factor:g}"
            parts[wname + ("[gather]" if only and only[0] == "hd_expand_embed" else "")] = d
        return {"workload": "+".join(parts), "parts": parts}
    w = wl.WORKLOADS[name]
    B = w.B if batch is None else batch
    return {"workload": w.name, "n": w.n, "L": w.L, "B": B, "Hq": w.Hq, "Hkv": w.Hkv,
            "D": w.D, "vocab": w.vocab, "d_model": w.d_model,
            "ids": f"zipf{w.zipf_a}" if w.ids == "zipf" else w.ids}


def baseline_workload(name: str) -> wl.Workload:
    """The workload whose dominant op the oracle samples (the composite's
    prefill part: its cross-stream layer is the step's largest kernel)."""
    return wl.WORKLOADS[HEADLINE_PARTS[0][0] if name == HEADLINE else name]


def run_reference(args, w, rank, config=None):
    if rank != 0:
        return
    per_step, wall = [], []
    desc = ""
    threads = 0
    for _ in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        v, unit, threads, desc = cpu_baseline(
            w, target_s=max(2.0, 60.0 / (args.steps + args.warmup)))
        wall.append(time.perf_counter() - t0)
        per_step.append(v)
    vals = per_step[args.warmup:]
    value = statistics.median(vals)
    # one step is one bounded sample of the workload (its wall time, host clock)
    ms_sample = 1e3 * statistics.mean(wall[args.warmup:])
    cfg = dict(config) if config else {"workload": w.name, "n": w.n, "L": w.L, "B": w.B,
                                        "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D}
    cfg["parallelism"] = "host cores"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_sample, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": cfg,
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


NOMINAL_HBM_GBS = 8000.0  # the "about 8 TB/s" HBM3e figure the bandwidth bars are quoted against


def targets_summary(kernels: dict, within_ratio, peaks=None):
    """The hot path's bars beside what this step measured: prefill >= 0.60 of
    the bf16 peak (burst and sustained), within-stream <= 1.2 x n x plain
    causal, decode and expansion >= 0.70 of HBM."""
    out = {}
    for kind in ("burst", "sustained"):
        pre = {k.split("@")[0].split("#")[0]: v.get(f"frac_bf16_{kind}")
               for k, v in kernels.items() if k.startswith("sfa_prefill_fwd")}
        if pre:
            out[f"prefill_frac_bf16_{kind}"] = {"bar": 0.60, **pre}
    if within_ratio is not None:
        out["within_vs_n_plain"] = {"bar": 1.2, "ratio": within_ratio}
    dec = {k.split("@")[0]: v.get("frac_hbm") for k, v in kernels.items()
           if k.startswith("sfa_decode")}
    if dec:
        out["decode_frac_hbm"] = {"bar": 0.70, **dec}
    gat = {k.split("@")[0]: v.get("frac_hbm") for k, v in kernels.items()
           if k.startswith("hd_expand_embed")}
    if gat:
        out["gather_frac_hbm"] = {"bar": 0.70, **gat}
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=HEADLINE, choices=[HEADLINE] + sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="hd", choices=["hd", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override a single workload's batch (reduced cases for profiler captures)")
    ap.add_argument("--only", default=None,
                    help="comma list of op-name prefixes to keep in a single workload's step, "
                         "e.g. 'sfa_prefill_fwd[cross]' (profiler captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.workload == HEADLINE and (args.batch is not None or args.only):
        ap.error("--batch and --only apply to a single workload")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    only = args.only.split(",") if args.only else None
    config = workload_config(args.workload, args.batch)

    if args.impl == "reference":
        run_reference(args, baseline_workload(args.workload), rank, config)
        return

    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(device)

    peaks, peak_kind = load_peaks()
    step = make_step(args.workload, device, only, args.batch)
    parts = step.parts if isinstance(step, CompositeStep) else [step]
    wmap = {st.w.name: st.w for st in parts}
    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    total_ms, per_op = time_steps(step, args.steps, args.warmup, world, rank)
    clocks = sampler.stop()
    status = step.status_value()

    e2e_ms, h2d, d2h = (None, 0, 0)
    if not args.no_e2e:
        e2e_steps = max(4, args.steps // 2)
        e2e_ms, h2d, d2h = time_e2e([step, make_step(args.workload, device, only, args.batch)],
                                    e2e_steps, 2, world)

    if world > 1:
        total_ms, e2e_max = max_over_ranks([total_ms, e2e_ms or 0.0], device)
        e2e_ms = e2e_max if e2e_ms is not None else None

    ms_per_step = total_ms / args.steps
    units_step, unit_scale, unit = step.units()
    value = job_throughput(world, units_step, args.steps, total_ms) * 1e12 / unit_scale

    kernels = {}
    dominant = None
    # A kernel timed inside a long run of back-to-back steps works under the
    # power cap: its roofline is the sustained matmul peak, not the burst one.
    long_run = total_ms >= LONG_RUN_MS
    tensor_peak = (peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) if long_run
                   else peaks["bf16_tflops"])
    tensor_peak_kind = ("bf16 dense sustained" if long_run else "bf16 dense burst")
    for (name, _, u), times in zip(step.ops, per_op):
        wo = wmap[u["workload"]]
        ms = statistics.median(times)
        entry = {"ms": round(ms, 4), "ms_mean": round(statistics.mean(times), 4)}
        if name.startswith("sfa_prefill"):
            # expanded tokens processed per second by this layer: B * n * L / t
            entry["expanded_tokens_per_s"] = round(wo.B * wo.n * wo.L / (ms * 1e-3), 1)
        if "flops" in u and u["flops"]:
            entry["tflops"] = round(u["flops"] / (ms * 1e-3) / 1e12, 2)
        if "bytes" in u:
            gbs = u["bytes"] / (ms * 1e-3) / 1e9
            entry["gbs"] = round(gbs, 1)
            entry["frac_hbm"] = round(gbs / peaks["hbm_gbs"], 4)
            entry["frac_hbm_nominal_8tbs"] = round(gbs / NOMINAL_HBM_GBS, 4)
        if name.startswith("sfa_prefill"):
            entry["frac_bf16_burst"] = round(entry["tflops"] / peaks["bf16_tflops"], 4)
            entry["frac_bf16_sustained"] = round(
                entry["tflops"] / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4)
        dram = measured_traffic(kernel_file_of(name), u["workload"] + ":" + u.get("mode", ""))
        if dram is not None:
            entry["dram_bytes_ncu"] = dram
        kernels[name] = entry
        if dominant is None or ms > kernels[dominant]["ms"]:
            dominant = name

    du = next(u for (nm, _, u) in step.ops if nm == dominant)
    dms = kernels[dominant]["ms_mean"]  # the roofline uses the average launch duration
    traffic_key = du["workload"] + ":" + du.get("mode", "")
    if "flops" in du and dominant.startswith("sfa_prefill"):
        achieved = du["flops"] / (dms * 1e-3) / 1e12
        roof = {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 2),
                "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": round(achieved / tensor_peak, 4),
                "peak_kind": f"{tensor_peak_kind}, {peak_kind}",
                "frac_burst": round(achieved / peaks["bf16_tflops"], 4),
                "timed_region_ms": round(total_ms, 1),
                "traffic": measured_traffic(kernel_file_of(dominant), traffic_key)}
    else:
        achieved = du["bytes"] / (dms * 1e-3) / 1e9
        roof = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_kind": f"HBM copy, {peak_kind}",
                "traffic": measured_traffic(kernel_file_of(dominant), traffic_key)}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {**config,
                   "step": [name for name, _, _ in step.ops],
                   "l2": "inputs larger than L2 (separate Q/K/V per layer; tables and "
                         "cache > L2); no flush",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": step.launches_per_step() * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    if e2e_ms is not None:
        line["e2e"] = {"value": round(job_throughput(world, units_step, e2e_steps, e2e_ms)
                                      * 1e12 / unit_scale, 2),
                       "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": round(e2e_ms / e2e_steps, 3),
                       "note": "inputs from pinned host memory and outputs back every step; two "
                               "buffer sets, copies on their own streams overlap compute"}
    within = [(fn, u) for (nm, fn, u) in step.ops if nm.startswith("sfa_prefill_fwd[within]")]
    within_ratio = None
    if within and wmap[within[0][1]["workload"]].n > 1:
        ww = wmap[within[0][1]["workload"]]
        t_within, t_plain = within_vs_plain_ms(ww, device, within[0][0])
        within_ratio = round(t_within / (ww.n * t_plain), 4)
        line["within_vs_n_plain"] = {
            "workload": ww.name, "plain_causal_ms": round(t_plain, 4),
            "within_ms": round(t_within, 4), "ratio": within_ratio,
            "note": "within-stream layer time / (n x plain causal n=1 time at the same L, B, "
                    "heads), timed alternately in one loop"}
    line["targets"] = targets_summary(kernels, within_ratio, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cunit, cores, desc = cpu_baseline(wmap[du["workload"]])
        line["cpu_baseline"] = {"value": v, "unit": cunit, "cores": cores, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
