"""bench.py on the host: the reference arm's JSON line carries the contract's
keys, ranks other than 0 print nothing, and each kind of oracle CPU baseline
(prefill rows, training-side gradient, backward) runs and reports a rate."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from sequence_expanded_attention_b200 import workloads as wl  # noqa: E402


def _run(argv, monkeypatch, rank="0"):
    monkeypatch.setenv("RANK", rank)
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr(bench, "cpu_baseline",
                        lambda w, target_s=12.0: (0.01, "TFLOP/s", 4, "stub sample"))
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(argv)
    return buf.getvalue()


def test_reference_line_has_the_contract_keys(monkeypatch):
    out = _run(["--impl", "reference", "--steps", "2", "--warmup", "3"], monkeypatch)
    lines = [line for line in out.splitlines() if line.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    # the default step's config names its parts: the MoE-shaped long prefill,
    # the 8.59 GB decode and the Qwen3-8B-shaped expansion
    assert d["config"]["workload"] == "moe_long_prefill+decode+qwen3_8b_prefill[gather]"
    assert set(d["config"]["parts"]) == {"moe_long_prefill", "decode",
                                         "qwen3_8b_prefill[gather]"}
    assert d["config"]["parts"]["decode"]["T"] == 8192
    assert set(d["cpu_baseline"]) >= {"value", "unit", "cores", "kind", "sample"}
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["ms_per_step"] is not None and d["ms_per_step"] >= 0  # one sample's wall time
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing(monkeypatch):
    assert _run(["--impl", "reference", "--steps", "1"], monkeypatch, rank="1").strip() == ""


def test_warmup_is_at_least_three(monkeypatch):
    d = json.loads(_run(["--impl", "reference", "--steps", "1", "--warmup", "1"],
                        monkeypatch).strip())
    assert d["warmup"] == 3


@pytest.mark.parametrize("name,unit", [("tiny", "TFLOP/s"), ("qwen3_8b_embed_train", "GB/s"),
                                       ("qwen3_8b_train_sfa", "TFLOP/s")])
def test_cpu_baseline_kinds(name, unit):
    v, u, cores, desc = bench.cpu_baseline(wl.WORKLOADS[name], target_s=0.2)
    assert v > 0 and u == unit and cores >= 1 and desc


@pytest.mark.parametrize("name,mode", [("qwen3_8b_prefill", "cross"),
                                       ("qwen3_8b_transient", "transient"),
                                       ("qwen3_8b_window", "cross_window")])
def test_cpu_baseline_samples_the_workloads_own_mask(name, mode):
    v, u, cores, desc = bench.cpu_baseline(wl.WORKLOADS[name], target_s=0.2)
    assert v > 0 and u == "TFLOP/s"
    assert f" {mode} prefill rows" in desc


def test_job_throughput_is_whole_job():
    # two ranks, 1e12 units each per step, 10 steps in 1000 ms -> 20 TFLOP/s for the job
    assert bench.job_throughput(2, 1e12, 10, 1000.0) == pytest.approx(20.0)


def test_reference_arm_single_workload(monkeypatch):
    d = json.loads(_run(["--impl", "reference", "--steps", "1", "--workload", "tiny"],
                        monkeypatch).strip())
    assert d["config"]["workload"] == "tiny" and d["config"]["parallelism"] == "host cores"


def test_headline_parts_are_the_largest_single_gpu_cases():
    parts = {name: wl.WORKLOADS[name] for name, _, _ in bench.HEADLINE_PARTS}
    pre = parts["moe_long_prefill"]
    assert (pre.n, pre.L, pre.B, pre.Hq, pre.Hkv, pre.D) == (4, 8192, 2, 64, 4, 128)
    dec = parts["decode"]
    assert dec.decode and (dec.B, dec.n, dec.L) == (64, 4, 8192)
    # the cache read per decode call: 8.59 GB of K and V
    assert wl.decode_bytes(dec.n, dec.L, dec.B, dec.Hq, dec.Hkv, dec.D) == pytest.approx(
        8.59e9, rel=2e-3)


def test_targets_summary_reads_the_bars():
    k = {"sfa_prefill_fwd[cross]#1@m": {"frac_bf16_burst": 0.65, "frac_bf16_sustained": 0.75},
         "sfa_decode_fwd[within]@d": {"frac_hbm": 0.9},
         "hd_expand_embed[uniform ids]@q": {"frac_hbm": 0.8}}
    t = bench.targets_summary(k, 0.97)
    assert t["prefill_frac_bf16_burst"] == {"bar": 0.60, "sfa_prefill_fwd[cross]": 0.65}
    assert t["prefill_frac_bf16_sustained"] == {"bar": 0.60, "sfa_prefill_fwd[cross]": 0.75}
    assert t["within_vs_n_plain"] == {"bar": 1.2, "ratio": 0.97}
    assert t["decode_frac_hbm"]["sfa_decode_fwd[within]"] == 0.9
    assert t["gather_frac_hbm"]["hd_expand_embed[uniform ids]"] == 0.8


def test_kernel_file_of_each_op():
    assert bench.kernel_file_of("sfa_prefill_fwd[cross]#1") == "k_sfa_prefill.cu"
    assert bench.kernel_file_of("sfa_prefill_bwd[cross]#1") == "k_sfa_backward.cu"
    assert bench.kernel_file_of("sfa_decode_fwd[within]") == "k_sfa_decode.cu"
    assert bench.kernel_file_of("hd_expand_embed[uniform ids]") == "k_expand_embed.cu"
    assert bench.kernel_file_of("hd_expand_embed_backward") == "k_train_embed.cu"
    assert bench.kernel_file_of("hd_final_stream_rows") == "k_train_embed.cu"
