"""Host-side arithmetic of bench.py's JSON line (CPU, no kernel runs): the
roofline object of the dominant kernel, the per-stage rates, and the rule that a
DRAM-traffic record is reported only while the kernel's source is unchanged."""
import importlib.util
import json
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _FakeTg:
    def __init__(self, kernel):
        self.kernel = kernel

    def attention_kernel(self, cu_kept, hq, hkv, dh, dtype, with_workspace):
        return self.kernel + " (plan)"


class _FakeLayer:
    def __init__(self, work):
        self._work = work
        self.cu_kept_host = np.array([0, 2304], np.int32)
        self.workspace = None

    def work(self):
        return dict(self._work)


# per-launch work of the 16k layer: flops and bytes as the layer reports them
WORK = dict(gate_flops=16384 * 2.0 * 2048 * 256, gate_bytes=68763904.0, topk_bytes=74000.0,
            gather_bytes=2 * 2304 * 12288.0 + 12 * 2304, attn_flops=2.0 * 128 * 16 * 2304 * 2305)
PK = dict(hbm=6543.4, bf16=1651.8, bf16_sustained=1393.4, source="measured")


def _workload(dtype="bf16"):
    from learned_token_pruning_gate_b200 import inputs as gen
    w = gen.WORKLOADS["qwen_16k"]
    return w if dtype == "bf16" else gen.WORKLOADS["tiny_fp32"]


def test_attention_dominant_roofline(bench):
    ms = dict(gate=0.0269, topk=0.0143, gather=0.0225, attention=0.0419)
    stages, roof = bench._stages_and_roofline(_FakeTg("attn_pair_kernel"), _FakeLayer(WORK),
                                              _workload(), "no_such_workload", ms, PK)
    tflops = WORK["attn_flops"] / 41.9 / 1e6  # flop per µs -> TFLOP/s
    assert roof["kernel"] == "attn_pair_kernel" and roof["bound"] == "tensor"
    assert roof["unit"] == "TFLOP/s" and roof["peak"] == PK["bf16"]
    assert roof["achieved"] == pytest.approx(tflops, rel=1e-12)
    assert roof["frac"] == pytest.approx(tflops / PK["bf16"], rel=1e-12)
    assert roof["traffic"] is None  # no record for this workload
    assert stages["attention"]["kernel"] == "attn_pair_kernel"
    assert stages["gather"]["gbs"] == pytest.approx(WORK["gather_bytes"] / 22.5 / 1e3)
    assert stages["gather"]["frac_hbm"] == pytest.approx(stages["gather"]["gbs"] / PK["hbm"])
    tg_us = 14.3 + 22.5
    assert stages["topk+gather"]["us"] == pytest.approx(tg_us)
    assert stages["topk+gather"]["gbs"] == pytest.approx(
        (WORK["topk_bytes"] + WORK["gather_bytes"]) / tg_us / 1e3)
    assert stages["gate"]["tflops"] == pytest.approx(WORK["gate_flops"] / 26.9 / 1e6)


def test_gate_dominant_roofline_picks_the_binding_resource(bench):
    ms = dict(gate=0.05, topk=0.01, gather=0.01, attention=0.02)
    # the 16k gate moves 4 KB per token for 1 Mflop: flops and bytes take about
    # the same time at the measured peaks, so the larger of the two decides
    t_flop = WORK["gate_flops"] / (PK["bf16"] * 1e12)
    t_byte = WORK["gate_bytes"] / (PK["hbm"] * 1e9)
    _, roof = bench._stages_and_roofline(_FakeTg("attn_pair_kernel"), _FakeLayer(WORK), _workload(),
                                         "no_such_workload", ms, PK)
    assert roof["kernel"] == "gate_tc2_kernel"
    if t_flop >= t_byte:
        assert roof["bound"] == "tensor" and roof["achieved"] == pytest.approx(WORK["gate_flops"] / 50 / 1e6)
    else:
        assert roof["bound"] == "hbm" and roof["achieved"] == pytest.approx(WORK["gate_bytes"] / 50 / 1e3)
    # a gate with four times the bytes per flop is HBM-bound
    heavy = dict(WORK, gate_bytes=WORK["gate_bytes"] * 4)
    _, roof = bench._stages_and_roofline(_FakeTg("attn_pair_kernel"), _FakeLayer(heavy), _workload(),
                                         "no_such_workload", ms, PK)
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["peak"] == PK["hbm"]


def test_fp32_attention_is_reported_against_the_fp32_alu_peak(bench):
    ms = dict(gate=0.01, topk=0.01, gather=0.01, attention=0.09)
    _, roof = bench._stages_and_roofline(_FakeTg("attn_simt_kernel"), _FakeLayer(WORK),
                                         _workload("fp32"), "no_such_workload", ms, PK)
    assert roof["bound"] == "alu" and roof["peak"] == pytest.approx(bench.FP32_FMA_TFLOPS)
    assert roof["peak"] == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def test_traffic_record_only_while_the_source_is_unchanged(bench, tmp_path, monkeypatch):
    csrc = tmp_path / "learned_token_pruning_gate_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_text("__global__ void k() {}\n")
    sha = bench._sha(str(src))
    rec = {"k_kernel": {"wl": {"source": "k.cu", "sha256": sha, "bytes_per_launch": 1234}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k_kernel", "wl") == 1234
    assert bench._traffic("k_kernel", "other") is None
    assert bench._traffic("other_kernel", "wl") is None
    src.write_text("__global__ void k() { /* changed */ }\n")
    assert bench._traffic("k_kernel", "wl") is None


def test_committed_traffic_records_name_existing_sources(bench):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    recs = json.load(open(path))
    for kernel, per in recs.items():
        for wl, rec in per.items():
            assert os.path.exists(os.path.join(ROOT, "learned_token_pruning_gate_b200", "csrc",
                                               rec["source"])), (kernel, wl)
            assert rec["bytes_per_launch"] == rec["read"] + rec["write"], (kernel, wl)
            assert len(rec["sha256"]) == 16


def _run_bench(args, env_extra=None, timeout=300):
    import subprocess
    import sys
    env = dict(os.environ, **(env_extra or {}))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=timeout)
    assert p.returncode == 0, p.stderr[-2000:]
    return [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    # the oracle on the host cores: one bounded sample per step, no device
    (line,) = _run_bench(["--impl", "reference", "--workload", "tiny_fp32", "--steps", "1",
                          "--warmup", "0"])
    assert line["impl"] == "reference" and line["metric"] == "gated-prefill input tok/s"
    assert line["unit"] == "tok/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["dtype"] == "f64" and line["vs_baseline"] is None
    assert line["config"]["workload"] == "tiny_fp32"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    assert _run_bench(["--impl", "reference", "--workload", "tiny_fp32", "--steps", "1",
                       "--warmup", "0"], env_extra={"RANK": "1", "WORLD_SIZE": "2"}) == []
