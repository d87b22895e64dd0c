"""Host-side pieces of bench.py, checked on the CPU.

The timed GPU arm needs a B200; these tests cover what the JSON line is
built from without one: the workload description, the DRAM-traffic lookup
keyed by the fused kernel's source hash, the clock-sample parsing (and its
throttle-reason flags), and the oracle reference arm's line.
"""

import io
import json
import shutil
from contextlib import redirect_stdout
from types import SimpleNamespace

import bench
from synth import WORKLOADS


def test_workload_config_names_sizes_and_pairs():
    c = bench.workload_config(WORKLOADS["causal_16k_h64"])
    assert c["workload"] == "causal_16k_h64" and c["H"] == 64 and c["d"] == 128 and c["topk"] == 2048
    assert c["pairs_per_step"] == 16384 * 16385 // 2
    d = bench.workload_config(WORKLOADS["decode_64x128k_h64"])
    assert d["B"] == 64 and d["t_cap"] == 131072 and d["pairs_per_step"] == 64 * 131072


def test_traffic_lookup_follows_the_fused_kernel_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "sparse_attention_token_03_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.SCORE_KERNEL_SOURCES:
        shutil.copy(bench.ROOT / "sparse_attention_token_03_b200" / "csrc" / name, csrc / name)
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    h = bench.kernel_source_hash()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.txt").write_text(
        "# comment\n"
        f"causal_16k_h64  score_topk_kernel  {h}  123456   # summary\n"
        "chunk_1m_h64  score_topk_kernel  0000000000000000  999   # older capture\n")
    assert bench.recorded_traffic("causal_16k_h64", "score_topk_kernel") == 123456.0
    assert bench.recorded_traffic("chunk_1m_h64", "score_topk_kernel") is None  # stale hash
    assert bench.recorded_traffic("causal_16k_h64", "screen") is None
    # editing a file outside the fused kernel's sources keeps the record valid
    (csrc / "dsa_select.cu").write_text("// unrelated\n")
    assert bench.recorded_traffic("causal_16k_h64", "score_topk_kernel") == 123456.0
    # editing one of them voids it
    with open(csrc / "dsa_score.cu", "a") as f:
        f.write("\n// edit\n")
    assert bench.recorded_traffic("causal_16k_h64", "score_topk_kernel") is None


class _FakeSmi:
    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, ""


def test_clock_samples_median_and_throttle_reasons():
    lines = [
        "2026/12/02 10:00:00.000, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:00.100, 1950, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:00.200, 1965, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.proc = _FakeSmi("\n".join(lines))
    r = cs.stop()
    assert r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"]
    cs.proc = _FakeSmi(lines[0].replace("Not Active, Not Active, Not Active, Not Active",
                                        "Active, Not Active, Active, Not Active"))
    assert cs.stop()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    cs.proc = None
    assert cs.stop()["reasons"] == ["nvidia-smi unavailable"]


def test_reference_arm_prints_one_line_with_the_contract_keys(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    args = SimpleNamespace(steps=1, warmup=0, gpus=1, impl="reference", workload="causal_1k_h64")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, WORKLOADS["causal_1k_h64"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "pairs/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["config"]["workload"] == "causal_1k_h64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    # other ranks print nothing
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, WORKLOADS["causal_1k_h64"])
    assert buf.getvalue() == ""
