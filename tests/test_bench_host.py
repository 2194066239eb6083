"""Host logic of bench.py, on CPU: which kernel's sources a workload's
profile is tied to, the algorithmic bytes each roofline divides by (counted
here tensor by tensor from the workload's shapes), the rule that a recorded
DRAM figure is reported only while its source hash still matches, the
roofline arithmetic of one timed workload, and the reference arm's line."""
import pytest
import torch

import bench
from gated_delta_rule_93_b200.inputs import WORKLOADS


@pytest.mark.parametrize("name,launches,kind", [
    ("tiny_fp32", 1, "split"),
    ("gdn_b8_t4096_h16_d128", 1, "chunk"),
    ("gdn_b1_t65536_h16_d128", 4, "seg"),
    ("kda_b8_t4096_h16_d128", 1, "chunk"),
    ("gla_b8_t4096_h16_d128", 1, "chunk"),
    ("gdn_prologue_b8_t4096_h16_d128", 1, "chunk"),
    ("decode_n256_h16_d128_x1024", 1, "step"),
    ("gdn_bwd_b8_t4096_h16_d128", 3, "bwd"),
    ("dplr_b8_t4096_h16_d128", 1, "dplr"),
])
def test_kernel_kind_of_each_workload(name, launches, kind):
    assert bench.kernel_kind(WORKLOADS[name], launches) == kind
    assert kind in bench.KERNEL_SOURCES


def _nbytes(shape, dtype):
    n = 1
    for s in shape:
        n *= s
    return n * torch.empty((), dtype=dtype).element_size()


def test_algorithmic_bytes_of_the_350m_forward():
    """q, k, v bf16 in, g and beta fp32 in, o bf16 out, S_T fp32 out; no S0."""
    B, T, H, d = 8, 4096, 16, 128
    bf, f = torch.bfloat16, torch.float32
    expect = (3 * _nbytes((B, T, H, d), bf) + 2 * _nbytes((B, T, H), f)
              + _nbytes((B, T, H, d), bf) + _nbytes((B, H, d, d), f))
    assert expect == 549453824
    assert bench.algorithmic_bytes(WORKLOADS["gdn_b8_t4096_h16_d128"]) == expect


def test_algorithmic_bytes_of_the_per_channel_and_gla_forwards():
    B, T, H, d = 8, 4096, 16, 128
    bf, f = torch.bfloat16, torch.float32
    qkvo = 4 * _nbytes((B, T, H, d), bf)
    ST = _nbytes((B, H, d, d), f)
    kda = WORKLOADS["kda_b8_t4096_h16_d128"]
    assert bench.algorithmic_bytes(kda) == (qkvo + _nbytes((B, T, H, d), f)
                                            + _nbytes((B, T, H), f)
                                            + ST * (int(kda.with_S0) + int(kda.want_S_T)))
    gla = WORKLOADS["gla_b8_t4096_h16_d128"]  # no beta
    assert bench.algorithmic_bytes(gla) == (qkvo + _nbytes((B, T, H), f)
                                            + ST * (int(gla.with_S0) + int(gla.want_S_T)))


def test_algorithmic_bytes_of_the_decode_step():
    """One step per (b, h): the fp32 state read and written, q, k, v and o
    bf16, g and beta fp32."""
    w = WORKLOADS["decode_n256_h16_d128_x1024"]
    N, H, d = 256, 16, 128
    per = 2 * _nbytes((d, d), torch.float32) + 4 * _nbytes((d,), torch.bfloat16) + 4 + 4
    assert bench.algorithmic_bytes(w) == N * H * per


def test_recorded_traffic_needs_a_matching_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.txt").write_text(
        "# workload bytes hash\n"
        "wl_a 1000 aaaa\n"
        "wl_b 2000 bbbb\n"
        "# wl_c 3000 aaaa\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind="chunk": "aaaa")
    assert bench.recorded_traffic("wl_a") == 1000.0
    assert bench.recorded_traffic("wl_b") is None   # taken on other sources
    assert bench.recorded_traffic("wl_c") is None   # a comment line
    assert bench.recorded_traffic("wl_d") is None   # never captured


def test_roofline_fields_arithmetic(monkeypatch):
    w = WORKLOADS["gdn_b8_t4096_h16_d128"]
    monkeypatch.setattr(bench, "measured_peaks", lambda: (6000.0, 1500.0, "measured"))
    monkeypatch.setattr(bench, "recorded_traffic", lambda *a, **k: None)
    steps, per_launch = 4, [0.20, 0.22, 0.21, 0.21]
    total = 0.90
    f = bench.roofline_fields(w, total, per_launch, steps, 1, None)
    abytes = bench.algorithmic_bytes(w)
    achieved = abytes / (0.21e-3) / 1e9
    assert f["roofline"]["bound"] == "hbm"
    assert f["roofline"]["achieved"] == pytest.approx(achieved)
    assert f["roofline"]["frac"] == pytest.approx(achieved / 6000.0)
    assert f["ms_per_step"] == pytest.approx(total / steps)
    assert f["value"] == pytest.approx(w.B * w.T * steps / (total / 1e3))
    # two ranks: the whole job's tokens over the (max-over-ranks) time
    f2 = bench.roofline_fields(w, total, per_launch, steps, 2, None)
    assert f2["value"] == pytest.approx(2 * f["value"])


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` times the oracle on the host and prints the
    contract's line: impl, cpu_baseline, a zero-copy e2e and no GPU launch."""
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, bench.__file__, "--impl", "reference", "--workload",
                        "tiny_fp32", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["gpu_launches"] == 0
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["warmup"] >= 3 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny_fp32"
