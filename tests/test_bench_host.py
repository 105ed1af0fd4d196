"""Host-side checks of bench.py (no GPU): the algorithmic byte and FLOP counts against the
scope table's closed forms, the attainable-roofline fraction, the staleness rule of the recorded
ncu traffic, and the reference arm's JSON line (the fp64 oracle on a small sample)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_forward_bytes_and_flops_per_token_head():
    # bf16 q, k, v (768 B) + a bf16 o (256 B) + eta, g (8 B) = 1032 B per token-head
    assert bench.fwd_bytes(1, 1, 1, 128, 128, 2, False, s_out=False, out_elt=2) == 1032
    # the fp32 o the headline call writes: 256 B more
    assert bench.fwd_bytes(1, 1, 1, 128, 128, 2, False, s_out=False) == 1288
    # S0 read and S_T write at 64 KiB each per (b, h)
    assert bench.fwd_bytes(2, 10, 3, 128, 128, 2, True) == 2 * 10 * 3 * 1288 + 2 * 3 * 2 * 65536
    # 10 C d + 6 d^2 + (2/3) C^2 at C = 64
    assert round(bench.fwd_flops_per_token_head(128)) == 182955
    assert round(bench.fwd_flops_per_token_head(64)) == 68267


def test_decode_bytes_per_head_step():
    # the fp32 state read and written, q, k, v and o in bf16, eta and g
    assert bench.decode_bytes(1, 1, 128, 128, 2, out_elt=2) == 132104


def test_attainable_roofline_is_the_slower_floor():
    a = bench.attainable(1.6318e12, 6.5408e9, 1631.8, 6540.8, 2e-3)  # both floors 1 ms
    assert a["t_tensor_us"] == pytest.approx(1000.0) and a["t_hbm_us"] == pytest.approx(1000.0)
    assert a["frac"] == pytest.approx(0.5)
    a = bench.attainable(2.398e10, 1.73e8, 1631.8, 6540.8, 148.8e-6)  # the headline call
    assert a["bound"] == "hbm" and a["frac"] == pytest.approx(1.73e8 / 6540.8e9 / 148.8e-6)
    a = bench.attainable(1e13, 1e6, 1631.8, 6540.8, 10e-3)
    assert a["bound"] == "tensor" and a["frac"] == pytest.approx(1e13 / 1631.8e12 / 10e-3)


def test_recorded_traffic_is_null_once_a_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "gated_delta_rule_kla_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash(["k.cu"])
    (prof / "traffic.json").write_text(json.dumps(
        {"w": {"dram_bytes_per_launch": 123.0, "sources": ["k.cu"], "source_hash": h}}))
    assert bench.recorded_traffic("w") == 123.0
    assert bench.recorded_traffic("missing") is None
    (src / "k.cu").write_text("kernel v2\n")
    assert bench.recorded_traffic("w") is None


def test_committed_traffic_matches_the_sources():
    """Every entry of profiles/traffic.json was taken on the sources as committed."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for key, e in d.items():
        if isinstance(e, dict) and "sources" in e:
            assert e["source_hash"] == bench.kernel_source_hash(e["sources"]), key


def test_reference_arm_line():
    """The reference arm times the fp64 oracle on the host cores and prints the contract's line."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-pairs", "1"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "prefill_b8_t2048_h8_d128"
