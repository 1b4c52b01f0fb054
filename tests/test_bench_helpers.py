"""Host-side arithmetic of bench.py (no GPU): the roofline helpers and the
traffic-record lookup."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_sfu_roofline_is_one_at_the_exponential_peak(bench):
    # 16 results per clock per SM, 148 SMs, 1965 MHz, for exactly 1 ms
    n_exp = 16 * 148 * 1965 * 1000
    r = bench.sfu_roofline(n_exp, 1.0, 148, 1965.0)
    assert r["bound"] == "sfu" and r["unit"] == "exp/s"
    assert r["peak"] == pytest.approx(16 * 148 * 1965e6)
    assert r["frac"] == pytest.approx(1.0)


def test_sfu_roofline_of_the_sd_latent_broadcast(bench):
    # B*H*N*k exponentials: 2*8*16384*256; half the peak rate takes twice the time
    n_exp = 2 * 8 * 16384 * 256
    t_peak_ms = n_exp / (16 * 148 * 1965e6) * 1e3
    r = bench.sfu_roofline(n_exp, 2 * t_peak_ms, 148, 1965.0)
    assert r["frac"] == pytest.approx(0.5)
    assert r["exps_per_launch"] == n_exp


def test_traffic_record_applies_only_to_the_recorded_sources(bench, tmp_path, monkeypatch):
    shas = {k: bench.kernel_source_sha(k) for k in bench.ROOFLINE_SOURCES}
    assert all(len(v) == 16 for v in shas.values())
    # the broadcast's sources are a subset of the others': different hashes
    assert len(set(shas.values())) == len(shas)
    assert bench.recorded_traffic("agent_broadcast", "no_such_workload") is None
    assert bench.recorded_traffic("no_such_kernel", "sd_latent_1024") is None
    # a record applies only while its kernel's sources hash the same
    prof = tmp_path / "profiles"
    prof.mkdir()
    import json
    recs = {"records": [
        {"kernel": "agent_broadcast", "workload": "w", "source_sha": shas["agent_broadcast"],
         "dram_bytes_per_launch": 123},
        {"kernel": "agent_fused_small", "workload": "w", "source_sha": "0" * 16,
         "dram_bytes_per_launch": 456}]}
    (prof / "ncu_traffic.json").write_text(json.dumps(recs))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "efficient_vision_attention_b200" / "csrc"
    csrc.parent.mkdir()
    import shutil, os
    shutil.copytree(os.path.join(os.path.dirname(os.path.dirname(__file__)),
                                 "efficient_vision_attention_b200", "csrc"), csrc)
    assert bench.recorded_traffic("agent_broadcast", "w") == 123
    assert bench.recorded_traffic("agent_fused_small", "w") is None
