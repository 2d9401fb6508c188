"""Host logic of bench.py (no GPU): the reference arm's JSON line, the DRAM-traffic record's
staleness check and the clock sampler's parsing."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT,
                         env={**os.environ, "RANK": "0", "WORLD_SIZE": "1"})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "keys/s"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == bench.WORKLOAD


def test_reference_arm_is_silent_off_rank_zero():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT,
                         env={**os.environ, "RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [l for l in out.stdout.splitlines() if l.startswith("{")]


def test_traffic_record_is_used_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["stream_score_kernel"]
    got = bench.traffic_for("stream_score_kernel", 1000)
    fresh = bench.sources_sha256_16(rec["sources"]) == rec["sources_sha256_16"]
    assert (got == pytest.approx(rec["dram_bytes_per_unit"] * 1000)) if fresh else got is None
    # a record whose hash does not match the sources is ignored
    prof = tmp_path / "profiles"
    prof.mkdir()
    bad = dict(rec, sources_sha256_16="0" * 16)
    (prof / "traffic.json").write_text(json.dumps({"stream_score_kernel": bad}))
    for rel in rec["sources"]:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(ROOT, rel), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("stream_score_kernel", 1000) is None
    assert bench.traffic_for("no_such_kernel", 1000) is None


def test_clock_sampler_parses_reasons():
    cs = bench.ClockSampler(0)
    cs.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    cs.lines = ["0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
                "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
                "garbage"]
    import time as _time
    orig = _time.sleep
    _time.sleep = lambda s: None
    try:
        r = cs.stop()
    finally:
        _time.sleep = orig
    assert r["sm_max_mhz"] == 1965.0 and r["samples"] == 2
    assert r["sm_mhz"] == pytest.approx((1965 + 1800) / 2)
    assert r["reasons"] == ["sw_power_cap"]


@pytest.mark.parametrize("kind", ["prefill", "latent", "latent192", "hs_b1", "sparse_attention"])
def test_oracle_samples_run_on_small_cases(kind):
    # each workload's cpu_baseline: the oracle timed on a bounded sample of that workload's input
    import numpy as np
    import torch
    from sparse_attention_lightning_score_b200 import synth
    if kind == "prefill":
        case = synth.dsa_prefill(T=300, L=300)
    elif kind == "latent":
        case = synth.latent_group(B=2, L=3000, G=2)
    elif kind == "latent192":
        case = synth.latent_rope_nope(B=2, L=3000, G=2)
    elif kind == "hs_b1":
        case = synth.latent_hs(B=1, L=3000, n_cand=512, k_top=128)
    else:
        g = torch.Generator().manual_seed(0)
        q = torch.randn(2, 64, 576, generator=g).to(torch.bfloat16)
        kv = torch.randn(2, 700, 576, generator=g).to(torch.bfloat16)
        sel = np.stack([np.sort(np.random.default_rng(b).choice(700, 256, replace=False)) for b in range(2)])
        case = (q, kv, sel.astype(np.int32), 0.05)
    r = bench.oracle_sample(kind, case, budget_s=0.2)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1 and r["sample"]
