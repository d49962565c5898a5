"""Host-side logic that needs no GPU: the seeded input generators, the bench's traffic
lookup and its reference arm (the oracle timed on host cores)."""
import importlib.util
import json
import os
import subprocess
import sys

import torch

from gated_delta_rule_155_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_module():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_packed_lengths_follow_their_law():
    lens = inputs.packed_lengths(32768, 4096, 5)
    assert sum(lens) == 32768 and all(1 <= n <= 4096 for n in lens)
    assert lens == inputs.packed_lengths(32768, 4096, 5)          # seeded
    assert lens != inputs.packed_lengths(32768, 4096, 6)
    assert inputs.packed_lengths(10, 4096, 5) == [10]              # the last draw is trimmed


def test_varlen_inputs_layout():
    lens = [3, 0, 5]
    d = inputs.varlen_inputs(lens, 2, 64, 64, io="f32", seed=1, s0_std=0.1)
    assert d["q"].shape == (8, 2, 64) and d["v"].shape == (8, 2, 64) and d["beta"].shape == (8, 2)
    assert d["cu_seqlens"].dtype == torch.int32 and d["cu_seqlens"].tolist() == [0, 3, 3, 8]
    assert d["s0"].shape == (3, 2, 64, 64)
    assert inputs.varlen_inputs(lens, 2, 64, 64, io="f32", seed=1)["s0"] is None


def test_prefill_inputs_are_seeded_and_follow_the_laws():
    a = inputs.prefill_inputs(2, 33, 3, 64, 64, io="f32", seed=7, s0_std=0.02)
    b = inputs.prefill_inputs(2, 33, 3, 64, 64, io="f32", seed=7, s0_std=0.02)
    for n in ("q", "k", "v", "g", "beta", "s0"):
        assert torch.equal(a[n], b[n]), n
    qn = a["q"].double().norm(dim=-1)
    assert torch.allclose(qn, torch.ones_like(qn), atol=1e-6)      # unit rows
    assert bool((a["g"] <= 0).all()) and bool(((a["beta"] > 0) & (a["beta"] < 1)).all())
    c = inputs.prefill_inputs(2, 33, 3, 64, 64, io="bf16", seed=7)
    assert c["q"].dtype == torch.bfloat16
    # bf16 inputs are the fp32 draws rounded once
    assert torch.equal(c["v"], a["v"].to(torch.bfloat16))


def test_traffic_lookup_requires_the_captured_sources(monkeypatch, tmp_path):
    bench = _bench_module()
    sha = bench.kernel_source_sha()
    assert sha == bench.kernel_source_sha() and len(sha) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({
        "k_same": {"source_sha": sha, "dram_bytes_per_launch": 123},
        "k_old": {"source_sha": "0" * 16, "dram_bytes_per_launch": 456}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda kernel=None: sha)
    assert bench.traffic_for("k_same") == 123
    assert bench.traffic_for("k_old") is None        # kernel changed since the capture
    assert bench.traffic_for("missing") is None


def test_each_profiled_kernel_hashes_its_own_sources():
    bench = _bench_module()
    for k, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "gated_delta_rule_155_b200", "csrc", f)), (k, f)
    # the prefill and the backward are compiled from different files, so their hashes differ
    assert bench.kernel_source_sha("kda_chunk_tc") != bench.kernel_source_sha("kda_backward")
    assert bench.kernel_source_sha("kda_chunk_tc") == bench.kernel_source_sha("kda_chunk_tc_packed")


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` times the oracle on the host and prints the contract's line."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
