"""Host-side helpers of bench.py (no GPU): the DRAM-traffic figure is reported only while the kernel
sources still hash to the captured ones, and the oracle's decode baseline extrapolates steps/s of the
whole workload from a sample of (sequence, head) slices."""
import os
import shutil
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # the committed figures match the committed sources
    assert isinstance(bench.captured_traffic("prep_bf16_kernel"), int)
    assert bench.captured_traffic("no_such_kernel") is None
    # a copy of the tree whose kernel source differs by one byte reports nothing
    fake = tmp_path / "root"
    (fake / "profiles").mkdir(parents=True)
    csrc = fake / "kda_linear_attention_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    shutil.copy(os.path.join(ROOT, "profiles", "traffic.txt"), fake / "profiles" / "traffic.txt")
    for f in ("kda_chunk_bf16.cu", "kda_device.cuh"):
        shutil.copy(os.path.join(ROOT, "kda_linear_attention_02_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(fake))
    assert isinstance(bench.captured_traffic("prep_bf16_kernel"), int)     # identical copy: still reported
    assert isinstance(bench.captured_traffic("state_bf16_kernel"), int)
    with open(csrc / "kda_device.cuh", "a") as fh:
        fh.write("\n")
    assert bench.captured_traffic("prep_bf16_kernel") is None
    assert bench.captured_traffic("state_bf16_kernel") is None


def test_decode_oracle_baseline_samples_and_extrapolates():
    from kda_linear_attention_02_b200 import synth
    n, H, d, steps = 6, 4, 32, 20
    s0, q, k, v, la, b = synth.make_decode_inputs(n, H, d, d, dtype=torch.bfloat16, device="cpu", seed=5,
                                                  steps=steps)
    r = bench.cpu_oracle_decode_sample(s0, q, k, v, la, b, budget_s=5.0, max_slices=7)
    assert r["kind"] == "oracle" and r["unit"] == "steps/s" and r["cores"] >= 1
    assert r["sample"].startswith(f"7 of {n * H} (sequence, head) slices x {steps} steps")
    assert r["value"] > 0
