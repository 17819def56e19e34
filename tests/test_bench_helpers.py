"""Host-side helpers of bench.py (no GPU): the DRAM-traffic figure is reported only while the kernel
sources still hash to the captured ones, the oracle's decode baseline extrapolates steps/s of the
whole workload from a sample of (sequence, head) slices, and the other workloads' oracle samples and
roofline figures are built as stated."""
import os
import shutil
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _source_hash(root):
    import hashlib
    d = hashlib.sha256()
    for f in ("kda_chunk_bf16.cu", "kda_device.cuh"):
        with open(os.path.join(root, "kda_linear_attention_02_b200", "csrc", f), "rb") as fh:
            d.update(fh.read())
    return d.hexdigest()[:16]


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # a copy of the tree with a traffic record keyed to its kernel sources reports the figures
    fake = tmp_path / "root"
    (fake / "profiles").mkdir(parents=True)
    csrc = fake / "kda_linear_attention_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("kda_chunk_bf16.cu", "kda_device.cuh"):
        shutil.copy(os.path.join(ROOT, "kda_linear_attention_02_b200", "csrc", f), csrc / f)
    h = _source_hash(str(fake))
    (fake / "profiles" / "traffic.txt").write_text(
        "# kernel bytes_per_launch source_sha256_16\n"
        f"prep_bf16_kernel 1000 {h}\nstate_bf16_kernel 2000 {h}\nold_kernel 3000 0123456789abcdef\n")
    monkeypatch.setattr(bench, "ROOT", str(fake))
    assert bench.captured_traffic("prep_bf16_kernel") == 1000
    assert bench.captured_traffic("state_bf16_kernel") == 2000
    assert bench.captured_traffic("old_kernel") is None          # captured from other sources
    assert bench.captured_traffic("no_such_kernel") is None
    # one byte more in a kernel source: nothing is reported
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


def test_workload_oracle_baseline_and_roofline():
    from kda_linear_attention_02_b200 import synth
    inp = synth.make_inputs([300, 130], 4, 32, 32, dtype=torch.bfloat16, device="cpu", seed=3, with_state0=True)
    jobs = bench.host_slices(inp, [(0, 1), (1, 3)], ckpt=64, tok_limit=200)
    assert [j[1]["q"].shape[0] for j in jobs] == [200, 130]
    assert jobs[0][1]["marks"] == [64, 128, 192] and jobs[1][1]["marks"] == [64, 128]
    assert jobs[1][1]["s0"].shape == (32, 32)
    r = bench.cpu_oracle_jobs(jobs, 4, 430 * 4, "test")
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["value"] > 0
    assert "330 token-heads of 1720" in r["sample"]
    rl = bench.prefill_roofline(1000, 2.0, 5000.0, extra_bytes=460)
    assert rl["alg_bytes_per_launch"] == 1540 * 1000 + 460
    assert abs(rl["achieved"] - 1540460 / 2e-3 / 1e9) < 0.1 and rl["bound"] == "hbm"
