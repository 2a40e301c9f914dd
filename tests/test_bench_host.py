"""Host-side logic of bench.py (CPU only): the algorithmic work it divides by, the reference
arm's sampling, the JSON line of the reference arm, and the use of the committed ncu traffic
record (keyed on the FC GEMM's code)."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_scaled_moe_softmax_b200 import workloads  # noqa: E402


def test_algorithmic_work_closed_forms():
    wl = workloads.WORKLOADS["decode"]
    counts = np.zeros(wl.E, np.int64)
    counts[[3, 7, 11]] = [5, 1, 10]            # 3 experts hit, 16 pairs
    b, hit = bench.fc1_algorithmic_bytes(wl, counts)
    assert hit == 3
    # MXFP4 gate+up rows (half a byte per element) and their E8M0 scales, plus bf16 rows in and out
    per_expert = 2 * wl.I * wl.H // 2 + 2 * wl.I * wl.H // 32
    assert b == 3 * per_expert + 16 * (wl.H + wl.I) * 2
    assert bench.fc1_algorithmic_flops(wl, counts) == 2.0 * 16 * 2 * wl.I * wl.H
    assert bench.layer_weight_bytes(wl, 3) == 3 * (3 * wl.I * wl.H // 2 + 3 * wl.I * wl.H // 32)
    assert per_expert == 15_597_568  # 15.60 MB per hit expert at H = 7168, I = 2048


def test_cpu_baseline_uses_every_core():
    wl = workloads.WORKLOADS["tiny"]
    cb = bench.cpu_baseline(wl, 4, min_wall=0.05)
    assert cb["kind"] == "oracle" and cb["cores"] == 4 and cb["threads"] == 4 and cb["value"] > 0
    assert "4 at a time" in cb["sample"]


def test_reference_pairs():
    wl = workloads.WORKLOADS["tiny"]
    pairs, per_token = bench.reference_pairs(wl, [0, 1, 2])
    assert per_token == wl.top_k and len(pairs) == 3 * wl.top_k
    assert all(0 <= e < wl.E for _, e, _ in pairs)
    for t in range(3):  # a token's routed weights sum to 1
        assert abs(sum(w for tt, _, w in pairs if tt == t) - 1.0) < 1e-6
    sh = workloads.Workload("sh", 16, 256, 128, 8, 2, shared=2)
    pairs, per_token = bench.reference_pairs(sh, [0])
    assert per_token == 4 and [(e, w) for _, e, w in pairs[2:]] == [(8, 1.0), (9, 1.0)]
    ep = workloads.WORKLOADS["situ_ep8"]
    pairs, per_token = bench.reference_pairs(ep, list(range(8)))
    ids, _ = workloads.draw_topk(ep)
    ids = ids.numpy()
    assert per_token == pytest.approx(((ids >= 0) & (ids < ep.E)).sum() / ep.T)
    assert len(pairs) == int(((ids[:8] >= 0) & (ids[:8] < ep.E)).sum())


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "6", "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["steps"] == 6 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["pairs_per_token"] == 2.0


def test_kernel_source_hash_ignores_comments_only():
    """The traffic record is keyed on the FC GEMM's code: an edit of a comment or of whitespace
    keeps the hash, an edit of the code changes it."""
    csrc = os.path.join(ROOT, "block_scaled_moe_softmax_b200", "csrc")

    def read(name):
        with open(os.path.join(csrc, name)) as f:
            return f.read()

    base = bench.kernel_source_sha(read)
    assert base == bench.kernel_source_sha()
    commented = lambda n: read(n) + ("\n// a new remark\n/* and a block\n   comment */\n   \n" if n == "fc_gemm.cu" else "")
    assert bench.kernel_source_sha(commented) == base
    changed = lambda n: read(n) + ("\nconstexpr int kProbe = 1;\n" if n == "ptx.cuh" else "")
    assert bench.kernel_source_sha(changed) != base


def test_traffic_record_use(monkeypatch):
    """A committed capture is used for its own workload and scaled by algorithmic bytes for the
    workloads it lists under scales_to; nothing is reported once the kernel's code differs."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    caps = {c["workload"]: c for c in rec["fc1_captures"]}
    monkeypatch.setattr(bench, "kernel_source_sha", lambda read=None: rec["kernel_sha"])
    for name, cap in caps.items():
        dram = cap["dram_bytes_read"] + cap["dram_bytes_write"]
        assert cap["dram_bytes_read"] > 0.9 * cap["algorithmic_bytes"]  # the weights are read
        if name in workloads.WORKLOADS:
            assert bench.traffic_record(workloads.WORKLOADS[name], 123) == dram
        for target in cap.get("scales_to", []):
            got = bench.traffic_record(workloads.WORKLOADS[target], 2 * cap["algorithmic_bytes"])
            assert got == pytest.approx(2 * dram)
    assert bench.traffic_record(workloads.WORKLOADS["prefill"], 1) is None  # tensor-bound: no scaling
    monkeypatch.setattr(bench, "kernel_source_sha", lambda read=None: "0" * 16)
    assert bench.traffic_record(workloads.WORKLOADS["decode"], 1) is None


def test_one_launch_detection():
    """The stage times of a forward whose GEMMs ran as one launch (measured at one token: FC1
    stage 67 us, the empty FC2 stage 2.8 us) against separate launches (16 tokens: 293 and
    146 us; prefill: 2.75 and 1.56 ms)."""
    assert bench.one_launch_gemms({"fc1": 0.0670, "fc2": 0.0028})
    assert bench.one_launch_gemms({"fc1": 0.1072, "fc2": 0.0027})
    assert not bench.one_launch_gemms({"fc1": 0.2933, "fc2": 0.1465})
    assert not bench.one_launch_gemms({"fc1": 2.75, "fc2": 1.56})
    assert not bench.one_launch_gemms({"fc1": 0.0158, "fc2": 0.0134})  # tiny
