"""Host-side logic of bench.py that needs no GPU: the resumable JSON-lines sweep, the parity
statistics it records, and the config object both arms share."""
import json
import os
import subprocess
import sys
from types import SimpleNamespace

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_sweep_skips_workloads_already_recorded(tmp_path):
    rec = tmp_path / "records.jsonl"
    rec.write_text(json.dumps({"workload": "tiny", "step": 0}) + "\n" +
                   json.dumps({"workload": "n100", "step": 0}) + "\n")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--sweep", "tiny,n100",
                        "--records", str(rec)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.count("already recorded, skipped") == 2
    assert len(rec.read_text().splitlines()) == 2  # nothing appended


def test_sweep_rejects_unknown_workloads(tmp_path):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--sweep", "nope",
                        "--records", str(tmp_path / "r.jsonl")], capture_output=True, text=True,
                       timeout=120)
    assert r.returncode != 0 and "unknown workloads" in (r.stderr + r.stdout)


def _fake_ref(H=2, nq=3, k=4, L=150, seed=0):
    rng = np.random.default_rng(seed)
    blocks = [0, 1, 2]
    rows = np.concatenate([np.arange(64 * i, min(64 * i + 64, L)) for i in blocks])
    idx = np.stack([np.stack([rng.permutation(10)[:k] for _ in range(nq)]) for _ in range(H)])
    out = rng.standard_normal((rows.size, H, 8))
    gap = np.array([[1.0, 0.0, 1e-3], [0.0, 0.0, 0.0]])
    return SimpleNamespace(rows=rows, idx=idx.astype(np.int32), gap=gap, out=out)


def test_parity_stats_exact_and_one_block_differing():
    sys.path.insert(0, ROOT)
    import bench

    ref = _fake_ref()
    s = bench.parity_stats(ref.idx.copy(), ref.out.copy(), ref, 0)
    assert s["sets_equal"] == 1.0 and s["max_abs"] == 0.0 and s["rel_l2"] == 0.0
    assert s["gap_separated"] == 2 / 6
    idx = ref.idx.copy()
    idx[1, 2, 0] = 99  # head 1, query block 2: a different set
    out = ref.out.copy()
    out[128:, 1] += 5.0  # that block's rows of head 1 are wrong: excluded from the error
    out[0, 0, 0] += 1e-3  # a small error where the sets agree
    s = bench.parity_stats(idx, out, ref, 0)
    assert abs(s["sets_equal"] - 5 / 6) < 1e-12
    assert abs(s["max_abs"] - 1e-3) < 1e-12


def test_both_arms_share_the_config_object():
    sys.path.insert(0, ROOT)
    import bench

    wl = bench.WORKLOADS["n1000"]
    c1 = bench.workload_config(wl, 1, bench.l2_note(wl["L"], wl["H"]))
    c2 = bench.workload_config(wl, 1, bench.l2_note(wl["L"], wl["H"]))
    assert c1 == c2 and c1["L"] == 1374000 and "exceed L2" in c1["l2"]
