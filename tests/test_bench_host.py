"""Host-side accounting of bench.py: the algorithmic work per stage that the
roofline fractions divide by, on small synthetic plans (no GPU)."""

import numpy as np
import pytest
import torch

from tests.conftest import ROOT  # noqa: F401  (puts the repo on sys.path)


class _Plan:
    def __init__(self, topk):
        self.topk = torch.from_numpy(np.ascontiguousarray(topk, dtype=np.int32))


def _brute_selected(topk, pos, W):
    """|S(t)| row by row: top-K entries <= p - W, plus min(W, p + 1) window keys."""
    return sum(int(((r >= 0) & (r <= p - W)).sum()) + min(W, p + 1) for r, p in zip(topk, pos))


@pytest.mark.parametrize("rows", [None, 48])
def test_two_stage_work_counts(rows):
    import bench
    cfg = dict(kind="two_stage", N=200, Hq=4, d=64, H_I=2, D_I=32, block=16, keep=3, K=20, W=5)
    if rows:
        cfg["rows"] = rows
    T = rows or cfg["N"]
    pos = np.arange(cfg["N"] - T, cfg["N"])
    rng = np.random.default_rng(0)
    topk = np.full((T, cfg["K"]), -1, dtype=np.int64)
    for i, p in enumerate(pos):
        k = min(cfg["K"], p + 1)
        topk[i, :k] = np.sort(rng.choice(p + 1, size=k, replace=False))
    w = bench.stage_work(dict(cfg=cfg, plan=_Plan(topk), inp={}))
    sel = _brute_selected(topk, pos, cfg["W"])
    assert w["sum_selected"] == sel
    assert w["causal_pairs"] == sum(p + 1 for p in pos)
    blk, keep = cfg["block"], cfg["keep"]
    assert w["coarse_pairs"] == sum(p // blk for p in pos)
    assert w["fine_pairs"] == sum(min(keep, p // blk) * blk + p % blk + 1 for p in pos)
    st = w["stages"]
    assert st["attention"]["flops"] == 4.0 * cfg["Hq"] * cfg["d"] * sel
    assert st["attention"]["gathered"] == sel * cfg["d"] * 2 * 2          # one K and one V row per key
    # the fine scores write one fp32 score per candidate
    fixed = T * cfg["H_I"] * cfg["D_I"] * 2 + T * cfg["H_I"] * 2 + cfg["N"] * cfg["D_I"] * 2 + 4 * T * (keep + 1)
    assert st["fine_indexer"]["bytes"] == fixed + 4 * w["fine_pairs"]
    assert st["fine_topk"]["bytes"] == 4 * w["fine_pairs"] + 4 * T * keep + 4 * T * cfg["K"]
    assert st["coarse_topk"]["bytes"] == 4 * w["coarse_pairs"] + 4 * T + 4 * T * keep


def test_decode_work_counts():
    import bench
    lengths = np.array([1, 700, 5000], dtype=np.int32)
    cfg = dict(kind="decode", B=3, Hq=8, d=64, H_I=2, D_I=32, K=64, W=16)
    rng = np.random.default_rng(1)
    topk = np.full((3, cfg["K"]), -1, dtype=np.int64)
    for b, L in enumerate(lengths):
        k = min(cfg["K"], int(L))
        topk[b, :k] = np.sort(rng.choice(int(L), size=k, replace=False))
    w = bench.stage_work(dict(cfg=cfg, plan=_Plan(topk), inp=dict(lengths=lengths)))
    sel = _brute_selected(topk, lengths - 1, cfg["W"])
    assert w["sum_selected"] == sel and w["causal_pairs"] == int(lengths.sum())
    st = w["stages"]
    P = int(lengths.sum())
    # the fused select reads the keys once and writes only the selection
    assert st["indexer_topk"]["bytes"] == (3 * 2 * 32 * 2 + 3 * 2 * 2 + P * 32 * 2 + 4 * 3 * 64)
    assert st["indexer"]["bytes"] - st["indexer_topk"]["bytes"] == 4 * P - 4 * 3 * 64


def test_roofline_entry_fractions():
    import bench
    peaks = dict(hbm=1000.0, bf16=100.0)
    e = bench.roofline_entry("hbm", 2e9, 0.0, 1e-3, peaks)
    assert e["achieved"] == 2000.0 and e["frac"] == 2.0 and e["unit"] == "GB/s"
    t = bench.roofline_entry("tensor", 0.0, 5e10, 1e-3, peaks)
    assert t["achieved"] == 50.0 and t["frac"] == 0.5 and t["unit"] == "TFLOP/s"


def test_traffic_lookup_follows_the_source_hash(tmp_path, monkeypatch):
    # roofline.traffic comes from a capture of the exact sources that are built:
    # a matching hash gives bytes x scale, any other hash or stage gives None
    import json
    import os
    import bench
    (tmp_path / "profiles").mkdir()
    os.symlink(os.path.join(bench.ROOT, "fine_grained_top_b200"), tmp_path / "fine_grained_top_b200")
    real = bench.source_hash(bench.STAGE_SOURCE["attention"])
    entries = [dict(workload="w", stage="attention", sources="x", source_hash=real, bytes_per_launch=1000, scale=2.0),
               dict(workload="w", stage="fine_topk", sources="x", source_hash="000000000000", bytes_per_launch=5)]
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps({"entries": entries}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("w", "attention") == 2000
    assert bench.ncu_traffic("w", "fine_topk") is None         # captured from other sources
    assert bench.ncu_traffic("other", "attention") is None     # another workload
    assert bench.ncu_traffic("w", "no_such_stage") is None
