"""Host logic of bench.py, on CPU: the FLOP model against a brute-force count of
the (query head, key) pairs the oracle's own selection reads, and the guard
that reports recorded DRAM traffic only for unchanged kernel sources."""
import hashlib
import json
import os
import sys

import numpy as np
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import Config, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_flop_model_counts_the_selected_pairs():
    cfg = Config("flops", B=2, T=1000, Hq=4, Hkv=2, d=64, dp=32, topk=3)
    inp = make_inputs(cfg, seed=51, exact_proxy=True, parts=["qp", "kp"])
    m = O.Dims(B=cfg.B, T=cfg.T, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, dp=cfg.dp, topk=cfg.topk)
    idx, nsel, _ = O.select(m, inp["qp"].float().numpy(), inp["kp"].float().numpy())
    # brute force: keys j <= i of every selected block, per (b, group, i)
    pairs = 0
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            for i in range(cfg.T):
                for n in idx[b, g, i, :nsel[b, g, i]]:
                    pairs += min(128, i - 128 * int(n) + 1)
    f_proxy, f_fwd, f_bwd = bench.flops_from_nsel(cfg, bench.pair_count(cfg, torch.from_numpy(nsel)))
    assert f_fwd == 4.0 * cfg.d * cfg.G * pairs
    assert f_bwd == 2.5 * f_fwd
    # proxy: every key before the query's own block, for query tiles that rank
    scored = 0
    for qb in range((cfg.T + 127) // 128):
        if qb + 1 > cfg.topk:
            scored += min(128, cfg.T - 128 * qb) * 128 * qb
    assert f_proxy == 2.0 * cfg.dp * scored * cfg.B * cfg.Hkv


def test_pair_count_of_row_shards_adds_up():
    """The context-parallel bench counts each rank's rows from its own row
    offset: the shards' counts add up to the whole sequence's."""
    cfg = Config("shards", B=2, T=1000, Hq=4, Hkv=2, d=64, dp=32, topk=3)
    g = torch.Generator().manual_seed(5)
    i = torch.arange(cfg.T)
    nsel = torch.minimum(torch.randint(1, cfg.topk + 1, (cfg.B, cfg.Hkv, cfg.T), generator=g), i // 128 + 1)
    whole = bench.pair_count(cfg, nsel)["pairs"]
    brute = sum(128 * (int(nsel[b, h, r]) - 1) + r % 128 + 1
                for b in range(cfg.B) for h in range(cfg.Hkv) for r in range(cfg.T))
    assert whole == brute
    parts = sum(bench.pair_count(cfg, nsel[:, :, r0:r1], r0)["pairs"] for r0, r1 in ((0, 256), (256, 640), (640, 1000)))
    assert parts == whole


def test_recorded_traffic_needs_unchanged_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "block_sparse_attention_09_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "a.cu").write_bytes(b"kernel source")
    (csrc / "b.h").write_bytes(b"header")
    digest = hashlib.sha256(b"kernel source" + b"header").hexdigest()
    rec = {"records": [
        {"kernel": "k1", "workload": "w", "bytes_per_launch_captured": 15432.0, "scale_to_full": 8.0,
         "sources": ["a.cu", "b.h"], "sources_sha256": digest},
        {"kernel": "k2", "workload": "w", "bytes_per_launch_captured": 5.0, "scale_to_full": 1.0,
         "sources": ["a.cu"], "sources_sha256": "00"}]}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k1", "w") == 123456.0
    assert bench.recorded_traffic("k2", "w") is None          # hash differs
    assert bench.recorded_traffic("k3", "w") is None          # no record
    assert bench.recorded_traffic("k1", "other") is None      # no record for the workload
    (csrc / "a.cu").write_bytes(b"kernel source, edited")
    assert bench.recorded_traffic("k1", "w") is None          # changed since the capture


def test_workload_names():
    cfg = Config("x", B=1, T=256, Hq=4, Hkv=1, d=64, dp=32, topk=2, bias="recency")
    assert "recency" in bench.workload_name(cfg)
    assert "window" not in bench.workload_name(cfg)
    assert "forced window 4 blocks at dilation 2" in bench.workload_name(cfg, 4, 2)
    assert np.isfinite(bench.measured_peaks()[0]["hbm_gbs"])
