"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on CPU.

The path partitions by independent problems: each rank runs its own batch
(seed = rank) with no data-path collective, and the job figures combine the
ranks' timings (max) and work (sum).  These tests check that combination and
the per-rank inputs over a real two-process group, without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_09_b200.inputs import CONFIGS, make_inputs
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        # rank r takes 10 + r ms for 1000 * (r + 1) units
        ms, units = bench.combine_ranks(dist, world, torch.device("cpu"), 10.0 + rank, 1000.0 * (rank + 1))
        # a second call in the same order on every rank (the e2e figure)
        e_ms, _ = bench.combine_ranks(dist, world, torch.device("cpu"), 20.0 - rank, 1.0)
        x = make_inputs(CONFIGS["tiny"], seed=rank, parts=["q"])["q"]
        digest = float(x.float().sum())
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{ms} {units} {e_ms} {digest}\n")
    finally:
        dist.destroy_process_group()


def test_two_rank_combination(tmp_path):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    vals = [list(map(float, open(tmp_path / f"rank{r}.txt").read().split())) for r in range(world)]
    for ms, units, e_ms, _ in vals:
        assert ms == 11.0           # the slowest rank sets the job time
        assert units == 3000.0      # work of both ranks
        assert e_ms == 20.0
    # each rank draws its own batch
    assert vals[0][3] != vals[1][3]


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(None, 1, None, 5.0, 7.0) == (5.0, 7.0)
