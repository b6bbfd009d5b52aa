"""Context-parallel MSA (one sequence split by rows over the ranks), host
side, on CPU: the shard split, and a whole step over two and three gloo
ranks -- all-gather of the key side, per-rank selection, forward and
backward of its own query rows (q_begin), reduce-scatter of the fp32 partial
dK/dV -- against the oracle run on the unsplit sequence.

The per-rank attention here is the oracle behind the library's call
signatures (a test stand-in: on GPUs the same orchestration calls the CUDA
library, checked in test_gpu_zz_cp.py); what these tests pin is the
decomposition and the collectives, with a real process group.
"""
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_attention_09_b200 import cp  # noqa: E402
from block_sparse_attention_09_b200.inputs import Config, make_inputs  # noqa: E402


class OracleOps:
    """The oracle behind the library's Python call signatures (CPU tensors).
    Rows before q_begin are neither selected nor computed, as in the library."""

    import oracle as O

    @staticmethod
    def make_dims(B, T, Hq, Hkv, d, dp, topk, scale=0.0, window=1, dilation=1, q_begin=0):
        return types.SimpleNamespace(B=B, T=T, Hq=Hq, Hkv=Hkv, d=d, dp=dp, topk=topk, q_begin=q_begin)

    @staticmethod
    def step_workspace(dims, device):
        return {}

    @classmethod
    def _m(cls, B, T, Hq, Hkv, d, dp, topk):
        return cls.O.Dims(B=B, T=T, Hq=Hq, Hkv=Hkv, d=d, dp=dp, topk=topk)

    @classmethod
    def proxy_select(cls, qp, kp, topk, q_begin=0):
        B, T, Hp, dp = qp.shape
        m = cls._m(B, T, Hp, Hp, 64, dp, topk)
        rows = [(b * Hp + g) * T + i for b in range(B) for g in range(Hp) for i in range(q_begin, T)]
        idx, nsel, _ = cls.O.select(m, qp.float().numpy(), kp.float().numpy(), rows=rows)
        return torch.from_numpy(idx), torch.from_numpy(nsel)

    @classmethod
    def fwd(cls, q, k, v, idx, nsel, scale=0.0, ws=None, q_begin=0):
        B, T, Hq, d = q.shape
        m = cls._m(B, T, Hq, k.shape[2], d, 64, idx.shape[3])
        rows = [(b * Hq + h) * T + i for b in range(B) for h in range(Hq) for i in range(q_begin, T)]
        o, lse = cls.O.fwd(m, q.float().numpy(), k.float().numpy(), v.float().numpy(), idx.numpy(), nsel.numpy(),
                           rows=rows)
        return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).float()

    @classmethod
    def bwd(cls, q, k, v, o, dout, lse, idx, nsel, scale=0.0, ws=None, reuse_index=False, q_begin=0,
            dkv_f32=False):
        B, T, Hq, d = q.shape
        m = cls._m(B, T, Hq, k.shape[2], d, 64, idx.shape[3])
        rows = [(b * Hq + h) * T + i for b in range(B) for h in range(Hq) for i in range(q_begin, T)]
        x = [t.float().numpy() for t in (q, k, v, dout)]
        dq, D = cls.O.bwd_dq(m, *x, o.float().numpy().astype(np.float64), lse.numpy().astype(np.float64),
                             idx.numpy(), nsel.numpy(), rows=rows)
        # rows before q_begin selected nothing, so every block's selecting
        # queries are this shard's: the partial dK, dV of its rows
        dk, dv = cls.O.bwd_dkdv(m, *x, lse.numpy().astype(np.float64), D, idx.numpy(), nsel.numpy())
        kv = torch.float32 if dkv_f32 else torch.bfloat16
        return torch.from_numpy(dq).to(torch.bfloat16), torch.from_numpy(dk).to(kv), torch.from_numpy(dv).to(kv)

    @staticmethod
    def f32_to_bf16(x):
        return x.to(torch.bfloat16)


def test_shard_chunks_cover_the_sequence_and_balance_the_work():
    for T in (1, 127, 128, 640, 1000, 4096, 131072 + 77, 1 << 20):
        for world in (1, 2, 3, 4, 8):
            chunks = [cp.shard_chunks(T, world, r) for r in range(world)]
            flat = sorted(c for ch in chunks for c in ch)
            assert flat[0][0] == 0 and flat[-1][1] == T
            for (a0, a1), (c0, c1) in zip(flat, flat[1:]):
                assert a1 == c0                       # contiguous, disjoint
            for c0, c1 in flat:
                assert c0 % 128 == 0 and c0 < c1      # block aligned, non-empty
            for ch in chunks:
                assert ch == sorted(ch)               # a rank's rows in sequence order
            nblk = (T + 127) // 128
            if nblk >= 2 * world:
                # rows: within two blocks of each other
                nb = [sum((c1 - c0 + 127) // 128 for c0, c1 in ch) for ch in chunks]
                assert max(nb) - min(nb) <= 2
                # causal proxy work (keys scored per row ~ its position): the
                # zig-zag pairing keeps every rank within 2 % + two chunks'
                # rounding of the mean
                work = [sum(i for c0, c1 in ch for i in range(c0, c1, 128)) for ch in chunks]
                mean = sum(work) / world
                assert max(work) <= mean * 1.02 + 2 * 128 * nblk, (T, world, work)


def test_zigzag_pairs_early_and_late_chunks():
    ch = [cp.shard_chunks(16 * 128, 4, r) for r in range(4)]
    assert ch[0] == [(0, 256), (1792, 2048)]
    assert ch[3] == [(768, 1024), (1024, 1280)]
    x = torch.arange(16 * 128).view(1, -1)
    assert cp.take_rows(x, ch[1]).tolist()[0] == list(range(256, 512)) + list(range(1536, 1792))


CFG = Config("cp", B=1, T=1000, Hq=4, Hkv=2, d=64, dp=32, topk=3)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        x = make_inputs(CFG, seed=3, exact_proxy=True)
        chunks = cp.shard_chunks(CFG.T, world, rank)
        mine = {k: cp.take_rows(t, chunks) for k, t in x.items()}
        o, lse, dq, dk, dv = cp.step(mine["q"], mine["k"], mine["v"], mine["dout"], mine["qp"], mine["kp"],
                                     CFG.topk, CFG.T, ops=OracleOps)
        torch.save(dict(chunks=chunks, o=o, lse=lse, dq=dq, dk=dk, dv=dv), os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_cp_step_matches_the_unsplit_sequence(tmp_path, oracle_mod, world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    O = oracle_mod
    x = {k: t.float().numpy() for k, t in make_inputs(CFG, seed=3, exact_proxy=True).items()}
    m = O.Dims(B=CFG.B, T=CFG.T, Hq=CFG.Hq, Hkv=CFG.Hkv, d=CFG.d, dp=CFG.dp, topk=CFG.topk)
    # the unsplit sequence, with the backward's D taken from the bf16-stored O
    # as the library (and the stand-in) does
    idx, nsel, _ = O.select(m, x["qp"], x["kp"])
    o, lse = O.fwd(m, x["q"], x["k"], x["v"], idx, nsel)
    o16 = torch.from_numpy(o).to(torch.bfloat16).float().numpy().astype(np.float64)
    dq, D = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], o16, lse, idx, nsel)
    dk, dv = O.bwd_dkdv(m, x["q"], x["k"], x["v"], x["dout"], lse, D, idx, nsel)
    ref = dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)
    covered = 0
    for r in range(world):
        got = torch.load(tmp_path / f"rank{r}.pt")
        rows = np.concatenate([np.arange(c0, c1) for c0, c1 in got["chunks"]])
        covered += len(rows)
        # bf16 outputs: within the rounding of one bf16 store (dK/dV: several
        # chunks' fp32 partials added before the one rounding)
        for name, g, rf in (("o", got["o"], ref["o"][:, rows]), ("dq", got["dq"], ref["dq"][:, rows]),
                            ("dk", got["dk"], ref["dk"][:, rows]), ("dv", got["dv"], ref["dv"][:, rows])):
            err = np.abs(g.float().numpy() - rf)
            assert (err <= 1e-6 + 2.0 ** -8 * np.abs(rf)).all(), (name, r, float(err.max()))
        assert np.allclose(got["lse"].numpy(), ref["lse"][:, :, rows], rtol=1e-6, atol=1e-5)
    assert covered == CFG.T


def test_single_rank_without_a_process_group(oracle_mod):
    """No process group: the step is the whole sequence on one rank (q_begin
    0, fp32 gradients rounded once), equal to the unsplit oracle run."""
    O = oracle_mod
    x = make_inputs(CFG, seed=4, exact_proxy=True)
    o, lse, dq, dk, dv, idx, nsel = cp.step(x["q"], x["k"], x["v"], x["dout"], x["qp"], x["kp"], CFG.topk, CFG.T,
                                            ops=OracleOps, return_selection=True)
    xf = {k: t.float().numpy() for k, t in x.items()}
    m = O.Dims(B=CFG.B, T=CFG.T, Hq=CFG.Hq, Hkv=CFG.Hkv, d=CFG.d, dp=CFG.dp, topk=CFG.topk)
    ref = O.full(m, xf["qp"], xf["kp"], xf["q"], xf["k"], xf["v"], xf["dout"])
    assert np.array_equal(idx.numpy(), ref["idx"]) and np.array_equal(nsel.numpy(), ref["nsel"])
    err = np.abs(o.float().numpy() - ref["o"])
    assert (err <= 1e-6 + 2.0 ** -8 * np.abs(ref["o"])).all()
    assert np.allclose(lse.numpy(), ref["lse"], rtol=1e-6, atol=1e-5)
