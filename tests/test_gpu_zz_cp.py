"""GPU checks of the context-parallel pieces, on one GPU: the library calls
restricted to a shard's query rows (q_begin) and the fp32 partial gradients,
with the ranks of a context-parallel step run one after another, one call
per zig-zag chunk (the all-gather is a slice of the whole tensors, the
reduce-scatter a sum of the partials); the kernels of different ranks never
wait on one another.

The sharded step must give the selection of the unsplit call bit for bit,
O, L and dQ within two bf16 ulps of it (the fp32 reductions add in a
different order), dK/dV within the bf16 tolerance, and everything within the
parity tolerance of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import Config, make_inputs
from parity_util import compare, odims

pytestmark = pytest.mark.gpu


def close(a, b, ulps=2):
    a, b = a.float(), b.float()
    return bool(((a - b).abs() <= ulps * 2.0 ** -8 * b.abs() + 1e-3).all())


CASES = [
    ("w2_ragged", Config("w2_ragged", B=1, T=1000, Hq=8, Hkv=2, d=128, dp=64, topk=5), 2),
    ("w3_b2_d64", Config("w3_b2_d64", B=2, T=1536, Hq=4, Hkv=1, d=64, dp=32, topk=4), 3),
    ("w4_g8", Config("w4_g8", B=1, T=2048, Hq=8, Hkv=1, d=128, dp=64, topk=6), 4),
]


@pytest.mark.parametrize("name,cfg,world", CASES, ids=[c[0] for c in CASES])
def test_sharded_step_matches_unsplit(name, cfg, world):
    from block_sparse_attention_09_b200 import cp, msa
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=21, exact_proxy=True).items()}
    # the unsplit step
    idx, nsel = msa.proxy_select(x["qp"], x["kp"], cfg.topk, check=True)
    o, lse = msa.fwd(x["q"], x["k"], x["v"], idx, nsel, check=True)
    dq, dk, dv = msa.bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, idx, nsel, check=True)
    # the ranks of a context-parallel step, one after another, each over its
    # zig-zag chunks (one library call per chunk)
    chunks = [c for r in range(world) for c in cp.shard_chunks(cfg.T, world, r)]
    dk_sum = torch.zeros(x["k"].shape, dtype=torch.float32, device="cuda")
    dv_sum = torch.zeros_like(dk_sum)
    for r0, r1 in chunks:
        mine = {k: t[:, r0:r1].contiguous() for k, t in x.items()}
        pre = {k: x[k][:, :r1].contiguous() for k in ("k", "v", "kp")}
        o_r, lse_r, dq_r, dk_p, dv_p, idx_r, nsel_r = cp.local_step(
            mine["q"], pre["k"], pre["v"], mine["dout"], mine["qp"], pre["kp"], cfg.topk, r0, msa)
        torch.cuda.synchronize()
        assert torch.equal(idx_r[:, :, r0:], idx[:, :, r0:r1]), f"selection of rows {r0}..{r1}"
        assert torch.equal(nsel_r[:, :, r0:], nsel[:, :, r0:r1])
        assert close(o_r, o[:, r0:r1]) and close(lse_r, lse[:, :, r0:r1]) and close(dq_r, dq[:, r0:r1])
        dk_sum[:, :r1] += dk_p
        dv_sum[:, :r1] += dv_p
    dk_cp, dv_cp = msa.f32_to_bf16(dk_sum), msa.f32_to_bf16(dv_sum)
    torch.cuda.synchronize()
    assert close(dk_cp, dk) and close(dv_cp, dv)
    # and against the oracle
    xo = {k: v.float().cpu().numpy() for k, v in x.items()}
    ref = O.full(odims(cfg), xo["qp"], xo["kp"], xo["q"], xo["k"], xo["v"], xo["dout"])
    compare("dK (sharded)", dk_cp.float().cpu().numpy(), ref["dk"])
    compare("dV (sharded)", dv_cp.float().cpu().numpy(), ref["dv"])


def test_rows_before_q_begin_untouched():
    """q_begin: the forward writes rows q_begin .. T-1 of o and lse only; the
    backward's fp32 dK/dV then hold only those rows' contributions."""
    from block_sparse_attention_09_b200 import msa
    cfg = Config("qb", B=1, T=1024, Hq=4, Hkv=1, d=64, dp=32, topk=3)
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=22, exact_proxy=True).items()}
    q0 = 512
    idx, nsel = msa.proxy_select(x["qp"], x["kp"], cfg.topk, q_begin=q0, check=True)
    o = torch.full_like(x["q"], 7.0)
    lse = torch.full((cfg.B, cfg.Hq, cfg.T), 7.0, device="cuda")
    msa.fwd(x["q"], x["k"], x["v"], idx, nsel, out=(o, lse), q_begin=q0, check=True)
    torch.cuda.synchronize()
    assert bool((o[:, :q0] == 7.0).all()) and bool((lse[:, :, :q0] == 7.0).all())
    full_idx, full_nsel = msa.proxy_select(x["qp"], x["kp"], cfg.topk, check=True)
    o_full, lse_full = msa.fwd(x["q"], x["k"], x["v"], full_idx, full_nsel, check=True)
    assert close(o[:, q0:], o_full[:, q0:]) and close(lse[:, :, q0:], lse_full[:, :, q0:])
    # a key at position j is read only by queries i >= j, so the keys from q0
    # on receive their whole gradient from the rows q0 .. T-1
    dq, dk, dv = msa.bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, idx, nsel, q_begin=q0, dkv_f32=True,
                         check=True)
    _, dk_full, dv_full = msa.bwd(x["q"], x["k"], x["v"], o_full, x["dout"], lse_full, full_idx, full_nsel,
                                  check=True)
    torch.cuda.synchronize()
    assert dk.dtype == torch.float32
    assert close(msa.f32_to_bf16(dk)[:, q0:], dk_full[:, q0:]) and close(msa.f32_to_bf16(dv)[:, q0:],
                                                                          dv_full[:, q0:])


def test_empty_shard_computes_nothing():
    """q_begin = T: a shard with no query rows.  The forward's outputs and
    the dQ rows are left untouched, and the fp32 dK/dV partials are exactly
    zero (no query contributes)."""
    from block_sparse_attention_09_b200 import msa
    cfg = Config("empty", B=1, T=768, Hq=4, Hkv=1, d=64, dp=32, topk=3)
    x = {k: v.cuda() for k, v in make_inputs(cfg, seed=23, exact_proxy=True).items()}
    T = cfg.T
    msa.proxy_select(x["qp"], x["kp"], cfg.topk, q_begin=T, check=True)   # launches no tile
    idx, nsel = msa.proxy_select(x["qp"], x["kp"], cfg.topk, check=True)
    o = torch.full_like(x["q"], 7.0)
    lse = torch.full((cfg.B, cfg.Hq, T), 7.0, device="cuda")
    msa.fwd(x["q"], x["k"], x["v"], idx, nsel, out=(o, lse), q_begin=T, check=True)
    dq = torch.full_like(x["q"], 7.0)
    dk = torch.full(x["k"].shape, 7.0, dtype=torch.float32, device="cuda")
    dv = torch.full_like(dk, 7.0)
    msa.bwd(x["q"], x["k"], x["v"], o, x["dout"], lse, idx, nsel, out=(dq, dk, dv), q_begin=T, dkv_f32=True,
            check=True)
    torch.cuda.synchronize()
    assert bool((o == 7.0).all()) and bool((lse == 7.0).all()) and bool((dq == 7.0).all())
    assert bool((dk == 0).all()) and bool((dv == 0).all())
