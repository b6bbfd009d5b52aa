"""Proxy-head gradient on the GPU (msa_fwd_ex with MSA_BLOCK_MASS, then
msa_proxy_bwd) against the oracle of the same reading (oracle/proxy_grad.py:
a KL divergence from the Main Branch's per-block attention mass to the
softmax of the pooled proxy scores).  The pages do not define the proxy
heads' training signal, so this parity is of the reading, not of the pages:
PARITY UNPINNED against them.

Proxy inputs on the 1/8 grid make every proxy score exact in any order, so
both sides see the same pooled scores, the same argmax keys (lowest on ties)
and the same selection.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import CONFIGS, Config, make_inputs
from oracle import proxy_grad as PG
from parity_util import compare, f32, odims, oracle_inputs, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": CONFIGS["tiny"],
    "ragged_b2_g4": Config("ragged_b2_g4", B=2, T=1000, Hq=8, Hkv=2, d=128, dp=64, topk=3),
    "g8_d64_dp16": Config("g8_d64_dp16", B=1, T=640, Hq=8, Hkv=1, d=64, dp=16, topk=2),
    "g1_k5": Config("g1_k5", B=1, T=1300, Hq=2, Hkv=2, d=128, dp=32, topk=5),
}


def run(cfg, seed, q_begin=0):
    from block_sparse_attention_09_b200 import msa
    inp = make_inputs(cfg, seed=seed, exact_proxy=True)
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    dims = msa.make_dims(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.dp, cfg.topk)
    ws = msa.proxy_workspace(dims, dev["q"].device)
    o, lse = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, ws=ws, check=True, block_mass=True)
    # the main backward on the same workspace in between, as in a training step
    msa.bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, idx, nsel, ws=ws, reuse_index=True, check=True)
    dqp, dkp, loss = msa.proxy_bwd(dev["q"], dev["qp"], dev["kp"], idx, nsel, ws, check=True)
    torch.cuda.synchronize()
    return inp, idx, nsel, dqp, dkp, loss


@pytest.mark.parametrize("name", list(CASES))
def test_proxy_grad_matches_oracle(name):
    cfg = CASES[name]
    inp, idx, nsel, dqp, dkp, loss = run(cfg, seed=31)
    x = oracle_inputs(inp)
    m = odims(cfg)
    idx_o, nsel_o, _ = O.select(m, x["qp"], x["kp"])
    assert np.array_equal(idx.cpu().numpy(), idx_o) and np.array_equal(nsel.cpu().numpy(), nsel_o)
    _, lse_o = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o)
    loss_o, dqp_o, dkp_o = PG.loss_and_grad(m, x["qp"], x["kp"], x["q"], x["k"], lse_o, idx_o, nsel_o)
    gl = f32(loss)
    assert (gl >= -1e-6).all(), "a KL divergence is never negative"
    # rows with a single selected block have p = q = 1: loss 0
    single = f32(nsel) == 1
    assert np.abs(gl[single]).max(initial=0.0) <= 1e-6
    tot = float(gl.astype(np.float64).sum())
    assert abs(tot - loss_o) <= 1e-3 * abs(loss_o) + 2e-2, (tot, loss_o)
    compare("dqp", f32(dqp), dqp_o, rel=0.0)
    compare("dkp", f32(dkp), dkp_o, rel=0.0)


def test_proxy_grad_shape_of_the_gradient():
    """The gradient reaches only argmax keys of selected blocks: every key row
    of dkp that is non-zero is the first maximum of its block for some row;
    and dqp of a row is a combination of the proxy keys it selected."""
    cfg = CASES["tiny"]
    inp, idx, nsel, dqp, dkp, loss = run(cfg, seed=32)
    x = oracle_inputs(inp)
    g = f32(dkp)[0, :, 0]
    nz = np.nonzero(np.abs(g).sum(axis=1))[0]
    ii, nn = f32(idx)[0, 0], f32(nsel)[0, 0]
    argmaxes = set()
    for i in range(cfg.T):
        for s in range(int(nn[i])):
            n = int(ii[i, s])
            j1 = min((n + 1) * 128, i + 1)
            sc = x["kp"][0, n * 128:j1, 0].astype(np.float64) @ x["qp"][0, i, 0].astype(np.float64)
            argmaxes.add(n * 128 + int(np.argmax(sc)))
    assert set(nz.tolist()) <= argmaxes


def test_proxy_grad_of_a_shard():
    """q_begin: every call of the step restricted to the query rows from a
    block boundary on (a context-parallel shard).  dqp and the loss of those
    rows, and dkp from their contributions alone, against the oracle over
    the same rows; rows before q_begin of dqp and loss are left untouched."""
    from block_sparse_attention_09_b200 import msa
    cfg = CASES["ragged_b2_g4"]
    q0 = 512
    inp = make_inputs(cfg, seed=33, exact_proxy=True)
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, q_begin=q0, check=True)
    dims = msa.make_dims(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.dp, cfg.topk, q_begin=q0)
    ws = msa.proxy_workspace(dims, dev["q"].device)
    o, lse = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, ws=ws, check=True, block_mass=True, q_begin=q0)
    msa.bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, idx, nsel, ws=ws, reuse_index=True, check=True,
            q_begin=q0)
    dqp = torch.full(dev["qp"].shape, 7.0, dtype=torch.float32, device="cuda")
    dkp = torch.empty(dev["kp"].shape, dtype=torch.float32, device="cuda")
    loss = torch.full((cfg.B, cfg.Hkv, cfg.T), 7.0, dtype=torch.float32, device="cuda")
    msa.proxy_bwd(dev["q"], dev["qp"], dev["kp"], idx, nsel, ws, check=True, out=(dqp, dkp, loss), q_begin=q0)
    torch.cuda.synchronize()
    assert bool((dqp[:, :q0] == 7.0).all()) and bool((loss[:, :, :q0] == 7.0).all())
    x = oracle_inputs(inp)
    m = odims(cfg)
    idx_o, nsel_o, _ = O.select(m, x["qp"], x["kp"])
    gi, gn = idx.cpu().numpy(), nsel.cpu().numpy()
    assert np.array_equal(gi[:, :, q0:], idx_o[:, :, q0:]) and np.array_equal(gn[:, :, q0:], nsel_o[:, :, q0:])
    _, lse_o = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o)
    rows = [(b, g, i) for b in range(cfg.B) for g in range(cfg.Hkv) for i in range(q0, cfg.T)]
    loss_o, dqp_o, dkp_o = PG.loss_and_grad(m, x["qp"], x["kp"], x["q"], x["k"], lse_o, idx_o, nsel_o, rows=rows)
    tot = float(f32(loss)[:, :, q0:].astype(np.float64).sum())
    assert abs(tot - loss_o) <= 1e-3 * abs(loss_o) + 2e-2, (tot, loss_o)
    compare("dqp (shard)", f32(dqp)[:, q0:], dqp_o[:, q0:], rel=0.0)
    compare("dkp (shard)", f32(dkp), dkp_o, rel=0.0)
