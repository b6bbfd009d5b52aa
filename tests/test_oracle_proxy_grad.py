"""Pins of the proxy-head loss oracle (oracle/proxy_grad.py; parity unpinned
against the pages, which do not describe the mechanism -- these tests fix the
definition written there): its gradient against central finite differences
of its loss, the block masses against a dense softmax, the loss against a
library KL of independently built distributions, and the one-block rows,
whose loss and gradient vanish."""
import numpy as np
import pytest
import torch
from scipy.special import rel_entr

import oracle as O
from oracle import proxy_grad as PG
from block_sparse_attention_09_b200.inputs import Config, make_inputs

CFG = Config("pg", B=1, T=200, Hq=4, Hkv=2, d=16, dp=8, topk=3)


def problem(seed=0):
    x = {k: v.float().numpy() for k, v in make_inputs(CFG, seed=seed).items()}
    m = O.Dims(B=CFG.B, T=CFG.T, Hq=CFG.Hq, Hkv=CFG.Hkv, d=CFG.d, dp=CFG.dp, topk=CFG.topk, blk=32)
    idx, nsel, _ = O.select(m, x["qp"], x["kp"])
    _, lse = O.fwd(m, x["q"], x["k"], x["v"], idx, nsel)
    return m, x, idx, nsel, lse


def test_gradient_matches_finite_differences(oracle_mod):
    m, x, idx, nsel, lse = problem()
    qp, kp = x["qp"].astype(np.float64), x["kp"].astype(np.float64)
    loss, dqp, dkp = PG.loss_and_grad(m, qp, kp, x["q"], x["k"], lse, idx, nsel)
    assert loss > 0
    rng = np.random.default_rng(1)
    h = 1e-5
    for arr, grad in ((qp, dqp), (kp, dkp)):
        for _ in range(12):
            b, t, g, c = (int(rng.integers(s)) for s in arr.shape)
            keep = arr[b, t, g, c]
            arr[b, t, g, c] = keep + h
            lp = PG.loss_and_grad(m, qp, kp, x["q"], x["k"], lse, idx, nsel)[0]
            arr[b, t, g, c] = keep - h
            lm = PG.loss_and_grad(m, qp, kp, x["q"], x["k"], lse, idx, nsel)[0]
            arr[b, t, g, c] = keep
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[b, t, g, c]) <= 1e-6 + 1e-5 * abs(fd), (fd, grad[b, t, g, c])


def test_block_mass_is_the_forward_softmax(oracle_mod):
    """p_i(n) from a dense masked softmax per head (torch, float64), with the
    forward's own L: it sums to one over the selected blocks."""
    m, x, idx, nsel, lse = problem(seed=2)
    blk, G = m.blk, m.G
    scale = 1.0 / np.sqrt(m.d)
    q, k = torch.from_numpy(x["q"]).double(), torch.from_numpy(x["k"]).double()
    for g in range(m.Hkv):
        for i in (5, 40, 77, 130, 199):
            ns = int(nsel[0, g, i])
            sel = idx[0, g, i, :ns]
            mask = torch.zeros(m.T, dtype=torch.bool)
            for n in sel:
                mask[n * blk:min((n + 1) * blk, i + 1)] = True
            want = np.zeros(ns)
            for hh in range(G):
                s = scale * (k[0, :, g] @ q[0, i, g * G + hh])
                pr = torch.softmax(s.masked_fill(~mask, float("-inf")), 0)
                want += np.array([float(pr[n * blk:(n + 1) * blk].sum()) for n in sel]) / G
            got = PG.block_mass(m, x["q"], x["k"], lse, idx, nsel, 0, g, i)
            assert np.allclose(got, want, rtol=1e-9, atol=1e-12)
            assert abs(got.sum() - 1.0) < 1e-9


def test_loss_is_the_kl_of_independent_distributions(oracle_mod):
    m, x, idx, nsel, lse = problem(seed=3)
    blk = m.blk
    loss = PG.loss_and_grad(m, x["qp"], x["kp"], x["q"], x["k"], lse, idx, nsel)[0]
    want = 0.0
    for g in range(m.Hkv):
        S = x["kp"][0, :, g].astype(np.float64) @ x["qp"][0, :, g].astype(np.float64).T   # [key, query]
        for i in range(m.T):
            ns = int(nsel[0, g, i])
            sel = idx[0, g, i, :ns]
            z = np.array([S[n * blk:min((n + 1) * blk, i + 1), i].max() for n in sel])
            qd = np.exp(z - z.max()); qd /= qd.sum()
            p = PG.block_mass(m, x["q"], x["k"], lse, idx, nsel, 0, g, i)
            want += rel_entr(p, qd).sum()
    assert loss == pytest.approx(want, rel=1e-10)


def test_one_block_rows_have_no_loss_or_gradient(oracle_mod):
    """A row that reads one block (every row of block 0) has p = q = 1."""
    m, x, idx, nsel, lse = problem(seed=4)
    rows = [(0, g, i) for g in range(m.Hkv) for i in range(m.blk)]
    assert all(int(nsel[b, g, i]) == 1 for b, g, i in rows)
    loss, dqp, dkp = PG.loss_and_grad(m, x["qp"], x["kp"], x["q"], x["k"], lse, idx, nsel, rows=rows)
    assert abs(loss) < 1e-12 and np.abs(dqp).max() < 1e-12 and np.abs(dkp).max() < 1e-12
