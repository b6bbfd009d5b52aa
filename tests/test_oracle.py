"""Pins for the CPU oracle (no GPU).

The oracle is checked here against things other than itself:
* hand-derived selection cases (tests/golden/select_cases.json);
* brute force with whole matrices: the T x T proxy score matrix pooled by
  numpy, dense attention with an explicit per-query mask, torch's own
  scaled_dot_product_attention when every block is selected, torch autograd
  on the masked dense formulation;
* central finite differences of <dO, O>;
* invariants that hold for any input (dominance of the selected set, sums of
  dK and dV, constant V, zero Q).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from oracle import Dims

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_inputs(m: Dims, seed: int, grid: bool = False, scale: float = 1.0):
    rng = np.random.default_rng(seed)

    def r(*shape):
        x = rng.standard_normal(shape).astype(np.float32) * scale
        if grid:
            x = np.clip(np.round(x * 8), -64, 64).astype(np.float32) / 8
        return x

    return dict(
        qp=r(m.B, m.T, m.Hkv, m.dp), kp=r(m.B, m.T, m.Hkv, m.dp),
        q=r(m.B, m.T, m.Hq, m.d), k=r(m.B, m.T, m.Hkv, m.d), v=r(m.B, m.T, m.Hkv, m.d),
        dout=r(m.B, m.T, m.Hq, m.d))


# ---------------------------------------------------------------- brute force
def bf_pooled(m: Dims, qp, kp):
    """Whole causal proxy score matrix, then a max over each block's columns."""
    out = np.full((m.B, m.Hkv, m.T, m.nblk), -np.inf, dtype=np.float64)
    for b in range(m.B):
        for g in range(m.Hkv):
            S = qp[b, :, g, :].astype(np.float64) @ kp[b, :, g, :].astype(np.float64).T
            S[np.triu_indices(m.T, 1)] = -np.inf
            for n in range(m.nblk):
                out[b, g, :, n] = S[:, n * m.blk:(n + 1) * m.blk].max(axis=1)
    return out.astype(np.float32)


def sel_mask(m: Dims, idx, nsel, b, g):
    """T x T boolean: query i may read key j."""
    M = np.zeros((m.T, m.T), dtype=bool)
    for i in range(m.T):
        for n in idx[b, g, i, :nsel[b, g, i]]:
            M[i, n * m.blk:(n + 1) * m.blk] = True
    return M & np.tril(np.ones((m.T, m.T), dtype=bool))


def bf_fwd_torch(m: Dims, x, idx, nsel, grad=False):
    """Dense attention with an explicit mask, in float64 torch (autograd-able)."""
    scale = 1.0 / np.sqrt(m.d)
    q = torch.tensor(x["q"], dtype=torch.float64, requires_grad=grad)
    k = torch.tensor(x["k"], dtype=torch.float64, requires_grad=grad)
    v = torch.tensor(x["v"], dtype=torch.float64, requires_grad=grad)
    outs, lses = [], []
    for b in range(m.B):
        ob, lb = [], []
        for h in range(m.Hq):
            g = h // m.G
            M = torch.tensor(sel_mask(m, idx, nsel, b, g))
            S = scale * q[b, :, h, :] @ k[b, :, g, :].T
            S = S.masked_fill(~M, float("-inf"))
            L = torch.logsumexp(S, dim=1)
            P = torch.softmax(S, dim=1)
            ob.append(P @ v[b, :, g, :])
            lb.append(L)
        outs.append(torch.stack(ob, dim=1))
        lses.append(torch.stack(lb, dim=0))
    o = torch.stack(outs, dim=0)
    lse = torch.stack(lses, dim=0)
    return q, k, v, o, lse


# ---------------------------------------------------------------- selection
def test_select_golden_cases():
    with open(os.path.join(HERE, "golden", "select_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        pooled = np.array([c["pooled"]], dtype=np.float32)
        idx, nsel = O.select_from_pooled(pooled, [c["bi"]], c["topk"])
        assert idx[0].tolist() == c["idx"], c["why"]
        assert int(nsel[0]) == c["nsel"], c["why"]


def test_golden_selection_window_cases():
    """Hand-derived cases for the forced window / dilation pattern."""
    with open(os.path.join(HERE, "golden", "select_window_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        pooled = np.array([c["pooled"]], dtype=np.float32)
        idx, nsel = O.select_from_pooled(pooled, [c["bi"]], c["topk"], c["window"], c["dilation"])
        assert idx[0].tolist() == c["idx"], c["why"]
        assert int(nsel[0]) == c["nsel"], c["why"]


def test_window_one_is_the_plain_rule():
    """window 1 forces only the own block: the plain rule, for any dilation."""
    rng = np.random.default_rng(3)
    pooled = rng.integers(-3, 4, size=(400, 40)).astype(np.float32)   # many ties
    bi = rng.integers(0, 40, size=400).astype(np.int32)
    for topk in (1, 3, 8):
        a, na = O.select_from_pooled(pooled, bi, topk)
        for dil in (1, 2, 5):
            b, nb = O.select_from_pooled(pooled, bi, topk, 1, dil)
            assert np.array_equal(a, b) and np.array_equal(na, nb)


def test_window_selection_invariants():
    """For any scores: the forced blocks that exist are kept, the count is
    min(topk, bi+1), and every kept free block ranks above every dropped free
    block (higher score, or equal score and lower id)."""
    rng = np.random.default_rng(4)
    nb = 48
    pooled = rng.integers(-4, 5, size=(300, nb)).astype(np.float32)
    bi = rng.integers(0, nb, size=300).astype(np.int32)
    for topk, window, dil in ((6, 3, 1), (8, 4, 3), (5, 5, 2), (12, 2, 7)):
        idx, nsel = O.select_from_pooled(pooled, bi, topk, window, dil)
        for r in range(len(bi)):
            b_ = int(bi[r])
            sel = [int(x) for x in idx[r, :nsel[r]]]
            assert nsel[r] == min(topk, b_ + 1)
            assert sel == sorted(set(sel)) and all(0 <= x <= b_ for x in sel)
            assert all(x == -1 for x in idx[r, nsel[r]:])
            if b_ + 1 <= topk:
                assert sel == list(range(b_ + 1))
                continue
            forced = {b_ - m * dil for m in range(window) if b_ - m * dil >= 0}
            assert forced <= set(sel)
            free_kept = [x for x in sel if x not in forced]
            free_dropped = [x for x in range(b_ + 1) if x not in forced and x not in sel]
            assert len(free_kept) == topk - len(forced)
            for k in free_kept:
                for d_ in free_dropped:
                    sk, sd = pooled[r, k], pooled[r, d_]
                    assert sk > sd or (sk == sd and k < d_)


def check_selection_invariants(pooled_row, bi, topk, idx_row, nsel):
    sel = [int(x) for x in idx_row[:nsel]]
    assert nsel == min(topk, bi + 1)
    assert all(x == -1 for x in idx_row[nsel:])
    assert sel == sorted(set(sel)), "ascending and distinct"
    assert bi in sel, "own block kept"
    assert all(0 <= x <= bi for x in sel)
    chosen = [x for x in sel if x != bi]
    rest = [n for n in range(bi) if n not in chosen]
    for x in chosen:           # every chosen block beats every unchosen one
        for u in rest:
            px, pu = pooled_row[x], pooled_row[u]
            assert px > pu or (px == pu and x < u), (x, u, px, pu)


@pytest.mark.parametrize("blk,T,topk", [(4, 40, 3), (4, 37, 5), (128, 1024, 4), (128, 700, 2)])
def test_pool_matches_full_score_matrix(oracle_mod, blk, T, topk):
    m = Dims(B=2, T=T, Hq=4, Hkv=2, d=16, dp=32, topk=topk, blk=blk)
    x = rand_inputs(m, seed=blk + T, grid=True)
    idx, nsel, pooled = O.select(m, x["qp"], x["kp"], want_pooled=True)
    ref = bf_pooled(m, x["qp"], x["kp"]).reshape(-1, m.nblk)
    # grid inputs: every proxy score is exact, so equality is exact
    assert np.array_equal(pooled, ref)
    for r in range(pooled.shape[0]):
        i = r % m.T
        check_selection_invariants(pooled[r], i // blk, topk, idx.reshape(-1, topk)[r],
                                   int(nsel.reshape(-1)[r]))


@pytest.mark.parametrize("window,dil", [(3, 1), (4, 2), (2, 5)])
def test_select_window_end_to_end(oracle_mod, window, dil):
    """Proxy scores -> pool -> windowed selection agrees with the rule applied
    to the numpy-pooled full score matrix (the pooling pin above)."""
    m = Dims(B=1, T=1280, Hq=2, Hkv=2, d=16, dp=32, topk=6, blk=128, window=window, dilation=dil)
    x = rand_inputs(m, seed=window * 10 + dil, grid=True)
    idx, nsel, _ = O.select(m, x["qp"], x["kp"])
    ref = bf_pooled(m, x["qp"], x["kp"]).reshape(-1, m.nblk)
    bi = (np.arange(ref.shape[0]) % m.T) // m.blk
    ridx, rnsel = O.select_from_pooled(ref, bi, m.topk, window, dil)
    assert np.array_equal(idx.reshape(-1, m.topk), ridx)
    assert np.array_equal(nsel.reshape(-1), rnsel)


def test_pool_float_inputs_close(oracle_mod):
    m = Dims(B=1, T=512, Hq=2, Hkv=1, d=16, dp=64, topk=2)
    x = rand_inputs(m, seed=3)
    _, _, pooled = O.select(m, x["qp"], x["kp"], want_pooled=True)
    ref = bf_pooled(m, x["qp"], x["kp"]).reshape(-1, m.nblk)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(pooled))
    assert np.allclose(pooled[fin], ref[fin], rtol=1e-6, atol=1e-6)


def test_select_many_ties(oracle_mod):
    """Proxy keys all equal: every block pools to the same score, so the
    selection must be the lowest topk-1 blocks plus the own block."""
    m = Dims(B=1, T=1024, Hq=1, Hkv=1, d=16, dp=32, topk=3)
    x = rand_inputs(m, seed=5, grid=True)
    x["kp"][:] = 0.5
    idx, nsel, _ = O.select(m, x["qp"], x["kp"])
    for i in range(m.T):
        bi = i // 128
        want = list(range(min(bi, 2))) + [bi]
        assert idx[0, 0, i, :nsel[0, 0, i]].tolist() == want


def test_select_row_subset_matches_all(oracle_mod):
    m = Dims(B=2, T=640, Hq=4, Hkv=2, d=16, dp=32, topk=3)
    x = rand_inputs(m, seed=11)
    idx_all, nsel_all, _ = O.select(m, x["qp"], x["kp"])
    rows = [0, 5, 700, 1279, 2 * 640 + 3, 4 * 640 - 1]
    idx_s, nsel_s, _ = O.select(m, x["qp"], x["kp"], rows=rows)
    f_all, f_s = idx_all.reshape(-1, 3), idx_s.reshape(-1, 3)
    for r in rows:
        assert f_all[r].tolist() == f_s[r].tolist()
        assert nsel_all.reshape(-1)[r] == nsel_s.reshape(-1)[r]


# ---------------------------------------------------------------- forward
@pytest.mark.parametrize("T,topk,blk", [(48, 3, 8), (45, 2, 8), (256, 2, 128)])
def test_fwd_matches_masked_dense(oracle_mod, T, topk, blk):
    m = Dims(B=2, T=T, Hq=4, Hkv=2, d=16, dp=8, topk=topk, blk=blk)
    x = rand_inputs(m, seed=T)
    idx, nsel, _ = O.select(m, x["qp"], x["kp"])
    o, lse = O.fwd(m, x["q"], x["k"], x["v"], idx, nsel)
    _, _, _, o_ref, lse_ref = bf_fwd_torch(m, x, idx, nsel)
    assert np.allclose(o, o_ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, lse_ref.numpy(), rtol=1e-12, atol=1e-12)


def test_fwd_all_blocks_is_causal_sdpa(oracle_mod):
    """topk >= number of blocks: MSA reduces to dense causal GQA attention."""
    m = Dims(B=1, T=40, Hq=4, Hkv=2, d=8, dp=4, topk=5, blk=8)
    x = rand_inputs(m, seed=1)
    idx, nsel, _ = O.select(m, x["qp"], x["kp"])
    o, _ = O.fwd(m, x["q"], x["k"], x["v"], idx, nsel)
    q = torch.tensor(x["q"], dtype=torch.float64).permute(0, 2, 1, 3)
    k = torch.tensor(x["k"], dtype=torch.float64).permute(0, 2, 1, 3)
    v = torch.tensor(x["v"], dtype=torch.float64).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                           enable_gqa=True)
    assert np.allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12)


def test_fwd_constant_v_and_zero_q(oracle_mod):
    m = Dims(B=1, T=300, Hq=2, Hkv=1, d=8, dp=16, topk=2)
    x = rand_inputs(m, seed=9)
    idx, nsel, _ = O.select(m, x["qp"], x["kp"])
    xv = dict(x)
    xv["v"] = np.broadcast_to(np.arange(m.d, dtype=np.float32), x["v"].shape).copy()
    o, _ = O.fwd(m, xv["q"], xv["k"], xv["v"], idx, nsel)
    assert np.allclose(o, np.arange(m.d)[None, None, None, :], atol=1e-12)
    xq = dict(x)
    xq["q"] = np.zeros_like(x["q"])
    o, lse = O.fwd(m, xq["q"], xq["k"], xq["v"], idx, nsel)
    for i in (0, 1, 127, 128, 200, 299):
        keys = [j for n in idx[0, 0, i, :nsel[0, 0, i]] for j in range(n * 128, (n + 1) * 128)
                if j <= i and j < m.T]
        mean = x["v"][0, keys, 0, :].astype(np.float64).mean(axis=0)
        assert np.allclose(o[0, i, 0], mean, atol=1e-12)
        assert np.isclose(lse[0, 0, i], np.log(len(keys)), atol=1e-12)


# ---------------------------------------------------------------- backward
def test_bwd_matches_autograd(oracle_mod):
    m = Dims(B=2, T=44, Hq=4, Hkv=2, d=8, dp=4, topk=2, blk=8)
    x = rand_inputs(m, seed=21)
    r = O.full(m, x["qp"], x["kp"], x["q"], x["k"], x["v"], x["dout"])
    q, k, v, o, _ = bf_fwd_torch(m, x, r["idx"], r["nsel"], grad=True)
    (o * torch.tensor(x["dout"], dtype=torch.float64)).sum().backward()
    assert np.allclose(r["dq"], q.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(r["dk"], k.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(r["dv"], v.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_bwd_finite_differences(oracle_mod):
    """Central differences of L(q,k,v) = <dO, O> at float32-exact steps."""
    m = Dims(B=1, T=256, Hq=2, Hkv=1, d=16, dp=8, topk=2)
    x = rand_inputs(m, seed=33)
    r = O.full(m, x["qp"], x["kp"], x["q"], x["k"], x["v"], x["dout"])
    dout = x["dout"].astype(np.float64)
    rng = np.random.default_rng(0)
    eps = np.float32(2.0 ** -16)

    def loss(xx):
        o, _ = O.fwd(m, xx["q"], xx["k"], xx["v"], r["idx"], r["nsel"])
        return float((o * dout).sum())

    for name, grad in (("q", r["dq"]), ("k", r["dk"]), ("v", r["dv"])):
        gmax = np.abs(grad).max()
        for _ in range(12):
            pos = tuple(int(rng.integers(0, s)) for s in x[name].shape)
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][pos] += eps
            xm[name][pos] -= eps
            step = float(xp[name][pos]) - float(xm[name][pos])
            fd = (loss(xp) - loss(xm)) / step
            assert abs(fd - grad[pos]) <= 1e-6 * max(gmax, 1.0), (name, pos, fd, grad[pos])


def test_bwd_invariants(oracle_mod):
    m = Dims(B=2, T=384, Hq=4, Hkv=2, d=16, dp=16, topk=2)
    x = rand_inputs(m, seed=44)
    r = O.full(m, x["qp"], x["kp"], x["q"], x["k"], x["v"], x["dout"])
    dout = x["dout"].astype(np.float64)
    for b in range(m.B):
        for g in range(m.Hkv):
            heads = list(range(g * m.G, (g + 1) * m.G))
            # rows of P sum to one  ->  sum_j dV_j = sum_i sum_h dO_ih
            assert np.allclose(r["dv"][b, :, g].sum(0), dout[b][:, heads].sum((0, 1)), atol=1e-9)
            # sum_j dS_ij = 0 per row  ->  sum_j dK_j = 0
            assert np.abs(r["dk"][b, :, g].sum(0)).max() < 1e-9
    # constant V: every score gradient vanishes
    xv = dict(x)
    xv["v"] = np.ones_like(x["v"]) * 0.75
    rv = O.full(m, xv["qp"], xv["kp"], xv["q"], xv["k"], xv["v"], xv["dout"])
    assert np.abs(rv["dq"]).max() < 1e-12 and np.abs(rv["dk"]).max() < 1e-12


def test_bwd_block_subset_matches_all(oracle_mod):
    m = Dims(B=1, T=512, Hq=4, Hkv=2, d=16, dp=16, topk=2)
    x = rand_inputs(m, seed=55)
    r = O.full(m, x["qp"], x["kp"], x["q"], x["k"], x["v"], x["dout"])
    blocks = [1, 3, 4 + 2]
    dk, dv = O.bwd_dkdv(m, x["q"], x["k"], x["v"], x["dout"], r["lse"], r["D"], r["idx"],
                        r["nsel"], blocks=blocks)
    for bl in blocks:
        g, n = divmod(bl, m.nblk)
        sl = slice(n * 128, (n + 1) * 128)
        assert np.array_equal(dk[0, sl, g], r["dk"][0, sl, g])
        assert np.array_equal(dv[0, sl, g], r["dv"][0, sl, g])


def test_row_contributions_sum_to_block_gradients(oracle_mod):
    """dK/dV built per KV block equal the sum of every query row's own
    contributions (two different loop orders over the same definition)."""
    m = Dims(B=1, T=300, Hq=4, Hkv=2, d=8, dp=8, topk=2)
    x = rand_inputs(m, seed=66)
    r = O.full(m, x["qp"], x["kp"], x["q"], x["k"], x["v"], x["dout"])
    dkr, dvr = O.bwd_kv_rows(m, x["q"], x["k"], x["v"], x["dout"], r["lse"], r["D"], r["idx"],
                             r["nsel"], rows=None)
    dk = np.zeros_like(r["dk"])
    dv = np.zeros_like(r["dv"])
    for row in range(m.B * m.Hq * m.T):
        i = row % m.T
        h = (row // m.T) % m.Hq
        b = row // (m.T * m.Hq)
        g = h // m.G
        keys = [j for n in r["idx"][b, g, i, :r["nsel"][b, g, i]] for j in range(n * 128, (n + 1) * 128)
                if j <= i]
        for t, j in enumerate(keys):
            dk[b, j, g] += dkr[row, t]
            dv[b, j, g] += dvr[row, t]
    assert np.allclose(dk, r["dk"], atol=1e-12)
    assert np.allclose(dv, r["dv"], atol=1e-12)
