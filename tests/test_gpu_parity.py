"""Parity of the CUDA path (through the C ABI) with the CPU oracle on shapes
the oracle finishes in seconds: several tiles, ragged tails (down to a last
block of one row), every G the library supports (1, 2, 4, 8, 16), topk = 1,
topk >= number of blocks, a sequence shorter than one block, B > 1.

Proxy inputs sit on the 1/8 grid (exact_proxy) so that the proxy scores are
exact in any summation order: the GPU and the oracle then see identical
pooled scores and the block selection must match bit for bit, end to end.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import CONFIGS, Config, make_inputs
from parity_util import compare, f32, gpu_path, odims, oracle_inputs, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": CONFIGS["tiny"],
    "ragged_b2": Config("ragged_b2", B=2, T=1000, Hq=8, Hkv=2, d=128, dp=64, topk=3),
    "g1_d64": Config("g1_d64", B=1, T=640, Hq=2, Hkv=2, d=64, dp=16, topk=2),
    "g8": Config("g8", B=1, T=512, Hq=8, Hkv=1, d=128, dp=64, topk=2),
    "g16": Config("g16", B=1, T=384, Hq=16, Hkv=1, d=64, dp=48, topk=2),
    "dense": Config("dense", B=1, T=512, Hq=4, Hkv=1, d=128, dp=64, topk=8),
    "topk1": Config("topk1", B=1, T=640, Hq=4, Hkv=1, d=64, dp=32, topk=1),
    "short": Config("short", B=1, T=100, Hq=4, Hkv=1, d=64, dp=32, topk=2),
    "k5_ragged": Config("k5_ragged", B=1, T=1300, Hq=4, Hkv=1, d=128, dp=64, topk=5),
    "g2_one_row_tail": Config("g2_one_row_tail", B=3, T=129, Hq=4, Hkv=2, d=128, dp=64, topk=2),
}


def run_and_compare(cfg: Config, inp, report=None, input_scale=1.0, dq_scale=None):
    """input_scale: how much larger than N(0,1) the q/k inputs are; gradient
    rounding errors grow with it, so the absolute part of the bound does too
    (dq_scale, if given, for dQ alone).  dK and dV sum the rounding errors of
    G heads, which add in quadrature: their absolute bound grows as
    sqrt(G / 4) beyond the 4 heads per group of the stated workloads."""
    from parity_util import ABS_MAX
    kv_abs = ABS_MAX * input_scale * max(1.0, (cfg.G / 4) ** 0.5)
    dq_scale = input_scale if dq_scale is None else dq_scale
    dev = to_dev(inp)
    g = gpu_path(dev, cfg.topk, pooled=True)
    x = oracle_inputs(inp)
    m = odims(cfg)
    idx_o, nsel_o, pooled_o = O.select(m, x["qp"], x["kp"], want_pooled=True)
    # ---- Index Branch: identical pooled scores -> identical selection
    pg = f32(g["pooled"]).reshape(-1, m.nblk)
    assert np.array_equal(np.isfinite(pg), np.isfinite(pooled_o))
    fin = np.isfinite(pooled_o)
    assert np.array_equal(pg[fin], pooled_o[fin]), "pooled proxy scores differ"
    assert np.array_equal(g["nsel"].cpu().numpy(), nsel_o), "nsel differs"
    assert np.array_equal(g["idx"].cpu().numpy(), idx_o), "block selection differs"
    # ---- Main Branch
    o, lse = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o)
    dq, D = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], o, lse, idx_o, nsel_o)
    dk, dv = O.bwd_dkdv(m, x["q"], x["k"], x["v"], x["dout"], lse, D, idx_o, nsel_o)
    compare("O", f32(g["o"]), o, report=report)
    compare("L", f32(g["lse"]), lse, report=report, rel=0.0)   # fp32 output: plain 2e-2
    compare("dQ", f32(g["dq"]), dq, report=report, abs_max=ABS_MAX * dq_scale)
    compare("dK", f32(g["dk"]), dk, report=report, abs_max=kv_abs)
    compare("dV", f32(g["dv"]), dv, report=report, abs_max=kv_abs)
    return g


@pytest.mark.parametrize("name", list(CASES))
def test_parity(name):
    cfg = CASES[name]
    inp = make_inputs(cfg, seed=1, exact_proxy=True)
    run_and_compare(cfg, inp)


def test_parity_8k_group_bias_sampled():
    """The 8K workload (per-group low-rank proxy bias) at full size; the
    oracle runs on sampled query rows and sampled KV blocks."""
    from block_sparse_attention_09_b200.inputs import sample_rows
    cfg = CONFIGS["8k"]
    inp = make_inputs(cfg, seed=0, exact_proxy=True)
    dev = to_dev(inp)
    g = gpu_path(dev, cfg.topk)
    x = oracle_inputs(inp)
    m = odims(cfg)
    # every selection row (cheap: one row of proxy scores each)
    idx_o, nsel_o, _ = O.select(m, x["qp"], x["kp"])
    assert np.array_equal(g["idx"].cpu().numpy(), idx_o)
    assert np.array_equal(g["nsel"].cpu().numpy(), nsel_o)
    # groups select different blocks (the bias works as intended)
    assert not np.array_equal(idx_o[0, 0], idx_o[0, 1])
    rows = sample_rows(cfg.B * cfg.Hq * cfg.T, 1500, seed=3,
                       must=[0, cfg.T - 1, cfg.T * cfg.Hq - 1, 128, 129])
    o, lse = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o, rows=rows)
    dq, D = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], o, lse, idx_o, nsel_o, rows=rows)
    r = np.array(rows)
    h = (r // cfg.T) % cfg.Hq
    b = r // (cfg.T * cfg.Hq)
    i = r % cfg.T
    compare("O rows", f32(g["o"])[b, i, h], o[b, i, h])
    compare("L rows", f32(g["lse"])[b, h, i], lse[b, h, i], rel=0.0)
    compare("dQ rows", f32(g["dq"])[b, i, h], dq[b, i, h])
    # dK/dV on sampled blocks need L and D of every query that selected them
    # blocks whose selecting queries stay within an oracle budget; the most
    # selected buckets (block 0) first, then middle and last blocks
    cands = [0, m.nblk, 5 * m.nblk, 1, 17, m.nblk + 5, 3 * m.nblk + 40, m.nblk - 1, 4 * m.nblk + 63,
             8 * m.nblk - 1]
    need = np.zeros((cfg.B, cfg.Hkv, cfg.T), dtype=bool)
    blocks = []
    for bl in cands:
        n = bl % m.nblk
        bb, gg = divmod(bl // m.nblk, cfg.Hkv)
        sel = (idx_o[bb, gg] == n).any(axis=1)
        if need.sum() + sel.sum() > 6000 and blocks:
            continue
        need[bb, gg] |= sel
        blocks.append(bl)
    assert len(blocks) >= 5
    qrows = []
    for bb, gg, ii in zip(*np.nonzero(need)):
        for hh in range(gg * cfg.G, (gg + 1) * cfg.G):
            qrows.append((bb * cfg.Hq + hh) * cfg.T + ii)
    o2, lse2 = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o, rows=qrows)
    _, D2 = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], o2, lse2, idx_o, nsel_o, rows=qrows)
    dk, dv = O.bwd_dkdv(m, x["q"], x["k"], x["v"], x["dout"], lse2, D2, idx_o, nsel_o, blocks=blocks)
    for bl in blocks:
        n = bl % m.nblk
        bb, gg = divmod(bl // m.nblk, cfg.Hkv)
        sl = slice(n * 128, (n + 1) * 128)
        compare(f"dK blk {bl}", f32(g["dk"])[bb, sl, gg], dk[bb, sl, gg])
        compare(f"dV blk {bl}", f32(g["dv"])[bb, sl, gg], dv[bb, sl, gg])


def test_selection_float_inputs():
    """N(0,1) bf16 proxy inputs (sums rounded differently on each side):
    pooled scores agree to fp32 rounding; the GPU selection satisfies the
    selection rule on its own scores; any difference from the oracle's
    selection is a near-tie in the oracle's scores."""
    cfg = Config("f", B=2, T=2048, Hq=8, Hkv=2, d=64, dp=64, topk=5)
    inp = make_inputs(cfg, seed=4)
    from block_sparse_attention_09_b200 import msa
    idx, nsel, pooled = msa.proxy_select(inp["qp"].cuda(), inp["kp"].cuda(), cfg.topk, pooled=True, check=True)
    x = oracle_inputs(inp)
    m = odims(cfg)
    idx_o, nsel_o, pooled_o = O.select(m, x["qp"], x["kp"], want_pooled=True)
    pg = f32(pooled).reshape(-1, m.nblk)
    fin = np.isfinite(pooled_o)
    assert np.array_equal(np.isfinite(pg), fin)
    assert np.allclose(pg[fin], pooled_o[fin], rtol=1e-5, atol=1e-4)
    ig = idx.cpu().numpy().reshape(-1, cfg.topk)
    ng = nsel.cpu().numpy().reshape(-1)
    io = idx_o.reshape(-1, cfg.topk)
    mism = 0
    for r in range(ig.shape[0]):
        i = r % cfg.T
        bi = i // 128
        sel = [int(v) for v in ig[r, :ng[r]]]
        assert ng[r] == min(cfg.topk, bi + 1)
        assert sel == sorted(set(sel)) and bi in sel
        chosen = [v for v in sel if v != bi]
        rest = [v for v in range(bi) if v not in chosen]
        if chosen and rest:   # dominance on the GPU's own scores
            worst = min(chosen, key=lambda v: (pg[r, v], -v))
            best_rest = max(rest, key=lambda v: (pg[r, v], -v))
            assert (pg[r, worst] > pg[r, best_rest]) or (pg[r, worst] == pg[r, best_rest] and worst < best_rest)
        if not np.array_equal(ig[r], io[r]):
            mism += 1
            diff = set(ig[r]) ^ set(io[r])
            vals = [pooled_o[r, v] for v in diff if v >= 0]
            assert max(vals) - min(vals) <= 1e-4 * max(1.0, np.abs(vals).max()), (r, diff, vals)
    assert mism <= ig.shape[0] // 100


@pytest.mark.parametrize("topk", [48, 72])
def test_selection_both_shared_memory_layouts(topk):
    """The selection kernel splits shared memory between key stages and the
    maxima ring by topk: three stages and a deep ring while the heap is small
    (topk 48 here), two stages and a short ring above that (topk 72).  Both
    must select exactly what the oracle selects, for every row, over enough
    key blocks (100) that the ring wraps many times."""
    from block_sparse_attention_09_b200 import msa
    cfg = Config("sel", B=1, T=12800, Hq=8, Hkv=2, d=64, dp=32, topk=topk)
    inp = make_inputs(cfg, seed=11, exact_proxy=True, parts=("qp", "kp"))
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], topk, check=True)
    m = O.Dims(B=cfg.B, T=cfg.T, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, dp=cfg.dp, topk=topk)
    io, no, _ = O.select(m, inp["qp"].float().numpy(), inp["kp"].float().numpy())
    assert np.array_equal(nsel.cpu().numpy(), no)
    assert np.array_equal(idx.cpu().numpy(), io)


@pytest.mark.parametrize("dp", [8, 24, 40, 56])
def test_selection_proxy_dims_not_multiple_of_16(dp):
    """dp may be any multiple of 8 up to 64: the last K-step of the proxy MMA
    then covers columns past dp, which the tensor map zero-fills.  The
    selection must still match the oracle bit for bit (ragged T, B = 2)."""
    from block_sparse_attention_09_b200 import msa
    cfg = Config("dp", B=2, T=2000, Hq=4, Hkv=2, d=64, dp=dp, topk=5)
    inp = make_inputs(cfg, seed=12, exact_proxy=True, parts=("qp", "kp"))
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    m = O.Dims(B=cfg.B, T=cfg.T, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, dp=dp, topk=cfg.topk)
    io, no, _ = O.select(m, inp["qp"].float().numpy(), inp["kp"].float().numpy())
    assert np.array_equal(nsel.cpu().numpy(), no)
    assert np.array_equal(idx.cpu().numpy(), io)


def test_equal_scores_pick_lowest_blocks():
    cfg = Config("ties", B=1, T=1536, Hq=4, Hkv=1, d=64, dp=32, topk=4)
    inp = make_inputs(cfg, seed=2, exact_proxy=True)
    inp["kp"] = torch.full_like(inp["kp"], 0.5)
    g = gpu_path(to_dev(inp), cfg.topk)
    idx = g["idx"].cpu().numpy()
    for i in range(cfg.T):
        bi = i // 128
        want = list(range(min(bi, cfg.topk - 1))) + [bi]
        assert idx[0, 0, i, :len(want)].tolist() == want


def test_far_best_scores_use_exact_fallback():
    """Rows whose best score lies far above the score of their own key (here
    about 136 nats: keys alternate between +2 and -2 along q, so odd queries
    see their own key at the bottom) overflow the forward's fixed shift and
    must be redone exactly -- and still match the oracle."""
    from block_sparse_attention_09_b200 import msa
    cfg = Config("farbest", B=1, T=768, Hq=4, Hkv=1, d=128, dp=32, topk=3)
    inp = make_inputs(cfg, seed=5, exact_proxy=True)
    g = torch.Generator().manual_seed(55)
    q = 3.0 + 0.1 * torch.randn(inp["q"].shape, generator=g)
    sign = torch.where(torch.arange(cfg.T) % 2 == 0, 1.0, -1.0).view(1, -1, 1, 1)
    k = 2.0 * sign + 0.05 * torch.randn(inp["k"].shape, generator=g)
    inp["q"] = q.to(torch.bfloat16)
    inp["k"] = k.to(torch.bfloat16)
    run_and_compare(cfg, inp, input_scale=6.0)
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    dims = msa.make_dims(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.dp, cfg.topk)
    ws = msa.workspace(dims, msa.MSA_FWD, dev["q"].device)
    msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, ws=ws, check=True)
    assert msa.fallback_rows(ws) > 0


def test_key_outliers_need_no_fallback():
    """A few keys with about 8x the norm of the others (attention-sink-like)
    must not push the rows that read them onto the exact fallback: the
    forward's shift is bracketed by the own key's score, not only by a norm
    bound.  Parity on the whole path as well."""
    from block_sparse_attention_09_b200 import msa
    cfg = Config("outliers", B=1, T=4096, Hq=8, Hkv=2, d=128, dp=64, topk=8, k_outliers=16)
    inp = make_inputs(cfg, seed=3, exact_proxy=True)
    # dQ_i = scale sum_j dS_ij k_j: where an 8x key carries much of a row's
    # weight, the bf16 rounding of dS (and of O inside D = dO.O) is multiplied
    # by that key, and dS itself is a difference of two terms of the key's
    # size -- so dQ's absolute error bound is 8 x 2 times the N(0,1) one.
    run_and_compare(cfg, inp, input_scale=8.0, dq_scale=16.0)
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    dims = msa.make_dims(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.dp, cfg.topk)
    ws = msa.workspace(dims, msa.MSA_FWD, dev["q"].device)
    msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, ws=ws, check=True)
    assert msa.fallback_rows(ws) == 0


def test_malformed_indices_are_reported_not_used():
    from block_sparse_attention_09_b200 import msa
    cfg = Config("bad", B=1, T=512, Hq=4, Hkv=1, d=64, dp=32, topk=2)
    inp = make_inputs(cfg, seed=6)
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    bad = idx.clone()
    bad[0, 0, 300, 0] = 3        # block after the query's own (300 // 128 = 2)
    bad[0, 0, 10, 0] = -5
    with pytest.raises(msa.MsaError) as e:
        msa.fwd(dev["q"], dev["k"], dev["v"], bad, nsel, check=True)
    assert e.value.code == -9
    # the device is still healthy and a good call still works
    msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, check=True)
