"""Parity at the full workload sizes, in the launch configuration the
benchmark times (whole tensors on the GPU, one call per phase, one workspace
shared by the forward and the backward, which reuses the forward's inverse
index).

The oracle cannot run every row at T = 128K, so it checks sampled outputs it
computes one by one -- the selection of sampled queries (bit-exact: proxy
inputs on the 1/8 grid make every proxy score exact), O, L and dQ of sampled
query rows, dK and dV of the last KV blocks (whose selecting queries the
oracle can enumerate) -- and, over the whole tensors, identities that hold at
any size: softmax rows sum to one, so sum_j dV_j = sum_{i,h} dO_ih per group,
and sum_j dS_ij = 0, so sum_j dK_j = 0.

A second backward, in the same launch configuration, takes dO restricted to
a seeded set S of query tokens spread over the whole sequence (dO = 0
elsewhere).  Rows outside S then contribute exactly zero to every gradient
(dV gains P * 0, and dS = P (dO.v - dO.O) = 0), so dK and dV of ANY block are
sums over the S rows that selected it, which the oracle enumerates from its
own selection of those rows.  That checks, element by element and with the
unrounded fp32 dK/dV (MSA_DKV_F32) against the plain max-abs bound 2e-2, the
heavily shared blocks -- block 0, the block the S rows select most, a
mid-sequence block -- whose partials arrive from every query range of the
kernels' work items; dQ of every row outside S must be exactly zero.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import CONFIGS, make_inputs, sample_rows
from parity_util import compare, f32, odims, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("name,nsel_rows,nq_rows,s_tokens", [("32k", 256, 512, 1024), ("128k", 192, 384, 512)])
def test_full_size(name, nsel_rows, nq_rows, s_tokens, last_blocks=True):
    from block_sparse_attention_09_b200 import msa
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, seed=11, exact_proxy=True)
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    ws = msa.step_workspace(msa.make_dims(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.dp, cfg.topk), dev["q"].device)
    o, lse = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, ws=ws, check=True)
    dq, dk, dv = msa.bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, idx, nsel, ws=ws, check=True,
                         reuse_index=True)
    torch.cuda.synchronize()
    g_idx, g_nsel = idx.cpu().numpy(), nsel.cpu().numpy()
    x = {k: v.float().numpy() for k, v in inp.items()}
    m = odims(cfg)
    T, G, Hq, Hkv, nb = cfg.T, cfg.G, cfg.Hq, cfg.Hkv, m.nblk

    # ---- selection of sampled queries, plus every query of the last two blocks
    last = [(b * Hkv + g) * T + i for b in range(cfg.B) for g in range(Hkv) for i in range(T - 256, T)]
    if not last_blocks:   # the masked-dO check below covers dK/dV; sample the last blocks' rows
        last = last[::64]
    srows = sample_rows(cfg.B * Hkv * T, nsel_rows, seed=5, must=last)
    idx_o, nsel_o, _ = O.select(m, x["qp"], x["kp"], rows=srows)
    fi, fn = g_idx.reshape(-1, cfg.topk), g_nsel.reshape(-1)
    oi, on = idx_o.reshape(-1, cfg.topk), nsel_o.reshape(-1)
    for r in srows:
        assert np.array_equal(fi[r], oi[r]) and fn[r] == on[r], f"selection differs at row {r}"

    # ---- O, L, dQ for the heads of sampled (b, g, i)
    sample = sample_rows(cfg.B * Hkv * T, nq_rows // G, seed=6)
    qrows = []
    for r in sample:
        i, bg = r % T, r // T
        b, g = divmod(bg, Hkv)
        qrows += [(b * Hq + g * G + hh) * T + i for hh in range(G)]
    # the oracle's own selection for those rows
    O.select(m, x["qp"], x["kp"], rows=sample, idx=idx_o, nsel=nsel_o)
    oo, lo = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o, rows=qrows)
    dqo, Do = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], oo, lo, idx_o, nsel_o, rows=qrows)
    r = np.array(qrows)
    h, b, i = (r // T) % Hq, r // (T * Hq), r % T
    compare("O rows", f32(o)[b, i, h], oo[b, i, h])
    compare("L rows", f32(lse)[b, h, i], lo[b, h, i], rel=0.0)
    compare("dQ rows", f32(dq)[b, i, h], dqo[b, i, h])

    # ---- dK, dV of the last two KV blocks of every group: their selecting
    # queries are all in the last two query blocks, selected above
    if last_blocks:
        blocks = [(b * Hkv + g) * nb + n for b in range(cfg.B) for g in range(Hkv) for n in (nb - 2, nb - 1)]
        lrows = [(b * Hq + g * G + hh) * T + i for b in range(cfg.B) for g in range(Hkv)
                 for hh in range(G) for i in range(T - 256, T)]
        o2, l2 = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o, rows=lrows)
        _, D2 = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], o2, l2, idx_o, nsel_o, rows=lrows)
        dko, dvo = O.bwd_dkdv(m, x["q"], x["k"], x["v"], x["dout"], l2, D2, idx_o, nsel_o, blocks=blocks)
        sl = slice(T - 256, T)
        compare("dK last blocks", f32(dk)[:, sl], dko[:, sl])
        compare("dV last blocks", f32(dv)[:, sl], dvo[:, sl])

    # ---- whole-tensor identities (bf16 outputs: each element carries up to
    # 2^-8 relative rounding, so a sum of n of them may be off by about
    # sqrt(n) * 2^-8 * rms; the bound allows five times that)
    gdk = dk.double().cpu().numpy()
    gdv = dv.double().cpu().numpy()
    n = T
    for bb in range(cfg.B):
        for g in range(Hkv):
            kk = gdk[bb, :, g]
            vv = gdv[bb, :, g]
            tol_k = 5 * np.sqrt(n) * 2.0 ** -8 * np.sqrt((kk ** 2).mean()) + 1e-3
            tol_v = 5 * np.sqrt(n) * 2.0 ** -8 * np.sqrt((vv ** 2).mean()) + 1e-3
            assert np.abs(kk.sum(0)).max() <= tol_k, ("sum dK", np.abs(kk.sum(0)).max(), tol_k)
            want = x["dout"][bb][:, g * G:(g + 1) * G].sum((0, 1), dtype=np.float64)
            assert np.abs(vv.sum(0) - want).max() <= tol_v, ("sum dV", np.abs(vv.sum(0) - want).max(), tol_v)

    # ---- masked dO: heavily shared blocks, fp32 dK/dV, strict bound
    masked_dkdv_check(cfg, inp, x, dev, idx, nsel, o, lse, ws, s_tokens)


def masked_dkdv_check(cfg, inp, x, dev, idx, nsel, o, lse, ws, s_tokens):
    from block_sparse_attention_09_b200 import msa
    m = odims(cfg)
    T, G, Hq, Hkv, nb = cfg.T, cfg.G, cfg.Hq, cfg.Hkv, m.nblk
    toks = np.array(sample_rows(T, s_tokens, seed=21, must=[0, T // 2, T - 1]), dtype=np.int64)
    keep = np.zeros(T, dtype=np.float32)
    keep[toks] = 1.0
    dout_m = inp["dout"].float() * torch.from_numpy(keep).view(1, T, 1, 1)
    dout_m = dout_m.to(torch.bfloat16)
    dq_m, dk_m, dv_m = msa.bwd(dev["q"], dev["k"], dev["v"], o, dout_m.cuda(), lse, idx, nsel, ws=ws, check=True,
                               reuse_index=True, dkv_f32=True)
    torch.cuda.synchronize()
    assert dk_m.dtype == torch.float32
    # rows outside S: dQ exactly zero
    outside = np.ones(T, dtype=bool)
    outside[toks] = False
    assert not f32(dq_m)[:, outside].any(), "dQ of rows with dO = 0 is not zero"

    # the oracle on the S rows only: its own selection, O, L, D
    srows = [(b * Hkv + g) * T + int(t) for b in range(cfg.B) for g in range(Hkv) for t in toks]
    idx_s, nsel_s, _ = O.select(m, x["qp"], x["kp"], rows=srows)
    qrows = [(b * Hq + g * G + hh) * T + int(t) for b in range(cfg.B) for g in range(Hkv) for hh in range(G)
             for t in toks]
    xm = dict(x)
    xm["dout"] = dout_m.float().numpy()
    o_s, l_s = O.fwd(m, x["q"], x["k"], x["v"], idx_s, nsel_s, rows=qrows)
    _, D_s = O.bwd_dq(m, x["q"], x["k"], x["v"], xm["dout"], o_s, l_s, idx_s, nsel_s, rows=qrows)
    blocks, spans = [], []
    for b in range(cfg.B):
        for g in range(Hkv):
            sel = idx_s[b, g, toks]                           # [S, topk]
            counts = np.bincount(sel[sel >= 0].ravel(), minlength=nb)
            for n in sorted({0, int(counts.argmax()), nb // 2}):
                who = toks[(sel == n).any(axis=1)]
                # the query eighths of the sequence its S partials come from
                spans.append(len(set((who * 8 // T).tolist())))
                blocks.append((b * Hkv + g) * nb + n)
    assert max(spans) >= 4, ("shared blocks receive partials from few query ranges", spans)
    dko, dvo = O.bwd_dkdv(m, x["q"], x["k"], x["v"], xm["dout"], l_s, D_s, idx_s, nsel_s, blocks=blocks)
    gk, gv = f32(dk_m), f32(dv_m)
    for bl in blocks:
        n = bl % nb
        b, g = divmod(bl // nb, Hkv)
        sl = slice(n * 128, min((n + 1) * 128, T))
        compare(f"dK32 blk {n} g{g}", gk[b, sl, g], dko[b, sl, g], rel=0.0)
        compare(f"dV32 blk {n} g{g}", gv[b, sl, g], dvo[b, sl, g], rel=0.0)
