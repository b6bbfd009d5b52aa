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
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import CONFIGS, make_inputs, sample_rows
from parity_util import compare, f32, odims, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("name,nsel_rows,nq_rows", [("32k", 256, 512), ("128k", 192, 384)])
def test_full_size(name, nsel_rows, nq_rows):
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
    compare("L rows", f32(lse)[b, h, i], lo[b, h, i])
    compare("dQ rows", f32(dq)[b, i, h], dqo[b, i, h])

    # ---- dK, dV of the last two KV blocks of every group: their selecting
    # queries are all in the last two query blocks, selected above
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
    dout = x["dout"].astype(np.float64)
    n = T
    for bb in range(cfg.B):
        for g in range(Hkv):
            kk = gdk[bb, :, g]
            vv = gdv[bb, :, g]
            tol_k = 5 * np.sqrt(n) * 2.0 ** -8 * np.sqrt((kk ** 2).mean()) + 1e-3
            tol_v = 5 * np.sqrt(n) * 2.0 ** -8 * np.sqrt((vv ** 2).mean()) + 1e-3
            assert np.abs(kk.sum(0)).max() <= tol_k, ("sum dK", np.abs(kk.sum(0)).max(), tol_k)
            want = dout[bb][:, g * G:(g + 1) * G].sum((0, 1))
            assert np.abs(vv.sum(0) - want).max() <= tol_v, ("sum dV", np.abs(vv.sum(0) - want).max(), tol_v)
