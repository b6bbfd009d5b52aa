"""GPU parity of the decode path (msa_decode): one new token per sequence
against caches must give exactly what the training-path definitions give for
the last row of a sequence of that length -- the oracle's selection of that
row, bit for bit (grid proxy inputs make every proxy score exact), and its
O and L within the bf16 tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import Config, make_inputs
from parity_util import compare, oracle_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # name, config, lens (None: all T), window, dilation
    ("ragged_g4", Config("ragged_g4", B=3, T=3000, Hq=8, Hkv=2, d=128, dp=64, topk=6), [3000, 2049, 1], 1, 1),
    ("g16_d64", Config("g16_d64", B=2, T=2304, Hq=16, Hkv=1, d=64, dp=32, topk=4), [2304, 129], 1, 1),
    ("window", Config("window", B=2, T=4096, Hq=4, Hkv=1, d=64, dp=64, topk=8), [4096, 3333], 3, 2),
    ("few_blocks", Config("few_blocks", B=1, T=700, Hq=4, Hkv=1, d=128, dp=64, topk=8), None, 1, 1),
    ("g1_big_topk", Config("g1_big_topk", B=1, T=20000, Hq=2, Hkv=2, d=128, dp=48, topk=100), [19999], 1, 1),
]


@pytest.mark.parametrize("name,cfg,lens,window,dil", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_last_row(name, cfg, lens, window, dil):
    from block_sparse_attention_09_b200 import msa
    inp = make_inputs(cfg, seed=31, exact_proxy=True)
    ln = lens if lens is not None else [cfg.T] * cfg.B
    dev = {k: v.cuda() for k, v in inp.items()}
    # the new token of sequence b is its last cached position
    q = torch.stack([dev["q"][b, ln[b] - 1] for b in range(cfg.B)]).contiguous()
    qp = torch.stack([dev["qp"][b, ln[b] - 1] for b in range(cfg.B)]).contiguous()
    lens_t = torch.tensor(ln, dtype=torch.int32, device="cuda") if lens is not None else None
    o, lse, idx, nsel = msa.decode(q, qp, dev["k"], dev["v"], dev["kp"], cfg.topk, lens=lens_t, window=window,
                                   dilation=dil, check=True)
    torch.cuda.synchronize()
    o, lse, idx, nsel = o.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy(), nsel.cpu().numpy()
    x = oracle_inputs(inp)
    oo_all, lo_all = [], []
    for b in range(cfg.B):
        L = ln[b]
        m = O.Dims(B=1, T=L, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, dp=cfg.dp, topk=cfg.topk, window=window, dilation=dil)
        xb = {k: np.ascontiguousarray(v[b:b + 1, :L]) for k, v in x.items()}
        idx_o, nsel_o, _ = O.select(m, xb["qp"], xb["kp"], rows=[g * L + L - 1 for g in range(cfg.Hkv)])
        assert np.array_equal(idx[b], idx_o[0, :, L - 1]), f"selection of sequence {b}"
        assert np.array_equal(nsel[b], nsel_o[0, :, L - 1])
        oo, lo = O.fwd(m, xb["q"], xb["k"], xb["v"], idx_o, nsel_o, rows=[h * L + L - 1 for h in range(cfg.Hq)])
        oo_all.append(oo[0, L - 1])
        lo_all.append(lo[0, :, L - 1])
    compare("O", o, np.stack(oo_all))
    compare("L", lse, np.stack(lo_all))


def test_decode_bad_length_flagged():
    """A length outside 1..T is reported through the status word and yields an
    empty selection, without touching memory outside the caches."""
    from block_sparse_attention_09_b200 import msa
    cfg = Config("bad", B=2, T=512, Hq=4, Hkv=1, d=64, dp=32, topk=2)
    inp = make_inputs(cfg, seed=32)
    dev = {k: v.cuda() for k, v in inp.items()}
    q = dev["q"][:, -1].contiguous()
    qp = dev["qp"][:, -1].contiguous()
    lens = torch.tensor([512, 600], dtype=torch.int32, device="cuda")
    dims = msa.make_dims(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.dp, cfg.topk)
    ws = msa.workspace(dims, msa.MSA_DECODE, q.device)
    o, lse, idx, nsel = msa.decode(q, qp, dev["k"], dev["v"], dev["kp"], cfg.topk, lens=lens, ws=ws)
    assert msa.check_status(ws) == -9
    assert int(nsel[1].max()) == 0 and bool((idx[1] == -1).all())
    assert int(nsel[0].min()) == cfg.topk
