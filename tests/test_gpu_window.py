"""GPU parity of the forced block pattern (window of w blocks with dilation,
counted in topk; page "Flash-MSA: Train on a million tokens without breaking
the compute bank", section "Under the hood", with our reading of it).

Selection is compared bit for bit with the oracle on grid proxy inputs (every
proxy score exact in any order), across window sizes, dilations, the window
equal to topk, windows reaching below block 0, and topk in both sort
variants.  One configuration then runs the Main Branch forward and backward
over the windowed selection against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import Config, make_inputs
from parity_util import compare, f32, oracle_inputs, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    # name, config, window, dilation
    ("w3_d1", Config("w3_d1", B=1, T=2048, Hq=4, Hkv=2, d=64, dp=32, topk=6), 3, 1),
    ("w4_d3", Config("w4_d3", B=2, T=3000, Hq=8, Hkv=2, d=64, dp=64, topk=8), 4, 3),
    ("w_eq_topk", Config("w_eq_topk", B=1, T=1920, Hq=4, Hkv=1, d=64, dp=32, topk=4), 4, 2),
    ("w2_d7_big_topk", Config("w2_d7", B=1, T=12288, Hq=4, Hkv=1, d=64, dp=64, topk=80), 2, 7),
    ("w8_d1_recency", Config("w8_d1", B=1, T=16384, Hq=8, Hkv=2, d=64, dp=64, topk=16, bias="recency"), 8, 1),
]


def _dims(cfg, window, dil):
    return O.Dims(B=cfg.B, T=cfg.T, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, dp=cfg.dp, topk=cfg.topk,
                  window=window, dilation=dil)


@pytest.mark.parametrize("name,cfg,window,dil", CASES, ids=[c[0] for c in CASES])
def test_window_selection_bit_exact(name, cfg, window, dil):
    from block_sparse_attention_09_b200 import msa
    inp = make_inputs(cfg, seed=21, exact_proxy=True, parts=["qp", "kp"])
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True, window=window, dilation=dil)
    torch.cuda.synchronize()
    x = oracle_inputs(inp)
    idx_o, nsel_o, _ = O.select(_dims(cfg, window, dil), x["qp"], x["kp"])
    assert np.array_equal(nsel.cpu().numpy(), nsel_o)
    assert np.array_equal(idx.cpu().numpy(), idx_o)


def test_window_main_branch():
    from block_sparse_attention_09_b200 import msa
    cfg = Config("w3_d2_main", B=1, T=1536, Hq=8, Hkv=2, d=128, dp=64, topk=5)
    window, dil = 3, 2
    inp = make_inputs(cfg, seed=22, exact_proxy=True)
    dev = to_dev(inp)
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True, window=window, dilation=dil)
    o, lse = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, check=True)
    dq, dk, dv = msa.bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, idx, nsel, check=True)
    torch.cuda.synchronize()
    x = oracle_inputs(inp)
    m = _dims(cfg, window, dil)
    idx_o, nsel_o, _ = O.select(m, x["qp"], x["kp"])
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    oo, lo = O.fwd(m, x["q"], x["k"], x["v"], idx_o, nsel_o)
    dqo, Do = O.bwd_dq(m, x["q"], x["k"], x["v"], x["dout"], oo, lo, idx_o, nsel_o)
    dko, dvo = O.bwd_dkdv(m, x["q"], x["k"], x["v"], x["dout"], lo, Do, idx_o, nsel_o)
    compare("O", f32(o), oo)
    compare("L", f32(lse), lo)
    compare("dQ", f32(dq), dqo)
    compare("dK", f32(dk), dko)
    compare("dV", f32(dv), dvo)


def test_window_rejected_above_topk():
    from block_sparse_attention_09_b200 import msa
    qp = torch.zeros((1, 256, 1, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        msa.proxy_select(qp, qp, 3, window=4)
