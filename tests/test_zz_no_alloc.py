"""The allocation-free forward (msa_fwd_noalloc) against the regular one.

msa_fwd_noalloc exists for callers that cannot allocate device memory or
hand over a workspace (a plugin host that owns all device memory, a loop
where cudaMalloc would synchronise the device): its scratch is a fixed
64 MiB array inside the library.  This file runs last so that a failure
here cannot hide any other test's result.
"""
import ctypes

import pytest
import torch

from block_sparse_attention_09_b200.inputs import Config, make_inputs
from parity_util import compare, f32

pytestmark = pytest.mark.gpu


def test_fwd_noalloc_matches_fwd_on_two_calls_in_a_row():
    from block_sparse_attention_09_b200 import msa
    cfg = Config("noalloc", B=2, T=1000, Hq=8, Hkv=2, d=128, dp=64, topk=3)
    dev = {k: v.cuda() for k, v in make_inputs(cfg, seed=7).items()}
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    o_ref, lse_ref = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, check=True)
    torch.cuda.synchronize()
    for call in range(2):
        # outputs pre-filled with NaN: every element must be written by the call
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        msa.fwd_noalloc(dev["q"], dev["k"], dev["v"], idx, nsel, out=(o, lse))
        torch.cuda.synchronize()
        compare(f"O (call {call})", f32(o), f32(o_ref))
        compare(f"L (call {call})", f32(lse), f32(lse_ref))


def test_fwd_noalloc_rejects_problems_beyond_its_scratch():
    from block_sparse_attention_09_b200 import msa
    fn = msa.LIB.msa_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(msa.Dims)] + [ctypes.c_void_p] * 8
    fn.restype = ctypes.c_int
    big = msa.make_dims(2, 8192, 16, 4, 128, 64, 16)     # needs far more than 64 MiB
    assert msa.workspace_size(big, msa.MSA_FWD) > (64 << 20)
    P = ctypes.c_void_p(4096)
    assert fn(ctypes.byref(big), P, P, P, P, P, P, P, None) == -4


def test_fwd_noalloc_status_reports_malformed_indices():
    from block_sparse_attention_09_b200 import msa
    cfg = Config("noalloc_bad", B=1, T=512, Hq=4, Hkv=1, d=64, dp=32, topk=2)
    dev = {k: v.cuda() for k, v in make_inputs(cfg, seed=6).items()}
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    msa.fwd_noalloc(dev["q"], dev["k"], dev["v"], idx, nsel)
    assert msa.fwd_noalloc_status() == 0
    bad = idx.clone()
    bad[0, 0, 300, 0] = 3        # a block after the query's own (300 // 128 = 2)
    bad[0, 0, 10, 0] = -5
    msa.fwd_noalloc(dev["q"], dev["k"], dev["v"], bad, nsel)   # the launch itself succeeds
    assert msa.fwd_noalloc_status() == -9
    # the next call clears the words it reports
    o, _ = msa.fwd_noalloc(dev["q"], dev["k"], dev["v"], idx, nsel)
    assert msa.fwd_noalloc_status() == 0
    assert torch.isfinite(o.float()).all()
