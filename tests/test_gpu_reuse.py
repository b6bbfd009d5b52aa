"""Sharing the inverse index between a forward and its backward
(MSA_REUSE_INDEX on one workspace) must give the results of building it in
each call, for the C ABI and for the autograd wrapper.

The partial sums of O, dQ, dK and dV meet in fp32 reductions whose order
varies from run to run, so two runs agree to about one bf16 ulp, not bit for
bit; a wrong or stale index would be off by far more."""
import pytest
import torch

from block_sparse_attention_09_b200.inputs import Config, make_inputs

pytestmark = pytest.mark.gpu


def close(a, b):
    """Equal up to the run-to-run order of fp32 reductions: two bf16 ulps."""
    a, b = a.float(), b.float()
    return bool(((a - b).abs() <= 2.0 ** -7 * b.abs() + 1e-3).all())


def test_reused_index_bit_identical():
    from block_sparse_attention_09_b200 import msa
    cfg = Config("reuse", B=2, T=1500, Hq=8, Hkv=2, d=128, dp=64, topk=5)
    dev = {k: v.cuda() for k, v in make_inputs(cfg, seed=41).items()}
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk, check=True)
    o1, l1 = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, check=True)
    g1 = msa.bwd(dev["q"], dev["k"], dev["v"], o1, dev["dout"], l1, idx, nsel, check=True)
    dims = msa.make_dims(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, 64, cfg.topk)
    ws = msa.step_workspace(dims, dev["q"].device)
    o2, l2 = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel, ws=ws, check=True)
    g2 = msa.bwd(dev["q"], dev["k"], dev["v"], o2, dev["dout"], l2, idx, nsel, ws=ws, reuse_index=True, check=True)
    torch.cuda.synchronize()
    assert close(o2, o1) and close(l2, l1)
    for a, b in zip(g2, g1):
        assert close(a, b)


def test_autograd_wrapper_matches_calls():
    from block_sparse_attention_09_b200 import msa
    cfg = Config("autograd", B=1, T=1024, Hq=4, Hkv=1, d=64, dp=32, topk=3)
    dev = {k: v.cuda() for k, v in make_inputs(cfg, seed=42).items()}
    q, k, v = (dev[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    o = msa.MSAAttention.apply(q, k, v, dev["qp"], dev["kp"], cfg.topk)
    o.backward(dev["dout"])
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk)
    o_ref, lse = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel)
    dq, dk, dv = msa.bwd(dev["q"], dev["k"], dev["v"], o_ref, dev["dout"], lse, idx, nsel)
    torch.cuda.synchronize()
    assert close(o.detach(), o_ref)
    assert close(q.grad, dq) and close(k.grad, dk) and close(v.grad, dv)


def test_call_from_a_fresh_thread():
    """A host thread that has not touched CUDA yet (like an autograd worker)
    can call the library: it binds the device's context itself."""
    import threading
    from block_sparse_attention_09_b200 import msa
    cfg = Config("thread", B=1, T=512, Hq=4, Hkv=1, d=64, dp=32, topk=2)
    dev = {k: v.cuda() for k, v in make_inputs(cfg, seed=43).items()}
    idx, nsel = msa.proxy_select(dev["qp"], dev["kp"], cfg.topk)
    o, lse = msa.fwd(dev["q"], dev["k"], dev["v"], idx, nsel)
    ref = msa.bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, idx, nsel)
    torch.cuda.synchronize()
    res = {}

    def worker():
        try:
            res["g"] = msa.bwd(dev["q"], dev["k"], dev["v"], o, dev["dout"], lse, idx, nsel)
            torch.cuda.synchronize()
        except Exception as e:   # reported below
            res["err"] = e

    t = threading.Thread(target=worker)
    t.start()
    t.join()
    assert "err" not in res, res.get("err")
    for a, b in zip(res["g"], ref):
        assert close(a, b)

