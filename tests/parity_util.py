"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI binding and the CPU oracle on the same seeded inputs, compare."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle as O
from block_sparse_attention_09_b200.inputs import Config

# Acceptance (Flash-MSA verification: bf16 cosine-similarity sweeps with a
# 0.01 tolerance -> cosine >= 0.99), plus an element bound: an absolute
# 2e-2 on top of what storing the result in bf16 alone may cost.  A bf16
# number is within 2^-8 |x| of x (half a unit in the last place, 7 stored
# fraction bits), so for |x| >= 5 no bf16 output can be within 2e-2 of the
# exact value; the bound is |gpu - ref| <= 2e-2 + 2^-8 |ref|.
COS_MIN = 0.99
ABS_MAX = 2e-2
REL_BF16 = 2.0 ** -8


def odims(cfg: Config) -> O.Dims:
    return O.Dims(B=cfg.B, T=cfg.T, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, dp=cfg.dp, topk=cfg.topk)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def cosine(a, b) -> float:
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(a @ b / (na * nb))


# Every comparison of the session, for the summary conftest.py prints at
# the end of the run (and writes as JSON when MSA_PARITY_REPORT names a file).
REPORT = []


def compare(name, gpu, ref, cos_min=COS_MIN, abs_max=ABS_MAX, rel=REL_BF16, report=None):
    """Cosine >= cos_min and |gpu - ref| <= abs_max + rel |ref| element-wise.
    rel = 0 is the plain max-abs gate (fp32 results: L, fp32 dK/dV).  The
    figures are recorded whatever the outcome."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{name}: non-finite GPU values"
    c = cosine(gpu, ref)
    err = np.abs(gpu - ref)
    m = float(err.max()) if gpu.size else 0.0
    excess = err - (abs_max + rel * np.abs(ref))
    worst = int(excess.argmax()) if gpu.size else 0
    rec = dict(test=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], name=name, n=int(gpu.size),
               cos=c, max_abs=m, max_ref=float(np.abs(ref).max()) if ref.size else 0.0,
               abs_bound=float(abs_max), rel_bound=float(rel),
               n_over_abs=int((err > abs_max).sum()) if gpu.size else 0,
               worst_margin=float(-excess.flat[worst]) if gpu.size else 0.0)
    REPORT.append(rec)
    if report is not None:
        report[name] = rec
    assert c >= cos_min, f"{name}: cosine {c:.6f} < {cos_min}"
    assert not gpu.size or excess.flat[worst] <= 0, (
        f"{name}: |err| {err.flat[worst]:.3e} at |ref| {abs(ref.flat[worst]):.3e} exceeds "
        f"{abs_max} + {rel:.4g}|ref| (max abs err {m:.3e})")
    return c, m


def to_dev(inp, device="cuda"):
    return {k: v.to(device) for k, v in inp.items()}


def gpu_path(dev, topk, pooled=False):
    from block_sparse_attention_09_b200 import msa
    out = {}
    r = msa.proxy_select(dev["qp"], dev["kp"], topk, pooled=pooled, check=True)
    out["idx"], out["nsel"] = r[0], r[1]
    if pooled:
        out["pooled"] = r[2]
    out["o"], out["lse"] = msa.fwd(dev["q"], dev["k"], dev["v"], out["idx"], out["nsel"], check=True)
    out["dq"], out["dk"], out["dv"] = msa.bwd(dev["q"], dev["k"], dev["v"], out["o"], dev["dout"], out["lse"],
                                              out["idx"], out["nsel"], check=True)
    torch.cuda.synchronize()
    return out


def oracle_inputs(inp):
    return {k: f32(v) for k, v in inp.items()}
