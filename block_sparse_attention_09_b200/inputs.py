"""Seeded synthetic inputs for the MSA hot path.

This module only draws random numbers and applies the input recipes; it
holds none of the method's arithmetic.  Both the CUDA path's tests/benchmark
and the CPU oracle take their inputs from here.

Recipes (all values drawn in float32 on the CPU with ``torch.Generator``,
one stream per tensor, then rounded to bf16):

* Q, K, V, dO, proxy q/k ~ N(0, 1).
* ``bias="group"`` (8K workload): per group g a random unit vector u_g in
  R^dp and per-block offsets c[g, n] ~ N(0, 1); proxy keys of block n get
  ``+2 c[g, n] u_g`` and proxy queries get ``+2 u_g`` so that the pooled
  scores of each group gain ``4 c[g, n]`` and groups select different blocks.
* ``bias="recency"`` (128K workload): proxy dims 0..7 of token t are
  overwritten by ``alpha (cos w_f t, sin w_f t)``, f = 0..3,
  ``w_f = 2 pi / (4096 * 4**f)``, alpha = 2, so the proxy score of (i, j)
  gains ``alpha**2 sum_f cos(w_f (i - j))``, which favours nearby blocks.
* ``k_outliers=N`` (large-norm key variant): in every (batch, group), N key
  rows at seeded positions are multiplied by 8 (about 8x the norm of the
  others, as attention-sink-like keys of trained models have).
* ``exact_proxy=True``: proxy values are put on the grid k/8 (|k| <= 64) after
  the recipe.  Every product is then a multiple of 1/64 and every partial sum
  of <= 64 products fits a float32 mantissa, so the proxy scores are exact in
  any summation order and the GPU and the oracle see identical pooled scores.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

BLOCK = 128


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int
    dp: int
    topk: int
    bias: str = "none"   # "none" | "group" | "recency"
    k_outliers: int = 0  # large-norm (x8) key rows per (batch, group)

    @property
    def Hp(self) -> int:
        return self.Hkv

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nblk(self) -> int:
        return (self.T + BLOCK - 1) // BLOCK

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


# The five workloads (sizes as stated for the MSA training path), and the 1M point.
CONFIGS = {
    "tiny": Config("tiny", B=1, T=1024, Hq=4, Hkv=1, d=64, dp=32, topk=4),
    "8k": Config("8k", B=2, T=8192, Hq=16, Hkv=4, d=128, dp=64, topk=16, bias="group"),
    "32k": Config("32k", B=1, T=32768, Hq=32, Hkv=8, d=128, dp=64, topk=32),
    "128k": Config("128k", B=1, T=131072, Hq=32, Hkv=8, d=128, dp=64, topk=64, bias="recency"),
    "512k": Config("512k", B=1, T=524288, Hq=16, Hkv=4, d=128, dp=64, topk=128),
    # the top of the 512K -> 1M range the long-context speedups are quoted on,
    # with the 512K workload's head shape
    "1m": Config("1m", B=1, T=1048576, Hq=16, Hkv=4, d=128, dp=64, topk=128),
}

# stream ids: one independent generator per tensor
_STREAM = {"q": 1, "k": 2, "v": 3, "dout": 4, "qp": 5, "kp": 6, "bias_u": 7, "bias_c": 8, "outlier": 9}


def _gen(seed: int, name: str) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000003 + _STREAM[name])
    return g


def _randn(shape, seed, name):
    return torch.randn(*shape, generator=_gen(seed, name), dtype=torch.float32)


def _apply_group_bias(cfg: Config, qp, kp, seed):
    u = _randn((cfg.B, cfg.Hp, cfg.dp), seed, "bias_u")
    u = u / u.norm(dim=-1, keepdim=True)
    c = _randn((cfg.B, cfg.Hp, cfg.nblk), seed, "bias_c")
    blk_of = torch.arange(cfg.T) // BLOCK                      # [T]
    cb = c[:, :, blk_of].permute(0, 2, 1)                      # [B, T, Hp]
    kp += 2.0 * cb.unsqueeze(-1) * u.unsqueeze(1)
    qp += 2.0 * u.unsqueeze(1)


def _apply_recency_bias(cfg: Config, qp, kp, alpha=2.0):
    t = torch.arange(cfg.T, dtype=torch.float64)
    for f in range(4):
        w = 2.0 * math.pi / (4096.0 * 4.0 ** f)
        cs = (alpha * torch.cos(w * t)).float()
        sn = (alpha * torch.sin(w * t)).float()
        for x in (qp, kp):
            x[:, :, :, 2 * f] = cs.view(1, -1, 1)
            x[:, :, :, 2 * f + 1] = sn.view(1, -1, 1)


def _to_grid8(x):
    return torch.clamp(torch.round(x * 8.0), -64.0, 64.0) / 8.0


def make_inputs(cfg: Config, seed: int = 0, exact_proxy: bool = False, parts=None):
    """Return a dict of contiguous CPU bf16 tensors:
    q [B,T,Hq,d], k, v [B,T,Hkv,d], dout [B,T,Hq,d], qp, kp [B,T,Hp,dp].
    ``parts`` limits which tensors are drawn (the proxy pair is always drawn
    together)."""
    want = set(parts) if parts else {"q", "k", "v", "dout", "qp", "kp"}
    out = {}
    B, T = cfg.B, cfg.T
    for name, H, D in (("q", cfg.Hq, cfg.d), ("k", cfg.Hkv, cfg.d), ("v", cfg.Hkv, cfg.d),
                       ("dout", cfg.Hq, cfg.d)):
        if name in want:
            x = _randn((B, T, H, D), seed, name)
            if name == "k" and cfg.k_outliers > 0:
                g = _gen(seed, "outlier")
                for b in range(B):
                    for h in range(H):
                        pos = torch.randperm(T, generator=g)[:cfg.k_outliers]
                        x[b, pos, h] *= 8.0
            out[name] = x.to(torch.bfloat16).contiguous()
    if "qp" in want or "kp" in want:
        qp = _randn((B, T, cfg.Hp, cfg.dp), seed, "qp")
        kp = _randn((B, T, cfg.Hp, cfg.dp), seed, "kp")
        if cfg.bias == "group":
            _apply_group_bias(cfg, qp, kp, seed)
        elif cfg.bias == "recency":
            _apply_recency_bias(cfg, qp, kp)
        if exact_proxy:
            qp, kp = _to_grid8(qp), _to_grid8(kp)
        out["qp"] = qp.to(torch.bfloat16).contiguous()
        out["kp"] = kp.to(torch.bfloat16).contiguous()
    return out


def sample_rows(n_total: int, count: int, seed: int, must=()):
    """Seeded sample of distinct flat row ids plus the ones listed in ``must``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 7919 + 17)
    count = min(count, n_total)
    pick = torch.randperm(n_total, generator=g)[:count].tolist()
    return sorted(set(pick) | {int(m) for m in must if 0 <= int(m) < n_total})
