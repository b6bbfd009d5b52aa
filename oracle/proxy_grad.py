"""Oracle of a proxy-head training loss and its gradient -- TEST
INFRASTRUCTURE ONLY, and PARITY UNPINNED: the pages do not describe how the
proxy heads are trained.

The ai-beat post on Flash-MSA training (paragraph 2) says only that training
needs gradients through the "gating mechanism", and "Flash-MSA: Open-Source
Sparse Attention Kernels Debut" (section "How MSA works") calls MSA similar to
DeepSeek's sparse attention, whose indexer is trained to match the main
attention.  The reading written out here follows that: per query row
(b, g, i) with its selected blocks S_i,

    p_i(n) = (1/G) sum_{h in g} sum_{j in n, j <= i} P[b,h,i,j]
             (the forward's softmax mass on block n, held constant),
    z_i(n) = pooled(i, n) = max_{j in n, j <= i} qp_i . kp_j,
    q_i    = softmax over n in S_i of z_i(n),
    loss   = sum_i KL(p_i || q_i) = sum_i sum_n p_i(n) (log p_i(n) - log q_i(n)),

and the gradient d loss / d z_i(n) = q_i(n) sum_m p_i(m) - p_i(n) (which is
q_i(n) - p_i(n) when p_i sums to one) goes through the
max-pool to its argmax key j* (the lowest j on ties): dqp_i += dz kp_j*,
dkp_j* += dz qp_i.  The selection itself is fixed (passed in): top-k is
not differentiable.

Plain numpy in float64, one row at a time.  The tests pin it by finite
differences of the loss, the normalisation of p and q, and special cases --
checks of this definition, not of the pages.
"""
from __future__ import annotations

import numpy as np


def _own(i, blk):
    return i // blk


def block_mass(m, q, k, lse, idx, nsel, b, g, i):
    """p_i(n) for the row's selected blocks (order of idx): the forward's
    softmax weights, averaged over the group's heads."""
    G, blk = m.G, m.blk
    scale = m.scale if m.scale else 1.0 / np.sqrt(m.d)
    ns = int(nsel[b, g, i])
    out = np.zeros(ns)
    for s in range(ns):
        n = int(idx[b, g, i, s])
        j1 = min((n + 1) * blk, i + 1)
        keys = k[b, n * blk:j1, g].astype(np.float64)
        for hh in range(G):
            h = g * G + hh
            sc = scale * (keys @ q[b, i, h].astype(np.float64))
            out[s] += np.exp(sc - lse[b, h, i]).sum()
    return out / G


def pooled_argmax(m, qp, kp, idx, nsel, b, g, i):
    """z_i(n) and its argmax key for the row's selected blocks."""
    blk = m.blk
    ns = int(nsel[b, g, i])
    z, arg = np.zeros(ns), np.zeros(ns, dtype=np.int64)
    qv = qp[b, i, g].astype(np.float64)
    for s in range(ns):
        n = int(idx[b, g, i, s])
        j1 = min((n + 1) * blk, i + 1)
        sc = kp[b, n * blk:j1, g].astype(np.float64) @ qv
        a = int(np.argmax(sc))          # first maximum: the lowest key on ties
        z[s], arg[s] = sc[a], n * blk + a
    return z, arg


def loss_and_grad(m, qp, kp, q, k, lse, idx, nsel, rows=None):
    """Returns (loss, dqp, dkp) for the listed rows ((b, g, i) triples;
    default every row).  lse: the forward's natural-log L [B, Hq, T]."""
    if rows is None:
        rows = [(b, g, i) for b in range(m.B) for g in range(m.Hkv) for i in range(m.T)]
    dqp = np.zeros(qp.shape, dtype=np.float64)
    dkp = np.zeros(kp.shape, dtype=np.float64)
    total = 0.0
    for b, g, i in rows:
        if int(nsel[b, g, i]) <= 0:
            continue
        p = block_mass(m, q, k, lse, idx, nsel, b, g, i)
        z, arg = pooled_argmax(m, qp, kp, idx, nsel, b, g, i)
        zmax = z.max()
        lq = z - zmax - np.log(np.exp(z - zmax).sum())   # log q
        pos = p > 0
        total += float((p[pos] * (np.log(p[pos]) - lq[pos])).sum())
        dz = np.exp(lq) * p.sum() - p   # exact derivative, whatever the mass of p
        qv = qp[b, i, g].astype(np.float64)
        for s in range(len(z)):
            j = int(arg[s])
            dqp[b, i, g] += dz[s] * kp[b, j, g].astype(np.float64)
            dkp[b, j, g] += dz[s] * qv
    return total, dqp, dkp
