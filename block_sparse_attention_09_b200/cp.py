"""Context-parallel MSA: one long sequence split by rows over the ranks of a
process group (one process per GPU).

Rank j owns the rows [r0_j, r1_j) of the sequence: its queries, keys, values,
proxy queries/keys and output gradient.  A training step is

  1. all-gather of the key side (k, v, kp): rank j needs the causal prefix
     of keys [0, r1_j) its queries can see;
  2. on each rank, the library's selection, forward and backward restricted
     to its own query rows (q_begin = r0_j on buffers of length r1_j): the
     outputs o, lse, dq of those rows, and fp32 partial dK/dV over the keys
     [0, r1_j) -- the contributions of this rank's queries;
  3. reduce-scatter of the partial dK/dV, so each rank receives the sum over
     all ranks for its own key rows, rounded once to bf16.

Rows are split into equal, 128-aligned shards: the Main Branch costs the same
per query row wherever it sits (topk blocks each), so equal rows balance it.
The collectives go through ``torch.distributed`` (NCCL on GPUs); every step of
the attention itself runs in the library's kernels (``ops`` defaults to the
CUDA binding; tests substitute a CPU stand-in with the same signatures).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_bounds(T: int, world: int, rank: int):
    """Rows [r0, r1) of rank `rank` when T rows are split into `world`
    contiguous shards: whole 128-row blocks, as equal as possible, the
    remainder (and a ragged last block) on the last ranks."""
    nblk = (T + 127) // 128
    base, extra = divmod(nblk, world)
    b0 = rank * base + max(0, rank - (world - extra))
    b1 = b0 + base + (1 if rank >= world - extra else 0)
    return min(T, 128 * b0), min(T, 128 * b1)


def _gather_rows(x, group, world, bounds):
    """All-gather of per-rank row shards x [B, r1-r0, ...] into [B, T, ...]
    (shards padded to a common length for the collective)."""
    L = max(r1 - r0 for r0, r1 in bounds)
    pad = x.new_zeros((x.shape[0], L) + tuple(x.shape[2:]))
    pad[:, :x.shape[1]] = x
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([p[:, :r1 - r0] for p, (r0, r1) in zip(parts, bounds)], dim=1).contiguous()


def _reduce_scatter_rows(part, group, world, rank, bounds):
    """part [B, r1_rank, ...] fp32 holds this rank's contribution to the key
    rows [0, r1_rank).  Returns the sum over ranks of the rows this rank owns,
    [B, r1-r0, ...]."""
    L = max(r1 - r0 for r0, r1 in bounds)
    B, rest = part.shape[0], tuple(part.shape[2:])
    # row-major by owner: chunk j holds the rows of rank j's shard
    buf = part.new_zeros((world, L, B) + rest)
    for j, (r0, r1) in enumerate(bounds):
        hi = min(r1, part.shape[1])
        if hi > r0:
            buf[j, :hi - r0] = part[:, r0:hi].transpose(0, 1)
    if dist.get_backend(group) == "nccl":
        out = part.new_empty((L, B) + rest)
        dist.reduce_scatter_tensor(out, buf.view(world * L, B, *rest), group=group)
    else:   # gloo has no reduce-scatter: reduce everything, keep this rank's chunk
        dist.all_reduce(buf, group=group)
        out = buf[rank]
    r0, r1 = bounds[rank]
    return out[:r1 - r0].transpose(0, 1).contiguous()


def local_step(q, k_pre, v_pre, dout, qp, kp_pre, topk, r0, ops, scale=0.0):
    """The per-rank part of a context-parallel step (no communication).

    q, dout, qp: this rank's rows [B, r1-r0, ...]; k_pre, v_pre, kp_pre: the
    keys [0, r1) ([B, r1, ...]).  Returns o, lse of this rank's rows, dq of its
    rows, and fp32 partial dk, dv over the keys [0, r1)."""
    B, n, Hq, d = q.shape
    r1 = r0 + n
    assert k_pre.shape[1] == r1 and r0 % 128 == 0

    def placed(x):   # the rows in place in a buffer of length r1; rows < r0 are never read
        buf = x.new_empty((B, r1) + tuple(x.shape[2:]))
        buf[:, r0:] = x
        return buf

    qb, qpb, dob = placed(q), placed(qp), placed(dout)
    idx, nsel = ops.proxy_select(qpb, kp_pre, topk, q_begin=r0)
    dims = ops.make_dims(B, r1, Hq, k_pre.shape[2], d, qp.shape[3], topk, scale, q_begin=r0)
    ws = ops.step_workspace(dims, q.device)
    o, lse = ops.fwd(qb, k_pre, v_pre, idx, nsel, scale=scale, ws=ws, q_begin=r0)
    dq, dk, dv = ops.bwd(qb, k_pre, v_pre, o, dob, lse, idx, nsel, scale=scale, ws=ws, reuse_index=True,
                         q_begin=r0, dkv_f32=True)
    return (o[:, r0:].contiguous(), lse[:, :, r0:].contiguous(), dq[:, r0:].contiguous(), dk, dv, idx, nsel)


def step(q, k, v, dout, qp, kp, topk, T, group=None, ops=None, scale=0.0, return_selection=False):
    """One context-parallel MSA training step.  Every rank passes its own rows
    [r0, r1) = shard_bounds(T, world, rank) of q, k, v, dout, qp, kp
    ([B, r1-r0, H, d]).  Returns this rank's rows of o, lse ([B, Hq, r1-r0]),
    dq, and of dk, dv summed over every rank's queries (and, with
    return_selection, its rows' idx [B, Hp, r1-r0, topk] and nsel).  Without
    an initialised process group the step runs as the only rank."""
    if ops is None:
        from . import msa as ops
    if dist.is_available() and dist.is_initialized():
        world, rank = dist.get_world_size(group), dist.get_rank(group)
    else:
        world, rank = 1, 0
    if world == 1:
        o, lse, dq, dk_part, dv_part, idx, nsel = local_step(q, k, v, dout, qp, kp, topk, 0, ops, scale)
        out = (o, lse, dq, ops.f32_to_bf16(dk_part), ops.f32_to_bf16(dv_part))
        return out + (idx, nsel) if return_selection else out
    bounds = [shard_bounds(T, world, j) for j in range(world)]
    r0, r1 = bounds[rank]
    assert q.shape[1] == r1 - r0
    # 1. the key side of the causal prefix
    k_all = _gather_rows(k, group, world, bounds)
    v_all = _gather_rows(v, group, world, bounds)
    kp_all = _gather_rows(kp, group, world, bounds)
    k_pre, v_pre, kp_pre = (x[:, :r1].contiguous() for x in (k_all, v_all, kp_all))
    # 2. this rank's queries
    o, lse, dq, dk_part, dv_part, idx, nsel = local_step(q, k_pre, v_pre, dout, qp, kp_pre, topk, r0, ops, scale)
    # 3. gradients of this rank's keys, summed over all ranks, rounded once
    dk = ops.f32_to_bf16(_reduce_scatter_rows(dk_part, group, world, rank, bounds))
    dv = ops.f32_to_bf16(_reduce_scatter_rows(dv_part, group, world, rank, bounds))
    if return_selection:
        return o, lse, dq, dk, dv, idx[:, :, r0:].contiguous(), nsel[:, :, r0:].contiguous()
    return o, lse, dq, dk, dv
