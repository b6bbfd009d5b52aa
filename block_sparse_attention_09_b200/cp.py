"""Context-parallel MSA: one long sequence split by rows over the ranks of a
process group (one process per GPU).

The sequence's 128-row blocks are cut into 2W equal chunks (W ranks) and rank
j owns chunks j and 2W-1-j ("zig-zag"): its queries, keys, values, proxy
queries/keys and output gradient of those rows, concatenated in sequence
order.  The Main Branch costs about the same per query row wherever it sits
(topk blocks each), but the causal proxy scoring of a row grows with its
position; pairing an early chunk with the mirrored late one gives every rank
the same proxy work as well.  A training step is

  1. all-gather of the key side (k, v, kp): each of a rank's chunks needs the
     causal prefix of keys its queries can see;
  2. on each rank, per chunk [c0, c1): the library's selection, forward and
     backward restricted to those query rows (q_begin = c0 on buffers of
     length c1): the outputs o, lse, dq of those rows, and fp32 partial dK/dV
     over the keys [0, c1) -- the contributions of the chunk's queries;
  3. reduce-scatter of the partial dK/dV, so each rank receives the sum over
     all ranks for its own key rows, rounded once to bf16.

The collectives go through ``torch.distributed`` (NCCL on GPUs); every step of
the attention itself runs in the library's kernels (``ops`` defaults to the
CUDA binding; tests substitute a CPU stand-in with the same signatures).

Memory: a chunk's call holds query-side buffers of length c1 (rows before
c0 are never read or written), so the rank owning the last chunk holds
full-length query-side buffers for that call.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_chunks(T: int, world: int, rank: int):
    """The row chunks [(c0, c1), ...] rank `rank` owns, in sequence order:
    chunks `rank` and `2 world - 1 - rank` of the 2 world chunks of whole
    128-row blocks (as equal as possible; the remainder, and a ragged last
    block, on the later chunks).  Empty chunks are dropped."""
    nblk = (T + 127) // 128
    n = 2 * world
    base, extra = divmod(nblk, n)

    def chunk(c):
        b0 = c * base + max(0, c - (n - extra))
        b1 = b0 + base + (1 if c >= n - extra else 0)
        return min(T, 128 * b0), min(T, 128 * b1)

    out = [chunk(rank), chunk(n - 1 - rank)]
    return [(c0, c1) for c0, c1 in out if c1 > c0]


def shard_rows(T: int, world: int, rank: int) -> int:
    """Number of rows rank `rank` owns."""
    return sum(c1 - c0 for c0, c1 in shard_chunks(T, world, rank))


def take_rows(x, chunks, dim=1):
    """The rows of `chunks` of a full-length tensor, concatenated (a rank's
    local view of the sequence)."""
    return torch.cat([x.narrow(dim, c0, c1 - c0) for c0, c1 in chunks], dim=dim).contiguous()


def _gather_rows(x, group, world, chunks_of):
    """All-gather of per-rank row sets x [B, rows of the rank, ...] into the
    full sequence [B, T, ...] (row sets padded to a common length for the
    collective)."""
    L = max(sum(c1 - c0 for c0, c1 in ch) for ch in chunks_of)
    pad = x.new_zeros((x.shape[0], L) + tuple(x.shape[2:]))
    pad[:, :x.shape[1]] = x
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    T = max(c1 for ch in chunks_of for _, c1 in ch)
    out = x.new_empty((x.shape[0], T) + tuple(x.shape[2:]))
    for part, ch in zip(parts, chunks_of):
        at = 0
        for c0, c1 in ch:
            out[:, c0:c1] = part[:, at:at + c1 - c0]
            at += c1 - c0
    return out


def _reduce_scatter_rows(part, group, world, rank, chunks_of):
    """part [B, P, ...] fp32 holds this rank's contribution to the key rows
    [0, P).  Returns the sum over ranks of the rows this rank owns, in its
    local (chunk-concatenated) order."""
    L = max(sum(c1 - c0 for c0, c1 in ch) for ch in chunks_of)
    B, rest = part.shape[0], tuple(part.shape[2:])
    # row-major by owner: slot j holds the rows of rank j's chunks
    buf = part.new_zeros((world, L, B) + rest)
    for j, ch in enumerate(chunks_of):
        at = 0
        for c0, c1 in ch:
            hi = min(c1, part.shape[1])
            if hi > c0:
                buf[j, at:at + hi - c0] = part[:, c0:hi].transpose(0, 1)
            at += c1 - c0
    if dist.get_backend(group) == "nccl":
        out = part.new_empty((L, B) + rest)
        dist.reduce_scatter_tensor(out, buf.view(world * L, B, *rest), group=group)
    else:   # gloo has no reduce-scatter: reduce everything, keep this rank's slot
        dist.all_reduce(buf, group=group)
        out = buf[rank]
    n = sum(c1 - c0 for c0, c1 in chunks_of[rank])
    return out[:n].transpose(0, 1).contiguous()


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
    (the chunks shard_chunks(T, world, rank), concatenated in sequence order;
    take_rows builds them) of q, k, v, dout, qp, kp ([B, rows, H, d]).  Returns
    this rank's rows of o, lse ([B, Hq, rows]), dq, and of dk, dv summed over
    every rank's queries (and, with return_selection, its rows' idx
    [B, Hp, rows, topk] and nsel).  Without an initialised process group the
    step runs as the only rank over the whole sequence."""
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
    chunks_of = [shard_chunks(T, world, j) for j in range(world)]
    mine = chunks_of[rank]
    assert q.shape[1] == sum(c1 - c0 for c0, c1 in mine)
    # 1. the key side of the sequence (each chunk then takes its causal prefix)
    k_all = _gather_rows(k, group, world, chunks_of)
    v_all = _gather_rows(v, group, world, chunks_of)
    kp_all = _gather_rows(kp, group, world, chunks_of)
    # 2. this rank's queries, chunk by chunk; the fp32 partials add up over
    # the keys [0, end of the rank's last chunk)
    B, Hkv, d = k.shape[0], k.shape[2], k.shape[3]
    P = mine[-1][1] if mine else 0
    dk_part = torch.zeros((B, P, Hkv, d), dtype=torch.float32, device=k.device)
    dv_part = torch.zeros_like(dk_part)
    outs, at = [], 0
    for c0, c1 in mine:
        n = c1 - c0
        sl = slice(at, at + n)
        at += n
        o_c, lse_c, dq_c, dk_c, dv_c, idx_c, nsel_c = local_step(
            q[:, sl], k_all[:, :c1].contiguous(), v_all[:, :c1].contiguous(), dout[:, sl], qp[:, sl],
            kp_all[:, :c1].contiguous(), topk, c0, ops, scale)
        dk_part[:, :c1] += dk_c
        dv_part[:, :c1] += dv_c
        outs.append((o_c, lse_c, dq_c, idx_c[:, :, c0:], nsel_c[:, :, c0:]))
    if not outs:   # a rank with no rows (fewer blocks than chunks) still joins the collectives
        Hq = q.shape[2]
        o, dq = q.new_empty((B, 0, Hq, d)), q.new_empty((B, 0, Hq, d))
        lse = torch.empty((B, Hq, 0), dtype=torch.float32, device=q.device)
        idx0 = torch.empty((B, Hkv, 0, topk), dtype=torch.int32, device=q.device)
        outs_sel = (idx0, torch.empty((B, Hkv, 0), dtype=torch.int32, device=q.device))
    else:
        o = torch.cat([x[0] for x in outs], dim=1)
        lse = torch.cat([x[1] for x in outs], dim=2)
        dq = torch.cat([x[2] for x in outs], dim=1)
        outs_sel = (torch.cat([x[3] for x in outs], dim=2).contiguous(),
                    torch.cat([x[4] for x in outs], dim=2).contiguous())
    # 3. gradients of this rank's keys, summed over all ranks, rounded once
    dk = ops.f32_to_bf16(_reduce_scatter_rows(dk_part, group, world, rank, chunks_of))
    dv = ops.f32_to_bf16(_reduce_scatter_rows(dv_part, group, world, rank, chunks_of))
    if return_selection:
        return (o, lse, dq, dk, dv) + outs_sel
    return o, lse, dq, dk, dv
