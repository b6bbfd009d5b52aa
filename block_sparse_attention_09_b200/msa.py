"""Thin Python binding of libmsa.so (the C ABI in include/msa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  There is no
CPU or PyTorch fallback: if libmsa.so is missing the import fails.

    from block_sparse_attention_09_b200 import msa
    idx, nsel = msa.proxy_select(qp, kp, topk)              # Index Branch (cached)
    o, lse = msa.fwd(q, k, v, idx, nsel)                     # Main Branch forward
    dq, dk, dv = msa.bwd(q, k, v, o, dout, lse, idx, nsel)   # Main Branch backward
    o = msa.MSAAttention.apply(q, k, v, qp, kp, topk)        # autograd wrapper

Layouts: q, o, dout [B,T,Hq,d]; k, v [B,T,Hkv,d]; qp, kp [B,T,Hkv,dp], all
bf16 and contiguous; idx [B,Hkv,T,topk] int32; nsel [B,Hkv,T] int32;
lse [B,Hq,T] fp32.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

MSA_SELECT, MSA_FWD, MSA_BWD, MSA_DECODE, MSA_PROXY_BWD = 0, 1, 2, 3, 4
MSA_REUSE_INDEX, MSA_DKV_F32, MSA_BLOCK_MASS = 1, 2, 4
_ERR = {0: "ok", -1: "invalid dimensions", -2: "null pointer", -3: "misaligned pointer",
        -4: "workspace too small", -5: "CUDA launch failed", -6: "device wait timed out",
        -7: "device is not sm_100", -8: "tensor map encoding failed",
        -9: "block index out of range"}


class MsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {_ERR.get(code, 'unknown')} ({code})")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("Hp", ctypes.c_int), ("d", ctypes.c_int), ("dp", ctypes.c_int), ("block", ctypes.c_int),
                ("topk", ctypes.c_int), ("scale", ctypes.c_float), ("window", ctypes.c_int),
                ("dilation", ctypes.c_int), ("q_begin", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmsa.so not built ({LIB_PATH}); run `python -m block_sparse_attention_09_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, SZ, I, U64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64
    D = ctypes.POINTER(Dims)
    lib.msa_workspace_size.argtypes = [D, I]
    lib.msa_workspace_size.restype = SZ
    lib.msa_proxy_select.argtypes = [D, P, P, P, P, P, P, SZ, P]
    lib.msa_fwd.argtypes = [D, P, P, P, P, P, P, P, P, SZ, P]
    lib.msa_bwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.msa_check_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    lib.msa_strerror.argtypes = [I]
    lib.msa_strerror.restype = ctypes.c_char_p
    lib.msa_diag_umma.argtypes = [I, I, I, P, P, P, P, P]
    lib.msa_diag_wait_timeout.argtypes = [U64, P, P]
    lib.msa_set_kernel_events.argtypes = [I, P, P]
    lib.msa_fwd_ex.argtypes = [D, P, P, P, P, P, P, P, P, SZ, P, I]
    lib.msa_fwd_ex.restype = I
    lib.msa_bwd_ex.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P, I]
    lib.msa_bwd_ex.restype = I
    lib.msa_decode.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.msa_decode.restype = I
    lib.msa_f32_to_bf16.argtypes = [P, P, ctypes.c_int64, P]
    lib.msa_f32_to_bf16.restype = I
    lib.msa_proxy_bwd.argtypes = [D, P, P, P, P, P, P, P, P, SZ, P]
    lib.msa_proxy_bwd.restype = I
    lib.msa_fallback_rows.argtypes = [P, P, ctypes.POINTER(ctypes.c_int64)]
    lib.msa_fallback_rows.restype = I
    lib.msa_kernel_launches.argtypes = []
    lib.msa_kernel_launches.restype = U64
    for f in ("msa_proxy_select", "msa_fwd", "msa_bwd", "msa_check_status", "msa_diag_umma",
              "msa_diag_wait_timeout", "msa_set_kernel_events"):
        getattr(lib, f).restype = I
    return lib


LIB = _load()


def make_dims(B, T, Hq, Hkv, d, dp, topk, scale=0.0, window=1, dilation=1, q_begin=0) -> Dims:
    return Dims(int(B), int(T), int(Hq), int(Hkv), int(Hkv), int(d), int(dp), 128, int(topk), float(scale),
                int(window), int(dilation), int(q_begin))


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc, where):
    if rc != 0:
        raise MsaError(rc, where)


def workspace_size(dims: Dims, which: int) -> int:
    return int(LIB.msa_workspace_size(ctypes.byref(dims), which))


def workspace(dims: Dims, which: int, device) -> torch.Tensor:
    return torch.empty(max(workspace_size(dims, which), 256), dtype=torch.uint8, device=device)


def step_workspace(dims: Dims, device) -> torch.Tensor:
    """One workspace for a forward and the backward that reuses its index."""
    n = max(workspace_size(dims, MSA_FWD), workspace_size(dims, MSA_BWD), 256)
    return torch.empty(n, dtype=torch.uint8, device=device)


def check_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and read the status word a call left in ``ws``."""
    code = ctypes.c_uint32(0)
    rc = LIB.msa_check_status(_p(ws), _stream(stream), ctypes.byref(code))
    return rc


def fallback_rows(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and read how many rows the last forward on ``ws`` redid
    with its exact two-pass softmax."""
    n = ctypes.c_int64(0)
    _check(LIB.msa_fallback_rows(_p(ws), _stream(stream), ctypes.byref(n)), "msa_fallback_rows")
    return int(n.value)


def _bf16(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("expected contiguous CUDA bf16 tensors")


def dims_of(q, k, qp, topk, scale=0.0) -> Dims:
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    dp = qp.shape[3] if qp is not None else 64
    return make_dims(B, T, Hq, Hkv, d, dp, topk, scale)


def proxy_select(qp, kp, topk, pooled=False, stream=None, ws=None, check=False, window=1, dilation=1, q_begin=0):
    """Index Branch.  Returns (idx, nsel) or (idx, nsel, pooled_scores).
    window/dilation: forced block pattern (own block and the window-1 blocks
    every `dilation` blocks before it).  q_begin: first query row selected
    (a multiple of 128); earlier rows of the outputs are left unwritten."""
    _bf16(qp, kp)
    B, T, Hp, dp = qp.shape
    dims = make_dims(B, T, Hp, Hp, 64, dp, topk, window=window, dilation=dilation, q_begin=q_begin)
    idx = torch.empty((B, Hp, T, topk), dtype=torch.int32, device=qp.device)
    nsel = torch.empty((B, Hp, T), dtype=torch.int32, device=qp.device)
    nblk = (T + 127) // 128
    pool = torch.empty((B, Hp, T, nblk), dtype=torch.float32, device=qp.device) if pooled else None
    if ws is None:
        ws = workspace(dims, MSA_SELECT, qp.device)
    _check(LIB.msa_proxy_select(ctypes.byref(dims), _p(qp), _p(kp), _p(idx), _p(nsel), _p(pool), _p(ws),
                                ws.numel(), _stream(stream)), "msa_proxy_select")
    if check:
        _check(check_status(ws, stream), "msa_proxy_select (device)")
    return (idx, nsel, pool) if pooled else (idx, nsel)


def fwd(q, k, v, idx, nsel, scale=0.0, stream=None, ws=None, check=False, out=None, reuse_index=False,
        q_begin=0, block_mass=False):
    """Main Branch forward.  Returns (o bf16 [B,T,Hq,d], lse fp32 [B,Hq,T]).
    q_begin: first query row computed; earlier rows of o, lse are unwritten.
    block_mass: also keep each row's weight per selected block in ``ws`` (a
    proxy_workspace) for a following proxy_bwd."""
    _bf16(q, k, v)
    B, T, Hq, d = q.shape
    topk = idx.shape[3]
    dims = make_dims(B, T, Hq, k.shape[2], d, 64, topk, scale, q_begin=q_begin)
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    if ws is None:
        ws = workspace(dims, MSA_PROXY_BWD if block_mass else MSA_FWD, q.device)
    flags = (MSA_REUSE_INDEX if reuse_index else 0) | (MSA_BLOCK_MASS if block_mass else 0)
    _check(LIB.msa_fwd_ex(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(idx), _p(nsel), _p(o), _p(lse), _p(ws),
                          ws.numel(), _stream(stream), flags), "msa_fwd")
    if check:
        _check(check_status(ws, stream), "msa_fwd (device)")
    return o, lse


def bwd(q, k, v, o, dout, lse, idx, nsel, scale=0.0, stream=None, ws=None, check=False, out=None,
        reuse_index=False, q_begin=0, dkv_f32=False):
    """Main Branch backward.  Returns (dq, dk, dv), bf16.  reuse_index: ``ws``
    already holds the inverse index of these idx/nsel from an earlier call on
    the same workspace (e.g. the forward of the same step).  q_begin: first
    query row computed (dq rows before it are unwritten; dk, dv hold the
    contributions of the computed rows only).  dkv_f32: dk, dv are fp32
    unrounded sums, for adding the partials of several query shards."""
    _bf16(q, k, v, o, dout)
    B, T, Hq, d = q.shape
    topk = idx.shape[3]
    dims = make_dims(B, T, Hq, k.shape[2], d, 64, topk, scale, q_begin=q_begin)
    if out is None:
        dq = torch.empty_like(q)
        kv_dtype = torch.float32 if dkv_f32 else torch.bfloat16
        dk = torch.empty(k.shape, dtype=kv_dtype, device=k.device)
        dv = torch.empty(v.shape, dtype=kv_dtype, device=v.device)
    else:
        dq, dk, dv = out
    flags = (MSA_REUSE_INDEX if reuse_index else 0) | (MSA_DKV_F32 if dkv_f32 else 0)
    if ws is None:
        ws = workspace(dims, MSA_BWD, q.device)
    _check(LIB.msa_bwd_ex(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(o), _p(dout), _p(lse), _p(idx),
                          _p(nsel), _p(dq), _p(dk), _p(dv), _p(ws), ws.numel(), _stream(stream), flags), "msa_bwd")
    if check:
        _check(check_status(ws, stream), "msa_bwd (device)")
    return dq, dk, dv


def proxy_workspace(dims: Dims, device) -> torch.Tensor:
    """One workspace for a forward that keeps block masses, the backward
    that reuses its index, and the proxy-head gradient."""
    return torch.empty(max(workspace_size(dims, MSA_PROXY_BWD), 256), dtype=torch.uint8, device=device)


def proxy_bwd(q, qp, kp, idx, nsel, ws, stream=None, check=False, out=None, q_begin=0):
    """Proxy-head gradient (a KL distillation of the Main Branch's block
    weights into the proxy scores; see include/msa.h).  ``ws`` must hold what
    fwd(..., block_mass=True) left for these idx/nsel.  Returns (dqp, dkp fp32
    [B,T,Hp,dp], loss fp32 [B,Hp,T])."""
    _bf16(qp, kp)
    B, T, Hp, dp = qp.shape
    dims = make_dims(B, T, q.shape[2], Hp, q.shape[3], dp, idx.shape[3], q_begin=q_begin)
    if out is None:
        dqp = torch.zeros(qp.shape, dtype=torch.float32, device=qp.device)
        dkp = torch.empty(kp.shape, dtype=torch.float32, device=kp.device)
        loss = torch.zeros((B, Hp, T), dtype=torch.float32, device=qp.device)
    else:
        dqp, dkp, loss = out
    _check(LIB.msa_proxy_bwd(ctypes.byref(dims), _p(qp), _p(kp), _p(idx), _p(nsel), _p(dqp), _p(dkp), _p(loss),
                             _p(ws), ws.numel(), _stream(stream)), "msa_proxy_bwd")
    if check:
        _check(check_status(ws, stream), "msa_proxy_bwd (device)")
    return dqp, dkp, loss


def f32_to_bf16(src, out=None, stream=None):
    """bf16 copy of a contiguous fp32 CUDA tensor (numel a multiple of 8),
    rounded on the device by msa_f32_to_bf16."""
    if src.dtype != torch.float32 or not src.is_cuda or not src.is_contiguous():
        raise ValueError("expected a contiguous CUDA fp32 tensor")
    dst = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device) if out is None else out
    _check(LIB.msa_f32_to_bf16(_p(src), _p(dst), src.numel(), _stream(stream)), "msa_f32_to_bf16")
    return dst


class MSAAttention(torch.autograd.Function):
    """o = MSA(q, k, v; qp, kp, topk).  The block ids chosen in forward are
    cached for backward; no gradient flows to qp/kp (the selection is
    piecewise constant)."""

    @staticmethod
    def forward(ctx, q, k, v, qp, kp, topk, scale=0.0):
        idx, nsel = proxy_select(qp, kp, topk)
        B, T, Hq, d = q.shape
        ws = step_workspace(make_dims(B, T, Hq, k.shape[2], d, 64, topk, scale), q.device)
        o, lse = fwd(q, k, v, idx, nsel, scale, ws=ws)
        ctx.save_for_backward(q, k, v, o, lse, idx, nsel)
        ctx.scale = scale
        ctx.ws = ws   # holds the inverse index for the backward
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse, idx, nsel = ctx.saved_tensors
        dq, dk, dv = bwd(q, k, v, o, dout.contiguous(), lse, idx, nsel, ctx.scale, ws=ctx.ws, reuse_index=True)
        ctx.ws = None
        return dq, dk, dv, None, None, None, None


KERNEL_PROXY, KERNEL_FWD_MAIN, KERNEL_BWD_MAIN = 0, 1, 2


def set_kernel_events(kernel: int, start=None, stop=None) -> None:
    """Record torch.cuda.Event ``start``/``stop`` around the named kernel in
    later calls from this thread (None stops recording)."""
    s = ctypes.c_void_p(start.cuda_event) if start is not None else None
    e = ctypes.c_void_p(stop.cuda_event) if stop is not None else None
    _check(LIB.msa_set_kernel_events(kernel, s, e), "msa_set_kernel_events")


def decode(q, qp, k, v, kp, topk, lens=None, scale=0.0, window=1, dilation=1, stream=None, ws=None,
           check=False, out=None):
    """One new token per sequence against caches.  q [B,Hq,d], qp [B,Hp,dp],
    caches k, v [B,T,Hkv,d], kp [B,T,Hp,dp]; lens int32 [B] on the device (None:
    every sequence has length T).  Returns (o [B,Hq,d] bf16, lse [B,Hq] fp32,
    idx [B,Hp,topk], nsel [B,Hp])."""
    _bf16(q, qp, k, v, kp)
    B, T, Hkv, d = k.shape
    Hq, Hp, dp = q.shape[1], kp.shape[2], kp.shape[3]
    dims = make_dims(B, T, Hq, Hkv, d, dp, topk, scale, window, dilation)
    if out is None:
        o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        idx = torch.empty((B, Hp, topk), dtype=torch.int32, device=q.device)
        nsel = torch.empty((B, Hp), dtype=torch.int32, device=q.device)
    else:
        o, lse, idx, nsel = out
    if lens is not None:
        assert lens.dtype == torch.int32 and lens.is_cuda and lens.is_contiguous()
    if ws is None:
        ws = workspace(dims, MSA_DECODE, q.device)
    _check(LIB.msa_decode(ctypes.byref(dims), _p(lens), _p(q), _p(qp), _p(k), _p(v), _p(kp), _p(idx), _p(nsel),
                          _p(o), _p(lse), _p(ws), ws.numel(), _stream(stream)), "msa_decode")
    if check:
        _check(check_status(ws, stream), "msa_decode (device)")
    return o, lse, idx, nsel


def kernel_launches() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(LIB.msa_kernel_launches())


def diag_umma(mode: int, A: torch.Tensor, B: torch.Tensor) -> torch.Tensor:
    """One tcgen05 MMA D = A B^T with the given operand staging (see msa.h)."""
    _bf16(A, B)
    N, K = B.shape
    D = torch.empty((128, N), dtype=torch.float32, device=A.device)
    ws = torch.empty(256, dtype=torch.uint8, device=A.device)
    _check(LIB.msa_diag_umma(mode, N, K, _p(A), _p(B), _p(D), _p(ws), _stream(None)), "msa_diag_umma")
    return D


def diag_wait_timeout(limit_ns: int, device="cuda") -> int:
    ws = torch.zeros(256, dtype=torch.uint8, device=device)
    return int(LIB.msa_diag_wait_timeout(limit_ns, _p(ws), _stream(None)))


def fwd_noalloc(q, k, v, idx, nsel, scale=0.0, stream=None, out=None):
    """msa_fwd_noalloc: the forward with the library's fixed 64 MiB device
    scratch instead of a caller workspace, for callers that cannot allocate
    device memory.  Only problems whose forward workspace fits 64 MiB; calls
    that overlap on the GPU must be serialised (they share the scratch)."""
    fn = LIB.msa_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(Dims)] + [ctypes.c_void_p] * 8
    fn.restype = ctypes.c_int
    _bf16(q, k, v)
    B, T, Hq, d = q.shape
    dims = make_dims(B, T, Hq, k.shape[2], d, 64, idx.shape[3], scale)
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(fn(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(idx), _p(nsel), _p(o), _p(lse), _stream(stream)),
           "msa_fwd_noalloc")
    return o, lse


def fwd_noalloc_status(stream=None) -> int:
    """msa_fwd_noalloc_status: synchronise and read the status the last
    fwd_noalloc on the current device left in the library's scratch."""
    fn = LIB.msa_fwd_noalloc_status
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]
    fn.restype = ctypes.c_int
    code = ctypes.c_uint32(0)
    return int(fn(_stream(stream), ctypes.byref(code)))
