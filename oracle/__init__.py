"""CPU oracle for the MSA training hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it and it
never loads the CUDA library: the two share no code.

The arithmetic lives in ``msa_oracle.c`` (plain C, double precision, one row
or one KV block at a time).  This module builds it with gcc, loads it with
ctypes and converts numpy arrays.  Inputs are the bf16 tensors widened to
float32 (exact), so the oracle sees exactly the bits the GPU sees.

What each function follows (pages: "Flash-MSA: Open-Source Sparse Attention
Kernels Debut", section "How MSA works"; the ai-beat post on Flash-MSA
training, paragraphs 1-4):

* ``select``  -- proxy score per group, causal 128-key block max-pool, then the
  block selection (own block kept, best others by pooled score, ties to the
  lower block index; readings listed in the C source).
* ``fwd``     -- exact softmax attention of each query head over the keys of
  its group's selected blocks (GQA), returning O and the logsumexp L.
* ``bwd_dq``  -- dQ and D = dO . O per query row.
* ``bwd_dkdv``-- dK, dV per KV block, summed over every selecting query and
  every head of the group.

``proxy_grad`` (numpy) holds a proxy-head training loss and its gradient; the
pages do not describe one, so it is a reading, and its parity is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile msa_oracle.c into liboracle.so next to it (plain gcc, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC,
                               "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("d", ctypes.c_int), ("dp", ctypes.c_int),
                ("blk", ctypes.c_int), ("topk", ctypes.c_int), ("scale", ctypes.c_double),
                ("window", ctypes.c_int), ("dilation", ctypes.c_int)]


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        _lib.msa_oracle_select.argtypes = [ctypes.POINTER(_Dims), P, P, I64, P, P, P, P, ctypes.c_int]
        _lib.msa_oracle_select_from_pooled.argtypes = [I64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                       P, P, P, P]
        _lib.msa_oracle_fwd.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P, I64, P, P, P, ctypes.c_int]
        _lib.msa_oracle_bwd_dq.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P, P, P, P, I64, P,
                                           P, P, ctypes.c_int]
        _lib.msa_oracle_bwd_dkdv.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P, P, P, P, I64, P,
                                             P, P, ctypes.c_int]
        _lib.msa_oracle_bwd_kv_rows.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P, P, P, P, I64, P,
                                                P, P, ctypes.c_int]
    return _lib


@dataclass
class Dims:
    """Problem sizes.  ``blk`` is the KV block length (128 in MSA; smaller
    values are only used by brute-force self-tests of the oracle)."""
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int
    dp: int
    topk: int
    blk: int = 128
    scale: float = 0.0  # 0 -> 1/sqrt(d)
    window: int = 1     # forced blocks: own block and the window-1 before it,
    dilation: int = 1   # every `dilation`-th block

    @property
    def nblk(self) -> int:
        return (self.T + self.blk - 1) // self.blk

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def c(self) -> _Dims:
        s = self.scale if self.scale else 1.0 / np.sqrt(self.d)
        return _Dims(self.B, self.T, self.Hq, self.Hkv, self.d, self.dp, self.blk, self.topk, s,
                     self.window, self.dilation)


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


def _rows(rows, total):
    if rows is None:
        return np.arange(total, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def select(m: Dims, qp, kp, rows=None, want_pooled=False, idx=None, nsel=None, nthreads=None):
    """Index Branch for the listed rows ((b*Hp+g)*T+i; default all).

    Returns (idx [B,Hp,T,topk] int32, nsel [B,Hp,T] int32, pooled or None).
    Rows not listed keep the contents of the ``idx``/``nsel`` passed in (or
    -1/0).  ``pooled`` is [len(rows), nblk] float32 with -inf past the row's
    own block."""
    lib = _load()
    qp, kp = _f32(qp), _f32(kp)
    r = _rows(rows, m.B * m.Hkv * m.T)
    if idx is None:
        idx = np.full((m.B, m.Hkv, m.T, m.topk), -1, dtype=np.int32)
    if nsel is None:
        nsel = np.zeros((m.B, m.Hkv, m.T), dtype=np.int32)
    pooled = np.empty((len(r), m.nblk), dtype=np.float32) if want_pooled else None
    dm = m.c()
    lib.msa_oracle_select(ctypes.byref(dm), _ptr(qp), _ptr(kp), len(r), _ptr(r),
                          _ptr(pooled) if want_pooled else None, _ptr(idx), _ptr(nsel),
                          _threads(nthreads))
    return idx, nsel, pooled


def select_from_pooled(pooled, bi, topk, window=1, dilation=1):
    """The selection rule alone on given float32 scores [nrows, nblk] with the
    query's own block per row: returns (idx [nrows, topk], nsel [nrows])."""
    lib = _load()
    pooled = _f32(pooled)
    nrows, nb = pooled.shape
    bi = np.ascontiguousarray(np.asarray(bi, dtype=np.int32))
    idx = np.empty((nrows, topk), dtype=np.int32)
    nsel = np.empty((nrows,), dtype=np.int32)
    lib.msa_oracle_select_from_pooled(nrows, nb, topk, window, dilation, _ptr(pooled), _ptr(bi), _ptr(idx),
                                      _ptr(nsel))
    return idx, nsel


def fwd(m: Dims, q, k, v, idx, nsel, rows=None, o=None, lse=None, nthreads=None):
    """Main Branch forward for the listed rows ((b*Hq+h)*T+i; default all).
    Returns (O [B,T,Hq,d] float64, L [B,Hq,T] float64)."""
    lib = _load()
    q, k, v = _f32(q), _f32(k), _f32(v)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    nsel = np.ascontiguousarray(nsel, dtype=np.int32)
    r = _rows(rows, m.B * m.Hq * m.T)
    if o is None:
        o = np.zeros((m.B, m.T, m.Hq, m.d), dtype=np.float64)
    if lse is None:
        lse = np.zeros((m.B, m.Hq, m.T), dtype=np.float64)
    dm = m.c()
    lib.msa_oracle_fwd(ctypes.byref(dm), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(nsel),
                       len(r), _ptr(r), _ptr(o), _ptr(lse), _threads(nthreads))
    return o, lse


def bwd_dq(m: Dims, q, k, v, dout, o, lse, idx, nsel, rows=None, dq=None, D=None, nthreads=None):
    """dQ and D for the listed rows, from the oracle's own O and L."""
    lib = _load()
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    o = np.ascontiguousarray(o, dtype=np.float64)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    nsel = np.ascontiguousarray(nsel, dtype=np.int32)
    r = _rows(rows, m.B * m.Hq * m.T)
    if dq is None:
        dq = np.zeros((m.B, m.T, m.Hq, m.d), dtype=np.float64)
    if D is None:
        D = np.zeros((m.B, m.Hq, m.T), dtype=np.float64)
    dm = m.c()
    lib.msa_oracle_bwd_dq(ctypes.byref(dm), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(o),
                          _ptr(lse), _ptr(idx), _ptr(nsel), len(r), _ptr(r), _ptr(dq), _ptr(D),
                          _threads(nthreads))
    return dq, D


def bwd_dkdv(m: Dims, q, k, v, dout, lse, D, idx, nsel, blocks=None, dk=None, dv=None,
             nthreads=None):
    """dK, dV for the listed KV blocks ((b*Hkv+g)*nblk+n; default all).  Needs
    L and D of every query that selected each listed block."""
    lib = _load()
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    D = np.ascontiguousarray(D, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    nsel = np.ascontiguousarray(nsel, dtype=np.int32)
    bl = _rows(blocks, m.B * m.Hkv * m.nblk)
    if dk is None:
        dk = np.zeros((m.B, m.T, m.Hkv, m.d), dtype=np.float64)
    if dv is None:
        dv = np.zeros((m.B, m.T, m.Hkv, m.d), dtype=np.float64)
    dm = m.c()
    lib.msa_oracle_bwd_dkdv(ctypes.byref(dm), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse),
                            _ptr(D), _ptr(idx), _ptr(nsel), len(bl), _ptr(bl), _ptr(dk), _ptr(dv),
                            _threads(nthreads))
    return dk, dv


def bwd_kv_rows(m: Dims, q, k, v, dout, lse, D, idx, nsel, rows, nthreads=None):
    """Contributions of the listed query rows ((b*Hq+h)*T+i) to dK and dV of
    each key the row reads, [nrows, topk*blk, d] each (keys in the row's
    order, zero padded).  Needs the rows' L and D."""
    lib = _load()
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    D = np.ascontiguousarray(D, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    nsel = np.ascontiguousarray(nsel, dtype=np.int32)
    r = _rows(rows, m.B * m.Hq * m.T)
    dk = np.empty((len(r), m.topk * m.blk, m.d), dtype=np.float64)
    dv = np.empty((len(r), m.topk * m.blk, m.d), dtype=np.float64)
    dm = m.c()
    lib.msa_oracle_bwd_kv_rows(ctypes.byref(dm), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse),
                               _ptr(D), _ptr(idx), _ptr(nsel), len(r), _ptr(r), _ptr(dk), _ptr(dv),
                               _threads(nthreads))
    return dk, dv


def full(m: Dims, qp, kp, q, k, v, dout, nthreads=None):
    """The whole path on every row: selection, forward, backward."""
    idx, nsel, _ = select(m, qp, kp, nthreads=nthreads)
    o, lse = fwd(m, q, k, v, idx, nsel, nthreads=nthreads)
    dq, D = bwd_dq(m, q, k, v, dout, o, lse, idx, nsel, nthreads=nthreads)
    dk, dv = bwd_dkdv(m, q, k, v, dout, lse, D, idx, nsel, nthreads=nthreads)
    return dict(idx=idx, nsel=nsel, o=o, lse=lse, dq=dq, D=D, dk=dk, dv=dv)
