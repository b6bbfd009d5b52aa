"""C-ABI checks that need no GPU: the library loads, exports every function
include/msa.h declares, sizes its workspaces, and rejects bad arguments
before it would touch a device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_09_b200 import build
    build.build()
    from block_sparse_attention_09_b200 import msa
    return msa


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for required in ("msa_proxy_select", "msa_fwd", "msa_bwd", "msa_workspace_size", "msa_check_status",
                     "msa_strerror"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (msa_[a-z_0-9]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    # nothing but the C ABI leaks out of the library
    assert all(n.startswith("msa_") for n in exported)


def test_strerror(lib):
    assert lib.LIB.msa_strerror(0) == b"ok"
    assert lib.LIB.msa_strerror(-6) == b"device wait timed out"
    assert lib.LIB.msa_strerror(12345) == b"unknown status"


def dims(lib, **kw):
    base = dict(B=1, T=1024, Hq=4, Hkv=1, d=64, dp=32, topk=4)
    base.update(kw)
    return lib.make_dims(**base)


def test_window_fields_accepted(lib):
    """window 0..topk and any dilation >= 0 are valid; 0 means 1."""
    for w, s in ((0, 0), (1, 1), (4, 1), (3, 9), (2, 0)):
        assert lib.workspace_size(dims(lib, window=w, dilation=s), lib.MSA_SELECT) == 256


def test_decode_workspace(lib):
    """Decode keeps one index row per (sequence, group): a batch far beyond the
    training path's index bound is still valid there."""
    big = dims(lib, B=64, T=131072, Hq=32, Hkv=8, d=128, dp=64, topk=64)
    assert lib.workspace_size(big, lib.MSA_FWD) == 0
    ws = lib.workspace_size(big, lib.MSA_DECODE)
    # status + pooled [B*Hp*nblk] fp32 + partials [B*Hkv*topk*G*(d+2)] fp32
    assert ws >= 256 + 64 * 8 * 1024 * 4 + 64 * 8 * 64 * 4 * 130 * 4
    assert ws % 256 == 0


def test_workspace_sizes(lib):
    d = dims(lib)
    sel = lib.workspace_size(d, lib.MSA_SELECT)
    f = lib.workspace_size(d, lib.MSA_FWD)
    b = lib.workspace_size(d, lib.MSA_BWD)
    assert sel == 256
    nblk, rows = 8, 1024 * 4
    # index (count matrix, totals, pointers, token lists) + accumulators
    assert f >= 256 + nblk * nblk * 4 + 1024 * 4 * 4 + rows * 64 * 4
    assert b >= 256 + nblk * nblk * 4 + rows * 64 * 4
    assert f % 256 == 0 and b % 256 == 0


@pytest.mark.parametrize("bad", [dict(d=96), dict(dp=12), dict(dp=72), dict(topk=0), dict(topk=129),
                                 dict(Hq=6, Hkv=4), dict(Hq=12, Hkv=4), dict(T=-1), dict(T=(1 << 20) + 1),
                                 dict(window=5), dict(window=-1), dict(dilation=-2),
                                 dict(q_begin=64), dict(q_begin=-128), dict(q_begin=1152)])
def test_invalid_dims_rejected(lib, bad):
    d = dims(lib, **bad)
    assert lib.workspace_size(d, lib.MSA_FWD) == 0
    ws = ctypes.create_string_buffer(1 << 16)
    rc = lib.LIB.msa_fwd(ctypes.byref(d), 16, 16, 16, 16, 16, 16, 16, ctypes.addressof(ws), 1 << 16, None)
    assert rc == -1


def test_block_must_be_128(lib):
    d = dims(lib)
    d.block = 64
    assert lib.workspace_size(d, lib.MSA_SELECT) == 0


def test_hp_must_equal_hkv(lib):
    d = dims(lib)
    d.Hp = 2
    assert lib.workspace_size(d, lib.MSA_SELECT) == 0


def aligned_buffer(nbytes, align=256):
    raw = ctypes.create_string_buffer(nbytes + align)
    addr = (ctypes.addressof(raw) + align - 1) & ~(align - 1)
    return raw, addr


def test_argument_errors_before_any_launch(lib):
    d = dims(lib)
    need = lib.workspace_size(d, lib.MSA_FWD)
    raw, ws = aligned_buffer(64)
    P = 4096  # an aligned non-null stand-in; never dereferenced on these paths
    # workspace checks come first
    assert lib.LIB.msa_fwd(ctypes.byref(d), P, P, P, P, P, P, P, None, need, None) == -2
    assert lib.LIB.msa_fwd(ctypes.byref(d), P, P, P, P, P, P, P, ws + 16, need, None) == -3
    assert lib.LIB.msa_fwd(ctypes.byref(d), P, P, P, P, P, P, P, ws, need - 1, None) == -4
    # then tensor pointers
    assert lib.LIB.msa_fwd(ctypes.byref(d), None, P, P, P, P, P, P, ws, need, None) == -2
    assert lib.LIB.msa_fwd(ctypes.byref(d), P + 8, P, P, P, P, P, P, ws, need, None) == -3
    nb = lib.workspace_size(d, lib.MSA_BWD)
    assert lib.LIB.msa_bwd(ctypes.byref(d), P, P, P, P, P, P, P, P, P, P, None, ws, nb, None) == -2
    assert lib.LIB.msa_proxy_select(ctypes.byref(d), P, P + 4, P, P, None, ws, 256, None) == -3


def test_empty_problem_is_a_no_op(lib):
    raw, ws = aligned_buffer(1 << 12)
    for kw in (dict(T=0), dict(B=0)):
        d = dims(lib, **kw)
        need = lib.workspace_size(d, lib.MSA_FWD)
        assert lib.LIB.msa_fwd(ctypes.byref(d), None, None, None, None, None, None, None, ws, need,
                               None) == 0
        assert lib.LIB.msa_proxy_select(ctypes.byref(d), None, None, None, None, None, ws, 256, None) == 0


def test_no_gpu_reports_device_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    d = dims(lib)
    raw, ws = aligned_buffer(256)
    P = 4096
    assert lib.LIB.msa_proxy_select(ctypes.byref(d), P, P, P, P, None, ws, 256, None) == -7


def test_q_begin_fields(lib):
    """q_begin: a block boundary inside [0, T]; the workspaces keep their
    full-sequence size (the shard's rows sit in place in [0, T))."""
    full = lib.workspace_size(dims(lib), lib.MSA_FWD)
    for qb in (0, 128, 896, 1024):
        assert lib.workspace_size(dims(lib, q_begin=qb), lib.MSA_FWD) == full
    # ragged T: the last block boundary below T is valid, T itself too
    assert lib.workspace_size(dims(lib, T=1000, q_begin=896), lib.MSA_SELECT) == 256
    # decode has one query per sequence: no shard start
    assert lib.workspace_size(dims(lib, q_begin=128), lib.MSA_DECODE) == 0


def test_q_begin_at_t_only_clears_the_status(lib):
    """Nothing to compute: selection and forward read no tensor pointer and
    launch no kernel, but they clear the workspace's status words (so a
    following msa_check_status describes this call), which needs a device:
    without one they report MSA_ERR_DEVICE.  tests/test_gpu_zz_cp.py covers
    the device side."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    raw, ws = aligned_buffer(1 << 20)
    d = dims(lib, q_begin=1024)
    need = lib.workspace_size(d, lib.MSA_FWD)
    assert lib.LIB.msa_fwd(ctypes.byref(d), None, None, None, None, None, None, None, ws, need, None) == -7
    assert lib.LIB.msa_proxy_select(ctypes.byref(d), None, None, None, None, None, ws, 256, None) == -7
    # the backward zeroes dk, dv: it needs them (and a device)
    nb = lib.workspace_size(d, lib.MSA_BWD)
    assert lib.LIB.msa_bwd(ctypes.byref(d), None, None, None, None, None, None, None, None, None, None, None,
                           ws, nb, None) == -2


def test_noalloc_status_needs_a_device(lib):
    """The no-alloc status read looks up the library's scratch array on the
    current device; without a device it reports MSA_ERR_DEVICE."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    code = ctypes.c_uint32(7)
    assert lib.LIB.msa_fwd_noalloc_status(None, ctypes.byref(code)) == -7
    assert lib.LIB.msa_fwd_noalloc_status(None, None) == -7


def test_f32_to_bf16_argument_checks(lib):
    P = 4096
    assert lib.LIB.msa_f32_to_bf16(P, P, 12, None) == -1      # not a multiple of 8
    assert lib.LIB.msa_f32_to_bf16(P, P, -8, None) == -1
    assert lib.LIB.msa_f32_to_bf16(None, None, 0, None) == 0  # empty
    assert lib.LIB.msa_f32_to_bf16(None, P, 8, None) == -2
    assert lib.LIB.msa_f32_to_bf16(P + 4, P, 8, None) == -3

