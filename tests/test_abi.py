"""The C ABI on the CPU: the library loads, exports every symbol the header
declares, and rejects bad arguments with a status code before launching
anything (these calls never reach the GPU)."""
import ctypes
import os
import re

import pytest

import exact_io_aware_71_b200 as fa
from exact_io_aware_71_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

A = 0x7F0000000000   # a 16-byte-aligned fake device address: never dereferenced


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = fa.load()
    names = declared_functions()
    assert set(names) == set(binding.SYMBOLS)
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_status_strings():
    for code, name in binding.STATUS_NAMES.items():
        assert fa.fa_status_string(code) == name
    assert fa.fa_status_string(99) == "FA_ERR_UNKNOWN"


def fwd(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, Hq=2, Hkv=2, Nq=128, Nk=128, d=64, causal=0,
             scale=0.125, stream=None)
    a.update(kw)
    return fa.fa_fwd(**a)


def bwd(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, dO=A, dq=A, dk=A, dv=A, B=1, Hq=2, Hkv=2, Nq=128,
             Nk=128, d=64, causal=0, scale=0.125, workspace=A, workspace_bytes=1 << 40,
             stream=None)
    a.update(kw)
    return fa.fa_bwd(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(B=0), 1), (dict(Nq=0), 1), (dict(Nk=0), 1),
    (dict(Hq=3, Hkv=2), 1), (dict(Hkv=0), 1), (dict(scale=0.0), 1), (dict(scale=-1.0), 1),
    (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1), (dict(causal=2), 1),
    (dict(d=32), 2), (dict(d=96), 2), (dict(d=512), 2),
    (dict(q=A + 8), 3), (dict(o=A + 2), 3), (dict(v=A + 4), 3), (dict(lse=A + 2), 3),
    (dict(B=1 << 20, Hq=1 << 10, Hkv=1 << 10), 2),
])
def test_fwd_rejects_bad_arguments(kw, status):
    assert fwd(**kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(dO=None), 1), (dict(dq=None), 1), (dict(Hq=4, Hkv=3), 1), (dict(d=48), 2),
    (dict(dk=A + 8), 3), (dict(workspace=None), 4), (dict(workspace_bytes=16), 4),
    (dict(workspace=A + 4), 3),
])
def test_bwd_rejects_bad_arguments(kw, status):
    assert bwd(**kw) == status


@pytest.mark.parametrize("stage", [-1, 4, 99])
def test_bwd_stage_rejects_unknown_stage(stage):
    a = dict(q=A, k=A, v=A, o=A, lse=A, dO=A, dq=A, dk=A, dv=A, B=1, Hq=2, Hkv=2, Nq=128,
             Nk=128, d=64, causal=0, scale=0.125, workspace=A, workspace_bytes=1 << 40,
             stream=None)
    assert fa.fa_bwd_stage(stage, **a) == 1


@pytest.mark.parametrize("bad,status", [
    ({"s0": ("row", 4)}, 3), ({"s1": ("head", 0)}, 3), ({"s3": ("batch", -64)}, 3),
    ({"s2": ("row", 1 << 40)}, 3),
])
def test_strided_rejects_bad_strides(bad, status):
    b = {k: v for k, v in bad.items()}
    s4 = [binding.FaStrides(1 << 20, 1 << 14, 64) for _ in range(4)]
    for key, (field, val) in b.items():
        setattr(s4[int(key[1:])], field, val)
    st = fa.fa_fwd_strided(A, A, A, A, A, s4, 1, 2, 2, 128, 128, 64, 0, 0.125, None)
    assert st == status
    s8 = [binding.FaStrides(1 << 20, 1 << 14, 64) for _ in range(8)]
    for key, (field, val) in b.items():
        setattr(s8[int(key[1:])], field, val)
    st = fa.fa_bwd_strided(A, A, A, A, A, A, A, A, A, s8, 1, 2, 2, 128, 128, 64, 0, 0.125, A,
                           1 << 40, None)
    assert st == status


def test_strided_rejects_null_strides():
    assert fa.fa_fwd_strided(A, A, A, A, A, None, 1, 2, 2, 128, 128, 64, 0, 0.125, None) == 1
    assert fa.fa_bwd_strided(A, A, A, A, A, A, A, A, A, None, 1, 2, 2, 128, 128, 64, 0, 0.125,
                             A, 1 << 40, None) == 1


def test_workspace_size():
    assert fa.fa_bwd_workspace_size(1, 2, 2, 128, 128, 64, 0) > 0
    assert fa.fa_bwd_workspace_size(0, 2, 2, 128, 128, 64, 0) == 0
    assert fa.fa_bwd_workspace_size(1, 3, 2, 128, 128, 64, 0) == 0
    assert fa.fa_bwd_workspace_size(1, 2, 2, 128, 128, 80, 0) == 0
    # grows with the problem
    a = fa.fa_bwd_workspace_size(1, 2, 2, 128, 128, 128, 0)
    b = fa.fa_bwd_workspace_size(2, 2, 2, 128, 128, 128, 0)
    assert b >= 2 * a - 4096


def test_missing_library_fails_loudly(tmp_path):
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(ImportError):
            binding.load(str(tmp_path / "nope.so"))
    finally:
        binding._lib = saved


def test_block_sparse_rejects_bad_arguments():
    """A null mask is rejected; otherwise the sparse entry points run the
    same argument checks as the dense ones (NULL strides = contiguous)."""
    assert fa.fa_fwd_block_sparse(A, A, A, A, A, None, None, 1, 2, 2, 128, 128, 64, 0, 0.125,
                                  None) == 1
    assert fa.fa_bwd_block_sparse(A, A, A, A, A, A, A, A, A, None, None, 1, 2, 2, 128, 128, 64,
                                  0, 0.125, A, 1 << 40, None) == 1
    assert fa.fa_fwd_block_sparse(A, A, A, A, A, None, A, 1, 2, 2, 128, 128, 96, 0, 0.125,
                                  None) == 2
    assert fa.fa_fwd_block_sparse(A + 8, A, A, A, A, None, A, 1, 2, 2, 128, 128, 64, 0, 0.125,
                                  None) == 3
    assert fa.fa_bwd_block_sparse(A, A, A, A, A, A, A, A, A, None, A, 1, 2, 2, 128, 128, 64, 0,
                                  0.125, None, 0, None) == 4
    assert fa.fa_fwd_block_sparse(A, A, A, A, A, None, A, 0, 2, 2, 128, 128, 64, 0, 0.125,
                                  None) == 1
    # the mask is read in aligned 16-byte chunks: it must start on a 16-byte boundary
    assert fa.fa_fwd_block_sparse(A, A, A, A, A, None, A + 1, 1, 2, 2, 128, 128, 64, 0, 0.125,
                                  None) == 3
    assert fa.fa_bwd_block_sparse(A, A, A, A, A, A, A, A, A, None, A + 8, 1, 2, 2, 128, 128, 64,
                                  0, 0.125, A, 1 << 40, None) == 3


def test_residual_entry_points_reject_bad_arguments():
    """fa_fwd_residual / fa_bwd_residual: the residual pointer is required
    and 16-byte aligned; the other checks are those of fa_fwd / fa_bwd."""
    f = lambda **kw: fa.fa_fwd_residual(**dict(dict(
        q=A, k=A, v=A, o=A, o_res=A, lse=A, strides=None, B=1, Hq=2, Hkv=2, Nq=128, Nk=128,
        d=64, causal=0, scale=0.125, stream=None), **kw))
    assert f(o_res=None) == 1 and f(q=None) == 1 and f(B=0) == 1 and f(d=80) == 2
    assert f(o_res=A + 8) == 3 and f(o=A + 2) == 3
    b = lambda **kw: fa.fa_bwd_residual(**dict(dict(
        q=A, k=A, v=A, o=A, o_res=A, lse=A, dO=A, dq=A, dk=A, dv=A, strides=None, B=1, Hq=2,
        Hkv=2, Nq=128, Nk=128, d=64, causal=0, scale=0.125, workspace=A,
        workspace_bytes=1 << 40, stream=None), **kw))
    assert b(o_res=None) == 1 and b(dO=None) == 1 and b(Hq=3) == 1
    assert b(o_res=A + 4) == 3 and b(workspace=None) == 4 and b(workspace_bytes=16) == 4


def test_varlen_rejects_bad_arguments():
    def fwd(**kw):
        a = dict(q=A, k=A, v=A, o=A, lse=A, cu_q=A, cu_k=A, B=2, max_q=100, max_k=100,
                 total_q=150, total_k=150, Hq=4, Hkv=2, d=64, causal=0, scale=0.125, stream=None)
        a.update(kw)
        return fa.fa_fwd_varlen(**a)
    assert fwd(cu_q=None) == 1 and fwd(cu_k=None) == 1 and fwd(q=None) == 1
    assert fwd(total_q=0) == 1 and fwd(B=0) == 1 and fwd(max_k=0) == 1
    assert fwd(Hq=3) == 1 and fwd(scale=0.0) == 1 and fwd(d=80) == 2
    assert fwd(cu_q=A + 2) == 3 and fwd(q=A + 8) == 3 and fwd(lse=A + 1) == 3
    a = dict(q=A, k=A, v=A, o=A, lse=A, dO=A, dq=A, dk=A, dv=A, cu_q=A, cu_k=A, B=2, max_q=100,
             max_k=100, total_q=150, total_k=150, Hq=4, Hkv=2, d=64, causal=0, scale=0.125,
             workspace=A, workspace_bytes=1 << 40, stream=None)
    assert fa.fa_bwd_varlen(**dict(a, workspace=None)) == 4
    assert fa.fa_bwd_varlen(**dict(a, workspace_bytes=64)) == 4
    assert fa.fa_bwd_varlen(**dict(a, dk=A + 8)) == 3
    assert fa.fa_bwd_varlen(**dict(a, cu_k=None)) == 1
    assert fa.fa_bwd_varlen_workspace_size(2, 150, 150, 4, 2, 64) > 150 * 4 * 64 * 4
    assert fa.fa_bwd_varlen_workspace_size(2, 150, 150, 4, 3, 64) == 0
