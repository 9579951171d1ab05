"""ctypes binding of libfa's C ABI (include/fa.h).

Argument marshalling only: every step of the attention computation runs in
the CUDA kernels behind these calls.  There is no fallback; if the shared
library is missing, loading fails with an error that says how to build it.
The functions named like the C entry points take raw device pointers (ints);
``forward`` / ``backward`` accept contiguous torch CUDA tensors, allocate the
outputs with torch (device memory only) and call the same entry points on
torch's current stream.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa.so")

FA_OK = 0
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED",
                3: "FA_ERR_MISALIGNED", 4: "FA_ERR_WORKSPACE", 5: "FA_ERR_CUDA",
                6: "FA_ERR_DEVICE_TIMEOUT", 7: "FA_ERR_TOO_LARGE"}

# Exported symbols declared in include/fa.h.
SYMBOLS = ("fa_fwd", "fa_bwd", "fa_bwd_stage", "fa_bwd_workspace_size", "fa_status_string",
           "fa_device_status", "fa_bwd_noalloc", "fa_debug_inject", "fa_fwd_strided",
           "fa_bwd_strided", "fa_fwd_block_sparse", "fa_bwd_block_sparse", "fa_fwd_varlen",
           "fa_bwd_varlen", "fa_bwd_varlen_workspace_size", "fa_fwd_residual",
           "fa_bwd_residual")

# Rows / keys per block-mask entry (FA_MASK_BLOCK).
MASK_BLOCK = 128

# Bytes of the built-in scratch behind fa_bwd_noalloc (FA_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 64 << 20

FA_BWD_ALL, FA_BWD_PRE, FA_BWD_MAIN, FA_BWD_DQ = 0, 1, 2, 3


class FaStrides(ctypes.Structure):
    """fa_strides: element strides (batch, head, row) of a [B, H, N, d] view."""
    _fields_ = [("batch", ctypes.c_longlong), ("head", ctypes.c_longlong),
                ("row", ctypes.c_longlong)]


def strides_of(t) -> FaStrides:
    """fa_strides of a torch tensor viewed as [B, H, N, d] with d contiguous."""
    if t.stride(-1) != 1:
        raise ValueError("the last (head-dim) axis must be contiguous")
    return FaStrides(t.stride(0), t.stride(1), t.stride(2))


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python exact_io_aware_71_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp]
    lib.fa_fwd.restype = i
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp, sz, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_stage.argtypes = [i] + lib.fa_bwd.argtypes
    sp = ctypes.POINTER(FaStrides)
    lib.fa_fwd_strided.argtypes = [vp, vp, vp, vp, vp, sp, i, i, i, i, i, i, i, f, vp]
    lib.fa_fwd_strided.restype = i
    lib.fa_bwd_strided.argtypes = [vp] * 9 + [sp] + [i] * 7 + [f, vp, sz, vp]
    lib.fa_bwd_strided.restype = i
    lib.fa_bwd_stage.restype = i
    lib.fa_fwd_block_sparse.argtypes = [vp] * 5 + [sp, vp] + [i] * 7 + [f, vp]
    lib.fa_fwd_block_sparse.restype = i
    lib.fa_bwd_block_sparse.argtypes = [vp] * 9 + [sp, vp] + [i] * 7 + [f, vp, sz, vp]
    lib.fa_bwd_block_sparse.restype = i
    lib.fa_fwd_varlen.argtypes = [vp] * 7 + [i] * 9 + [f, vp]
    lib.fa_fwd_varlen.restype = i
    lib.fa_bwd_varlen.argtypes = [vp] * 11 + [i] * 9 + [f, vp, sz, vp]
    lib.fa_bwd_varlen.restype = i
    lib.fa_bwd_varlen_workspace_size.argtypes = [i] * 6
    lib.fa_bwd_varlen_workspace_size.restype = sz
    lib.fa_fwd_residual.argtypes = [vp] * 6 + [sp] + [i] * 7 + [f, vp]
    lib.fa_fwd_residual.restype = i
    lib.fa_bwd_residual.argtypes = [vp] * 10 + [sp] + [i] * 7 + [f, vp, sz, vp]
    lib.fa_bwd_residual.restype = i
    lib.fa_bwd_noalloc.argtypes = lib.fa_bwd.argtypes[:17] + [vp]
    lib.fa_bwd_noalloc.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.fa_device_status.restype = i
    lib.fa_debug_inject.argtypes = [i, ctypes.c_double]
    lib.fa_debug_inject.restype = i
    _lib = lib
    return lib


# ------------------------------------------------------------ raw C entry points
def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, stream) -> int:
    return load().fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, int(causal), float(scale),
                         stream)


def fa_fwd_strided(q, k, v, o, lse, strides, B, Hq, Hkv, Nq, Nk, d, causal, scale, stream) -> int:
    arr = (FaStrides * 4)(*strides) if strides is not None else None
    return load().fa_fwd_strided(q, k, v, o, lse, arr, B, Hq, Hkv, Nq, Nk, d, int(causal),
                                 float(scale), stream)


def fa_bwd_strided(q, k, v, o, lse, dO, dq, dk, dv, strides, B, Hq, Hkv, Nq, Nk, d, causal,
                   scale, workspace, workspace_bytes, stream) -> int:
    arr = (FaStrides * 8)(*strides) if strides is not None else None
    return load().fa_bwd_strided(q, k, v, o, lse, dO, dq, dk, dv, arr, B, Hq, Hkv, Nq, Nk, d,
                                 int(causal), float(scale), workspace, workspace_bytes, stream)


def fa_fwd_residual(q, k, v, o, o_res, lse, strides, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                    stream) -> int:
    arr = (FaStrides * 4)(*strides) if strides is not None else None
    return load().fa_fwd_residual(q, k, v, o, o_res, lse, arr, B, Hq, Hkv, Nq, Nk, d,
                                  int(causal), float(scale), stream)


def fa_bwd_residual(q, k, v, o, o_res, lse, dO, dq, dk, dv, strides, B, Hq, Hkv, Nq, Nk, d,
                    causal, scale, workspace, workspace_bytes, stream) -> int:
    arr = (FaStrides * 8)(*strides) if strides is not None else None
    return load().fa_bwd_residual(q, k, v, o, o_res, lse, dO, dq, dk, dv, arr, B, Hq, Hkv, Nq,
                                  Nk, d, int(causal), float(scale), workspace, workspace_bytes,
                                  stream)


def fa_fwd_block_sparse(q, k, v, o, lse, strides, block_mask, B, Hq, Hkv, Nq, Nk, d, causal,
                        scale, stream) -> int:
    arr = (FaStrides * 4)(*strides) if strides is not None else None
    return load().fa_fwd_block_sparse(q, k, v, o, lse, arr, block_mask, B, Hq, Hkv, Nq, Nk, d,
                                      int(causal), float(scale), stream)


def fa_bwd_block_sparse(q, k, v, o, lse, dO, dq, dk, dv, strides, block_mask, B, Hq, Hkv, Nq, Nk,
                        d, causal, scale, workspace, workspace_bytes, stream) -> int:
    arr = (FaStrides * 8)(*strides) if strides is not None else None
    return load().fa_bwd_block_sparse(q, k, v, o, lse, dO, dq, dk, dv, arr, block_mask, B, Hq,
                                      Hkv, Nq, Nk, d, int(causal), float(scale), workspace,
                                      workspace_bytes, stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, max_q, max_k, total_q, total_k, Hq, Hkv, d,
                  causal, scale, stream) -> int:
    return load().fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, max_q, max_k, total_q, total_k,
                                Hq, Hkv, d, int(causal), float(scale), stream)


def fa_bwd_varlen(q, k, v, o, lse, dO, dq, dk, dv, cu_q, cu_k, B, max_q, max_k, total_q, total_k,
                  Hq, Hkv, d, causal, scale, workspace, workspace_bytes, stream) -> int:
    return load().fa_bwd_varlen(q, k, v, o, lse, dO, dq, dk, dv, cu_q, cu_k, B, max_q, max_k,
                                total_q, total_k, Hq, Hkv, d, int(causal), float(scale),
                                workspace, workspace_bytes, stream)


def fa_bwd_varlen_workspace_size(B, total_q, total_k, Hq, Hkv, d) -> int:
    return load().fa_bwd_varlen_workspace_size(B, total_q, total_k, Hq, Hkv, d)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal, scale,
           workspace, workspace_bytes, stream) -> int:
    return load().fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, int(causal),
                         float(scale), workspace, workspace_bytes, stream)


def fa_bwd_stage(stage, q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                 workspace, workspace_bytes, stream) -> int:
    return load().fa_bwd_stage(stage, q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d,
                               int(causal), float(scale), workspace, workspace_bytes, stream)


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                   stream) -> int:
    """fa_bwd without a caller workspace: scratch is the library's built-in
    device array (for callers that cannot allocate device memory)."""
    return load().fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d,
                                 int(causal), float(scale), stream)


def fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d, causal) -> int:
    return load().fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d, int(causal))


def fa_status_string(status: int) -> str:
    return load().fa_status_string(status).decode()


def fa_debug_inject(stall_kv_loads: int, wait_limit_seconds: float) -> int:
    """Test control for the timeout path (see include/fa.h)."""
    return load().fa_debug_inject(int(stall_kv_loads), float(wait_limit_seconds))


def fa_device_status(stream=None):
    where = ctypes.c_int(0)
    st = load().fa_device_status(stream, ctypes.byref(where))
    return st, where.value


# ------------------------------------------------------------ torch convenience
def _stream_handle():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _dims(q, k):
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    return B, Hq, Hkv, Nq, Nk, d


def _mask_ptr(block_mask, Nq, Nk):
    """Device address of a [ceil(Nq/128), ceil(Nk/128)] uint8 / bool CUDA mask."""
    import torch
    shape = ((Nq + MASK_BLOCK - 1) // MASK_BLOCK, (Nk + MASK_BLOCK - 1) // MASK_BLOCK)
    if tuple(block_mask.shape) != shape:
        raise ValueError(f"block mask must have shape {shape}, got {tuple(block_mask.shape)}")
    if block_mask.dtype not in (torch.uint8, torch.bool) or not block_mask.is_cuda \
            or not block_mask.is_contiguous():
        raise ValueError("block mask must be a contiguous uint8 or bool CUDA tensor")
    return block_mask.data_ptr()


def forward(q, k, v, causal: bool, scale: float, out=None, lse=None, block_mask=None,
            o_res=None):
    """O, LSE for bf16 CUDA tensors q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] (any
    strides with a contiguous last axis, e.g. permuted [B,N,H,d] storage).
    block_mask: optional block-sparse mask, [ceil(Nq/128), ceil(Nk/128)].
    o_res: optional tensor shaped and strided like the output that receives
    its rounding residual (fa_fwd_residual; not with a block mask)."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=q.device)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr())
    strides = [strides_of(t) for t in (q, k, v, out)]
    if o_res is not None:
        if block_mask is not None or o_res.stride() != out.stride() or o_res.shape != out.shape:
            raise ValueError("o_res must be shaped and strided like the output, without a mask")
        st = fa_fwd_residual(*ptrs[:4], o_res.data_ptr(), ptrs[4], strides, B, Hq, Hkv, Nq, Nk, d,
                             causal, scale, _stream_handle())
        what = "fa_fwd_residual"
    elif block_mask is None:
        st = fa_fwd_strided(*ptrs, strides, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                            _stream_handle())
        what = "fa_fwd_strided"
    else:
        st = fa_fwd_block_sparse(*ptrs, strides, _mask_ptr(block_mask, Nq, Nk), B, Hq, Hkv, Nq,
                                 Nk, d, causal, scale, _stream_handle())
        what = "fa_fwd_block_sparse"
    if st != FA_OK:
        raise FaError(st, what)
    return out, lse


def backward(q, k, v, o, lse, do, causal: bool, scale: float, workspace=None, grads=None,
             block_mask=None, o_res=None):
    """dQ, dK, dV (bf16) for the forward inputs/outputs and dO; gradients
    take the strides of q, k, v unless `grads` gives the output tensors.
    block_mask: the forward pass's block-sparse mask, if it had one.
    o_res: the forward's residual output (fa_bwd_residual), if kept."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _dims(q, k)
    need = fa_bwd_workspace_size(B, Hq, Hkv, Nq, Nk, d, causal)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k),
                                                  torch.empty_like(v))
    ts = (q, k, v, o, do, dq, dk, dv)
    ptrs = (*(t.data_ptr() for t in ts[:4]), lse.data_ptr(), *(t.data_ptr() for t in ts[4:]))
    strides = [strides_of(t) for t in ts]
    if o_res is not None:
        if block_mask is not None or o_res.stride() != o.stride() or o_res.shape != o.shape:
            raise ValueError("o_res must be shaped and strided like o, without a mask")
        st = fa_bwd_residual(*ptrs[:4], o_res.data_ptr(), *ptrs[4:], strides, B, Hq, Hkv, Nq, Nk,
                             d, causal, scale, workspace.data_ptr(), workspace.numel(),
                             _stream_handle())
        what = "fa_bwd_residual"
    elif block_mask is None:
        st = fa_bwd_strided(*ptrs, strides, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                            workspace.data_ptr(), workspace.numel(), _stream_handle())
        what = "fa_bwd_strided"
    else:
        st = fa_bwd_block_sparse(*ptrs, strides, _mask_ptr(block_mask, Nq, Nk), B, Hq, Hkv, Nq,
                                 Nk, d, causal, scale, workspace.data_ptr(), workspace.numel(),
                                 _stream_handle())
        what = "fa_bwd_block_sparse"
    if st != FA_OK:
        raise FaError(st, what)
    return dq, dk, dv


def _varlen_dims(q, k, cu_q, cu_k):
    import torch
    for t in (q, k):
        if t.dim() != 3 or not t.is_contiguous():
            raise ValueError("packed q / k / v must be contiguous [total, H, d]")
    for c in (cu_q, cu_k):
        if c.dtype != torch.int32 or not c.is_cuda or not c.is_contiguous() or c.dim() != 1:
            raise ValueError("cu_seqlens must be contiguous int32 CUDA vectors of length B + 1")
    if cu_q.numel() != cu_k.numel() or cu_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 >= 2 entries")
    return cu_q.numel() - 1, q.shape[0], k.shape[0], q.shape[1], k.shape[1], q.shape[2]


def forward_varlen(q, k, v, cu_q, cu_k, max_q, max_k, causal: bool, scale: float, out=None,
                   lse=None):
    """O [total_q, Hq, d] and LSE [Hq, total_q] of a packed variable-length
    batch (q [total_q, Hq, d], k / v [total_k, Hkv, d], int32 cumulative
    offsets cu_q / cu_k of length B + 1, all on the GPU)."""
    import torch
    B, tq, tk, Hq, Hkv, d = _varlen_dims(q, k, cu_q, cu_k)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, tq, dtype=torch.float32, device=q.device)
    st = fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                       cu_q.data_ptr(), cu_k.data_ptr(), B, int(max_q), int(max_k), tq, tk, Hq,
                       Hkv, d, causal, scale, _stream_handle())
    if st != FA_OK:
        raise FaError(st, "fa_fwd_varlen")
    return out, lse


def backward_varlen(q, k, v, o, lse, do, cu_q, cu_k, max_q, max_k, causal: bool, scale: float,
                    workspace=None, grads=None):
    """dQ, dK, dV (packed, bf16) of a variable-length batch; `grads` may
    give contiguous output tensors shaped like q, k, v."""
    import torch
    B, tq, tk, Hq, Hkv, d = _varlen_dims(q, k, cu_q, cu_k)
    need = fa_bwd_varlen_workspace_size(B, tq, tk, Hq, Hkv, d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k),
                                                  torch.empty_like(v))
    st = fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                       cu_q.data_ptr(), cu_k.data_ptr(), B, int(max_q), int(max_k), tq, tk, Hq,
                       Hkv, d, causal, scale, workspace.data_ptr(), workspace.numel(),
                       _stream_handle())
    if st != FA_OK:
        raise FaError(st, "fa_bwd_varlen")
    return dq, dk, dv
