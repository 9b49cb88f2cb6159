"""B200-native (sm_100a) mean-pooled top-k block-sparse attention.

Thin Python binding over the C ABI in include/bsa.h (libbsa.so, built in-tree
by ``python -m block_sparse_attention_14_b200.build``).  This module only
marshals arguments -- it checks tensor devices, dtypes and shapes, allocates
outputs and the workspace with torch, and passes raw pointers and the current
CUDA stream.  Every step of the computation runs in the library's kernels;
there is no CPU or eager fallback, and the calls raise if the library is
missing.

API, after "SpargeAttention Documentation":

* ``sparse_attn_topk(q, k, v, topk=0.5, is_causal=False)`` -- selection plus
  attention, the counterpart of spas_sage2_attn_meansim_topk_cuda;
* ``block_sparse_attn_fwd(q, k, v, mask_id=None, is_causal=False)`` --
  attention over a caller mask, the counterpart of block_sparse_sage2_attn_cuda;
* ``sparse_attn_select(q, k, topk)`` -- the selection mask alone, so that a
  mask can be computed once and re-applied (the build_plan / apply_plan split
  of the AB-Attention README);
* ``sparse_attn_block_scores(q, k)`` -- the compressed block-score map.

q, k, v are CUDA bf16 tensors of shape [B, H, N, d] (d = 64 or 128).

Every call is asynchronous on the current CUDA stream.  The kernels' waits are
bounded; a call whose wait ran out leaves some output rows unwritten, which the
library reports only through its device status word.  ``check=True`` reads that
word after the call (synchronising the stream) and raises ``BsaError`` with
status BSA_ERR_TIMEOUT; ``last_device_status(workspace)`` does the same later.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "BsaError", "sparse_attn_topk", "block_sparse_attn_fwd", "sparse_attn_select",
    "sparse_attn_block_scores", "sparse_attn_select_cdf", "sparse_attn_cdf", "workspace_bytes", "make_workspace", "last_device_status",
    "set_wait_timeout_ns", "token_permutation", "permute_tokens", "block_sparse_attn_plan", "block_sparse_attn_apply",
    "sparse_attn_topk_host", "sparse_attn_topk_noalloc", "noalloc_status", "block_counts", "library_path", "lib",
]

BLOCK_Q = 128
BLOCK_K = 64
_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libbsa.so")
_LIB = None

STATUS = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED", 3: "BSA_ERR_CUDA",
          4: "BSA_ERR_TIMEOUT"}


class BsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libbsa.so (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_attention_14_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, sz, i32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        L.bsa_abi_version.restype = i32
        L.bsa_status_string.restype = ctypes.c_char_p
        L.bsa_status_string.argtypes = [i32]
        L.bsa_last_error_message.restype = ctypes.c_char_p
        L.bsa_workspace_bytes.restype = sz
        L.bsa_workspace_bytes.argtypes = [Shape]
        L.sparse_attn_block_scores.restype = i32
        L.sparse_attn_block_scores.argtypes = [vp, vp, Shape, vp, vp, sz, vp]
        L.sparse_attn_select.restype = i32
        L.sparse_attn_select.argtypes = [vp, vp, Shape, f32, i32, vp, vp, sz, vp]
        L.block_sparse_attn_fwd.restype = i32
        L.block_sparse_attn_fwd.argtypes = [vp, vp, vp, Shape, vp, i32, vp, vp, sz, vp]
        L.sparse_attn_topk.restype = i32
        L.sparse_attn_topk.argtypes = [vp, vp, vp, Shape, f32, i32, vp, vp, vp, sz, vp]
        L.sparse_attn_select_cdf.restype = i32
        L.sparse_attn_select_cdf.argtypes = [vp, vp, Shape, f32, vp, vp, sz, vp]
        L.sparse_attn_cdf.restype = i32
        L.sparse_attn_cdf.argtypes = [vp, vp, vp, Shape, f32, i32, vp, vp, vp, sz, vp]
        L.sparse_attn_topk_host.restype = i32
        L.sparse_attn_topk_host.argtypes = [vp, vp, vp, Shape, f32, i32, vp, vp, vp, vp, vp, vp, sz, i32, vp]
        L.block_sparse_attn_plan.restype = i32
        L.block_sparse_attn_plan.argtypes = [vp, Shape, i32, vp, sz, vp]
        L.block_sparse_attn_apply.restype = i32
        L.block_sparse_attn_apply.argtypes = [vp, vp, vp, Shape, i32, vp, vp, sz, vp]
        L.bsa_token_permutation.restype = i32
        L.bsa_token_permutation.argtypes = [i32, i32, i32, i32, i32, vp]
        L.bsa_permute_tokens.restype = i32
        L.bsa_permute_tokens.argtypes = [vp, vp, Shape, vp, i32, vp]
        L.bsa_last_device_status.restype = i32
        L.bsa_last_device_status.argtypes = [vp, vp]
        L.bsa_set_wait_timeout_ns.restype = None
        L.bsa_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        L.sparse_attn_topk_noalloc.restype = i32
        L.sparse_attn_topk_noalloc.argtypes = [vp, vp, vp, Shape, f32, i32, vp, vp, vp]
        L.sparse_attn_topk_noalloc_status.restype = i32
        L.sparse_attn_topk_noalloc_status.argtypes = [vp]
        _LIB = L
    return _LIB


def _check(status: int) -> None:
    if status != 0:
        raise BsaError(status, lib().bsa_last_error_message().decode())


def block_counts(N: int) -> tuple[int, int]:
    return -(-N // BLOCK_Q), -(-N // BLOCK_K)


def _shape_of(q: torch.Tensor) -> Shape:
    B, H, N, d = q.shape
    return Shape(B, H, N, d)


def _qkv(*ts: torch.Tensor) -> None:
    ref = ts[0]
    if ref.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    for t in ts:
        if not t.is_cuda:
            raise ValueError("q, k, v must be CUDA tensors")
        if t.dtype != torch.bfloat16:
            raise ValueError("q, k, v must be bf16")
        if t.shape != ref.shape:
            raise ValueError(f"shape mismatch: {tuple(t.shape)} vs {tuple(ref.shape)}")
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous [B, H, N, d]")
        if t.device != ref.device:
            raise ValueError("q, k, v must be on one device")


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().bsa_workspace_bytes(Shape(B, H, N, d)))


def make_workspace(B: int, H: int, N: int, d: int, device="cuda") -> torch.Tensor:
    """A workspace for the shape; its device status word (the first 256 bytes) starts
    cleared, so last_device_status reports BSA_OK before any call has used it."""
    n = workspace_bytes(B, H, N, d)
    if n == 0:
        raise BsaError(1, lib().bsa_last_error_message().decode() or "shape rejected")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def _ws(q: torch.Tensor, workspace):
    B, H, N, d = q.shape
    if workspace is None:
        workspace = make_workspace(B, H, N, d, q.device)
    return workspace, workspace.data_ptr(), workspace.numel()


def _mask_arg(mask: torch.Tensor, q: torch.Tensor) -> torch.Tensor:
    B, H, N, _ = q.shape
    Qb, Kb = block_counts(N)
    if tuple(mask.shape) != (B, H, Qb, Kb):
        raise ValueError(f"mask_id must have shape {(B, H, Qb, Kb)}, got {tuple(mask.shape)}")
    if mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    if mask.dtype != torch.uint8:
        raise ValueError("mask_id must be uint8 or bool")
    if not mask.is_cuda or mask.device != q.device or not mask.is_contiguous():
        raise ValueError("mask_id must be a contiguous tensor on q's device")
    return mask


def _checked(ws, check: bool) -> None:
    if check:
        last_device_status(ws)


def sparse_attn_topk(q, k, v, topk: float = 0.5, is_causal: bool = False, *, out=None,
                     return_mask: bool = False, workspace=None, check: bool = False):
    """Top-k block selection followed by block-sparse attention.

    Returns out (bf16 [B, H, N, d]), or (out, mask) with return_mask=True.
    """
    _qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    _qkv(q, out)
    B, H, N, _ = q.shape
    mask = torch.empty(B, H, *block_counts(N), dtype=torch.uint8, device=q.device) if return_mask else None
    ws, wp, wn = _ws(q, workspace)
    _check(lib().sparse_attn_topk(q.data_ptr(), k.data_ptr(), v.data_ptr(), _shape_of(q), float(topk),
                                  int(bool(is_causal)), out.data_ptr(),
                                  mask.data_ptr() if mask is not None else None, wp, wn, _stream(q)))
    _checked(ws, check)
    return (out, mask) if return_mask else out


def sparse_attn_topk_host(q_host, k_host, v_host, topk: float = 0.5, is_causal: bool = False, *,
                          out_host=None, device_buffers=None, workspace=None, chunks: int = 0,
                          device="cuda", check: bool = False):
    """sparse_attn_topk on pinned host tensors, with the host<->device copies
    pipelined over chunks of heads.  device_buffers: (q, k, v, out) device tensors
    of the same shape (allocated if None).  Runs on the current stream of
    `device`; returns out_host once that stream has finished."""
    for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_pinned():
            raise ValueError(f"{name} must be a contiguous pinned bf16 host tensor")
        if t.shape != q_host.shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(q_host.shape)}")
    if out_host is None:
        out_host = torch.empty(q_host.shape, dtype=torch.bfloat16).pin_memory()
    if device_buffers is None:
        device_buffers = tuple(torch.empty(q_host.shape, dtype=torch.bfloat16, device=device) for _ in range(4))
    qd, kd, vd, od = device_buffers
    _qkv(qd, kd, vd)
    _qkv(qd, od)
    ws, wp, wn = _ws(qd, workspace)
    _check(lib().sparse_attn_topk_host(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                                       _shape_of(qd), float(topk), int(bool(is_causal)),
                                       out_host.data_ptr(), qd.data_ptr(), kd.data_ptr(), vd.data_ptr(),
                                       od.data_ptr(), wp, wn, int(chunks), _stream(qd)))
    torch.cuda.current_stream(qd.device).synchronize()
    _checked(ws, check)
    return out_host


def block_sparse_attn_fwd(q, k, v, mask_id=None, is_causal: bool = False, *, out=None, workspace=None,
                          check: bool = False):
    """Attention over the kept 128 x 64 tiles of mask_id ([B, H, ceil(N/128), ceil(N/64)],
    nonzero = keep; None = dense)."""
    _qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    _qkv(q, out)
    m = _mask_arg(mask_id, q) if mask_id is not None else None
    ws, wp, wn = _ws(q, workspace)
    _check(lib().block_sparse_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), _shape_of(q),
                                       m.data_ptr() if m is not None else None, int(bool(is_causal)),
                                       out.data_ptr(), wp, wn, _stream(q)))
    _checked(ws, check)
    return out


def sparse_attn_select(q, k, topk: float, is_causal: bool = False, *, mask_out=None,
                       workspace=None) -> torch.Tensor:
    """Selection mask alone: uint8 [B, H, ceil(N/128), ceil(N/64)].  With is_causal,
    row i chooses among its key blocks 0 .. 2i+1 only."""
    _qkv(q, k)
    B, H, N, _ = q.shape
    if mask_out is None:
        mask_out = torch.empty(B, H, *block_counts(N), dtype=torch.uint8, device=q.device)
    mask_out = _mask_arg(mask_out, q)
    ws, wp, wn = _ws(q, workspace)
    _check(lib().sparse_attn_select(q.data_ptr(), k.data_ptr(), _shape_of(q), float(topk),
                                    int(bool(is_causal)), mask_out.data_ptr(), wp, wn, _stream(q)))
    return mask_out


def sparse_attn_select_cdf(q, k, threshold: float, *, mask_out=None, workspace=None) -> torch.Tensor:
    """cdfthreshd selection mask: per row, the shortest score-ordered prefix of key
    blocks whose block-score mass reaches `threshold` (uint8 [B, H, Qb, Kb])."""
    _qkv(q, k)
    B, H, N, _ = q.shape
    if mask_out is None:
        mask_out = torch.empty(B, H, *block_counts(N), dtype=torch.uint8, device=q.device)
    mask_out = _mask_arg(mask_out, q)
    ws, wp, wn = _ws(q, workspace)
    _check(lib().sparse_attn_select_cdf(q.data_ptr(), k.data_ptr(), _shape_of(q), float(threshold),
                                        mask_out.data_ptr(), wp, wn, _stream(q)))
    return mask_out


def sparse_attn_cdf(q, k, v, threshold: float = 0.9, is_causal: bool = False, *, out=None,
                    return_mask: bool = False, workspace=None, check: bool = False):
    """cdfthreshd selection followed by block-sparse attention."""
    _qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    _qkv(q, out)
    B, H, N, _ = q.shape
    mask = torch.empty(B, H, *block_counts(N), dtype=torch.uint8, device=q.device) if return_mask else None
    ws, wp, wn = _ws(q, workspace)
    _check(lib().sparse_attn_cdf(q.data_ptr(), k.data_ptr(), v.data_ptr(), _shape_of(q), float(threshold),
                                 int(bool(is_causal)), out.data_ptr(),
                                 mask.data_ptr() if mask is not None else None, wp, wn, _stream(q)))
    _checked(ws, check)
    return (out, mask) if return_mask else out


def sparse_attn_block_scores(q, k, *, out=None, workspace=None) -> torch.Tensor:
    """Compressed block-score map softmax(Qbar Kbar^T / sqrt(d)): fp32 [B, H, Qb, Kb]."""
    _qkv(q, k)
    B, H, N, _ = q.shape
    if out is None:
        out = torch.empty(B, H, *block_counts(N), dtype=torch.float32, device=q.device)
    if out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != (B, H, *block_counts(N)):
        raise ValueError("out must be a contiguous fp32 [B, H, Qb, Kb] tensor")
    ws, wp, wn = _ws(q, workspace)
    _check(lib().sparse_attn_block_scores(q.data_ptr(), k.data_ptr(), _shape_of(q), out.data_ptr(),
                                          wp, wn, _stream(q)))
    return out


def block_sparse_attn_plan(q, mask_id=None, is_causal: bool = False, *, workspace=None) -> torch.Tensor:
    """Compact mask_id (None = dense) into a reusable plan held in the returned workspace."""
    B, H, N, d = q.shape
    m = _mask_arg(mask_id, q) if mask_id is not None else None
    ws, wp, wn = _ws(q, workspace)
    _check(lib().block_sparse_attn_plan(m.data_ptr() if m is not None else None, _shape_of(q),
                                        int(bool(is_causal)), wp, wn, _stream(q)))
    return ws


def block_sparse_attn_apply(q, k, v, workspace, is_causal: bool = False, *, out=None, check: bool = False):
    """Attention over the plan held in `workspace` (from sparse_attn_select,
    sparse_attn_topk or block_sparse_attn_plan on the same shape)."""
    _qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    _qkv(q, out)
    _check(lib().block_sparse_attn_apply(q.data_ptr(), k.data_ptr(), v.data_ptr(), _shape_of(q),
                                         int(bool(is_causal)), out.data_ptr(), workspace.data_ptr(),
                                         workspace.numel(), _stream(q)))
    _checked(workspace, check)
    return out


REORDER_MODES = {"raster": 0, "cube": 1, "morton": 2}


def token_permutation(T: int, Hg: int, Wg: int, text: int = 0, mode: str = "cube") -> torch.Tensor:
    """perm[new] = old for a [text | T x Hg x Wg video] sequence (host int32 tensor)."""
    perm = torch.empty(text + T * Hg * Wg, dtype=torch.int32)
    _check(lib().bsa_token_permutation(T, Hg, Wg, text, REORDER_MODES[mode], perm.data_ptr()))
    return perm


def permute_tokens(x: torch.Tensor, perm: torch.Tensor, inverse: bool = False, *, out=None) -> torch.Tensor:
    """Reorder the token axis of a contiguous CUDA bf16 [B, H, N, d] tensor by perm
    (a CUDA int32 permutation of 0..N-1): out[:, :, n] = x[:, :, perm[n]], or the
    inverse with inverse=True."""
    _qkv(x)
    if not (perm.is_cuda and perm.dtype == torch.int32 and perm.numel() == x.shape[2] and perm.is_contiguous()):
        raise ValueError("perm must be a contiguous CUDA int32 tensor of N entries")
    out = torch.empty_like(x) if out is None else out
    _qkv(x, out)
    _check(lib().bsa_permute_tokens(x.data_ptr(), out.data_ptr(), _shape_of(x), perm.data_ptr(),
                                    int(bool(inverse)), _stream(x)))
    return out


def sparse_attn_topk_noalloc(q, k, v, topk: float = 0.5, is_causal: bool = False, *, out=None,
                             return_mask: bool = False, check: bool = False):
    """sparse_attn_topk with the library's static device scratch in place of a
    workspace, for callers that cannot allocate device memory for one (only
    `out` and the optional mask are allocated here, unless passed in).  Calls on
    one device share the scratch: order them on one stream."""
    _qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    _qkv(q, out)
    B, H, N, _ = q.shape
    mask = torch.empty(B, H, *block_counts(N), dtype=torch.uint8, device=q.device) if return_mask else None
    _check(lib().sparse_attn_topk_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), _shape_of(q), float(topk),
                                          int(bool(is_causal)), out.data_ptr(),
                                          mask.data_ptr() if mask is not None else None, _stream(q)))
    if check:
        noalloc_status(q.device)
    return (out, mask) if return_mask else out


def noalloc_status(device="cuda") -> None:
    """Synchronise and raise BsaError if the last no-allocation call on `device`
    recorded a failure."""
    dev = torch.device(device)
    with torch.cuda.device(dev):
        _check(lib().sparse_attn_topk_noalloc_status(torch.cuda.current_stream(dev).cuda_stream))


def last_device_status(workspace: torch.Tensor) -> None:
    """Synchronise and raise BsaError if the last call on `workspace` recorded a failure."""
    _check(lib().bsa_last_device_status(workspace.data_ptr(), _stream(workspace)))


def set_wait_timeout_ns(ns: int) -> None:
    """Limit of the kernels' bounded waits in nanoseconds (0 restores the 10 s default)."""
    lib().bsa_set_wait_timeout_ns(int(ns))
