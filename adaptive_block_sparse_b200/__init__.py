"""Thin Python binding of the NABLA C ABI (``include/nabla.h``) for torch tensors.

Argument marshalling only: every step of the hot path runs in ``libnabla.so``'s CUDA
kernels.  torch is used for device memory and streams.  Functions carry the C names:

  nabla_reorder, nabla_build_mask, nabla_mask_lists, nabla_attn_fwd, nabla_attn_bwd,
  nabla_mask_workspace_bytes, nabla_fwd_workspace_bytes, nabla_bwd_workspace_bytes,
  nabla_read_device_status, nabla_status_string.

The library is loaded on first use; a call raises ``ImportError`` if it has not been
built (``python -m adaptive_block_sparse_b200.build``).  There is no fallback
implementation of any step.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnabla.so")

_lib = None

NABLA_OK = 0
NABLA_ERR_INVALID_ARG = 1
NABLA_ERR_UNSUPPORTED = 2
NABLA_ERR_WORKSPACE = 3
NABLA_ERR_CUDA = 4
NABLA_ERR_DEVICE_CHECK = 5
NABLA_BF16 = 0
NABLA_F32 = 1
NABLA_F16 = 2
NABLA_LAYOUT_REORDERED = 0
NABLA_LAYOUT_NATURAL = 1

EXPORTED = (
    "nabla_status_string", "nabla_reorder", "nabla_mask_workspace_bytes", "nabla_build_mask",
    "nabla_mask_lists", "nabla_fwd_workspace_bytes", "nabla_attn_fwd",
    "nabla_bwd_workspace_bytes", "nabla_attn_bwd", "nabla_read_device_status",
    "nabla_attn_fwd_noalloc", "nabla_attn_fwd_noalloc_status", "nabla_build_mask_sweep",
    "nabla_selftest_bounded_wait",
)


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "T", "Hg", "W", "D", "P")]


class _Window(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("t", "h", "w")]


_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i32 = ctypes.c_int32

_sigs = {
    "nabla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nabla_reorder": (ctypes.c_int, [_vp, ctypes.c_int, _vp, ctypes.c_int, _vp, _Shape, _i32, _vp]),
    "nabla_mask_workspace_bytes": (_sz, [_Shape]),
    "nabla_build_mask": (ctypes.c_int, [_vp, _vp, _vp, _vp, _Shape, ctypes.c_double, _Window,
                                        ctypes.c_double, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, _vp,
                                        _sz, _vp]),
    "nabla_mask_lists": (ctypes.c_int, [_vp, _Shape, _vp, _vp, _vp, _vp, _vp]),
    "nabla_build_mask_sweep": (ctypes.c_int, [_vp, _vp, _vp, _vp, _Shape, _vp, ctypes.c_int, _Window,
                                              ctypes.c_double, _vp, _vp, _vp, _sz, _vp]),
    "nabla_fwd_workspace_bytes": (_sz, [_Shape]),
    "nabla_attn_fwd": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _vp, _Shape, ctypes.c_float,
                                      _vp, ctypes.c_int, _vp, ctypes.c_int, _vp, _sz, _vp]),
    "nabla_bwd_workspace_bytes": (_sz, [_Shape]),
    "nabla_attn_bwd": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _vp, ctypes.c_int, _vp, _vp, _vp,
                                      _vp, _vp, _vp, _Shape, ctypes.c_float, _vp, _vp, _vp,
                                      ctypes.c_int, _vp, _sz, _vp]),
    "nabla_read_device_status": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_uint32), _vp]),
    "nabla_selftest_bounded_wait": (ctypes.c_int, [_vp, _sz, _vp]),
    "nabla_attn_fwd_noalloc": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _vp, _Shape,
                                              ctypes.c_float, _vp, ctypes.c_int, _vp, ctypes.c_int,
                                              _vp]),
    "nabla_attn_fwd_noalloc_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _vp]),
}


def load_library():
    """Load ``libnabla.so`` (once) and declare the C signatures; raises if missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libnabla.so is not built ({LIB_PATH}); run "
                              "`python -m adaptive_block_sparse_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class NablaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {nabla_status_string(status)}")


@dataclass(frozen=True)
class Shape:
    """Problem shape: [B, H, S, D] with S = T*Hg*W tokens, P x P patches (N = P*P)."""

    B: int
    H: int
    T: int
    Hg: int
    W: int
    D: int
    P: int = 8

    @property
    def S(self):
        return self.T * self.Hg * self.W

    @property
    def N(self):
        return self.P * self.P

    @property
    def nb(self):
        return self.S // self.N

    @property
    def nw(self):
        return (self.nb + 31) // 32

    def c(self) -> _Shape:
        return _Shape(self.B, self.H, self.T, self.Hg, self.W, self.D, self.P)


def dtype_code(t) -> int:
    """nabla_dtype of a tensor (bf16, f32 or f16)."""
    codes = {torch.bfloat16: NABLA_BF16, torch.float32: NABLA_F32, torch.float16: NABLA_F16}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc, where):
    if rc != NABLA_OK:
        raise NablaError(rc, where)


def nabla_status_string(status: int) -> str:
    return load_library().nabla_status_string(status).decode()


REORDER_FORWARD = 0      # natural -> reordered
REORDER_INVERSE = 1      # reordered -> natural
REORDER_KEEP = 2         # natural -> natural (dtype conversion, optional pools)


def nabla_reorder(src, dst, shape: Shape, inverse=False, pool_out=None, stream=None):
    """Natural <-> reordered token order ([B,H,S,D]); optional fp64 block means.

    Forward: bf16 ``src`` into a bf16 or fp16 ``dst``.  Inverse: same dtype both sides.
    Forward with ``dst=None`` and ``pool_out``: the block means only.  ``inverse`` may
    also be REORDER_KEEP: bf16 ``src`` into a bf16 or fp16 ``dst`` in the same order.
    """
    _check(load_library().nabla_reorder(_ptr(src), dtype_code(src), _ptr(dst),
                                        dtype_code(dst) if dst is not None else NABLA_BF16,
                                        _ptr(pool_out), shape.c(), int(inverse),
                                        _stream(stream)), "nabla_reorder")
    return dst


def nabla_mask_workspace_bytes(shape: Shape) -> int:
    return int(load_library().nabla_mask_workspace_bytes(shape.c()))


def nabla_fwd_workspace_bytes(shape: Shape) -> int:
    return int(load_library().nabla_fwd_workspace_bytes(shape.c()))


def nabla_bwd_workspace_bytes(shape: Shape) -> int:
    return int(load_library().nabla_bwd_workspace_bytes(shape.c()))


def nabla_build_mask(q, k, shape: Shape, thr: float, window=(0, 0, 0), scale=None,
                     mask_bits=None, row_idx=None, row_cnt=None, col_idx=None, col_cnt=None,
                     q_pool=None, k_pool=None, workspace=None, stream=None,
                     layout=NABLA_LAYOUT_REORDERED):
    """NABLA block mask.  Returns (mask_bits, row_idx, row_cnt, col_idx, col_cnt).
    ``layout``: token order of ``q`` and ``k`` when they are read (no pools given)."""
    dev = next(t.device for t in (q, q_pool, mask_bits, workspace) if t is not None)
    if mask_bits is None:
        mask_bits = torch.empty(shape.B, shape.H, shape.nb, shape.nw, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(nabla_mask_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(shape.D)
    _check(load_library().nabla_build_mask(_ptr(q), _ptr(k), _ptr(q_pool), _ptr(k_pool), shape.c(),
                                 float(thr), _Window(*window), float(scale), _ptr(mask_bits),
                                 _ptr(row_idx), _ptr(row_cnt), _ptr(col_idx), _ptr(col_cnt),
                                 int(layout), _ptr(workspace), workspace.numel(), _stream(stream)),
           "nabla_build_mask")
    return mask_bits, row_idx, row_cnt, col_idx, col_cnt


def nabla_build_mask_sweep(q, k, shape: Shape, thrs, window=(0, 0, 0), scale=None,
                           mask_bits=None, row_cnt=None, counts=True, q_pool=None, k_pool=None,
                           workspace=None, stream=None):
    """NABLA block masks of several thresholds from one pooled map.

    Returns (mask_bits [n_thr, B, H, nb, nw], row_cnt [n_thr, B, H, nb] or None).
    """
    thrs = [float(t) for t in thrs]
    n = len(thrs)
    dev = next(t.device for t in (q, q_pool, mask_bits, workspace) if t is not None)
    if mask_bits is None:
        mask_bits = torch.empty(n, shape.B, shape.H, shape.nb, shape.nw, dtype=torch.int32, device=dev)
    if row_cnt is None and counts:
        row_cnt = torch.empty(n, shape.B, shape.H, shape.nb, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(nabla_mask_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(shape.D)
    arr = (ctypes.c_double * max(n, 1))(*thrs)
    _check(load_library().nabla_build_mask_sweep(
        _ptr(q), _ptr(k), _ptr(q_pool), _ptr(k_pool), shape.c(), ctypes.cast(arr, ctypes.c_void_p), n,
        _Window(*window), float(scale), _ptr(mask_bits), _ptr(row_cnt), _ptr(workspace),
        workspace.numel(), _stream(stream)), "nabla_build_mask_sweep")
    return mask_bits, row_cnt


def sparsity_curve(row_cnt, shape: Shape):
    """Sparsity 1 - kept / (B*H*nb^2) of each mask of a sweep, from its row counts."""
    kept = row_cnt.to(torch.int64).reshape(row_cnt.shape[0], -1).sum(dim=1)
    total = shape.B * shape.H * shape.nb * shape.nb
    return [1.0 - int(x) / total for x in kept.cpu()]


def nabla_mask_lists(mask_bits, shape: Shape, row_idx=None, row_cnt=None, col_idx=None,
                     col_cnt=None, stream=None):
    _check(load_library().nabla_mask_lists(_ptr(mask_bits), shape.c(), _ptr(row_idx), _ptr(row_cnt),
                                 _ptr(col_idx), _ptr(col_cnt), _stream(stream)), "nabla_mask_lists")
    return row_idx, row_cnt, col_idx, col_cnt


def nabla_attn_fwd(q, k, v, mask_bits, shape: Shape, scale=None, o=None,
                   o_dtype=NABLA_BF16, lse=None, workspace=None, stream=None,
                   layout=NABLA_LAYOUT_REORDERED):
    """Block-sparse attention forward.  Returns (o, lse).  ``layout``: token order of
    q, k, v, o and lse (reordered, or the latent's natural order)."""
    if scale is None:
        scale = 1.0 / math.sqrt(shape.D)
    if o is None:
        o = torch.empty(q.shape, dtype=torch.float32 if o_dtype == NABLA_F32 else torch.bfloat16,
                        device=q.device)
    if workspace is None:
        workspace = torch.zeros(nabla_fwd_workspace_bytes(shape), dtype=torch.uint8, device=q.device)
    _check(load_library().nabla_attn_fwd(_ptr(q), _ptr(k), _ptr(v), dtype_code(v), _ptr(mask_bits),
                               shape.c(),
                               float(scale), _ptr(o), int(o_dtype), _ptr(lse), int(layout),
                               _ptr(workspace), workspace.numel(), _stream(stream)), "nabla_attn_fwd")
    return o, lse


def nabla_attn_bwd(q, k, v, o, dout, lse, row_idx, row_cnt, col_idx, col_cnt, shape: Shape,
                   scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None,
                   layout=NABLA_LAYOUT_REORDERED):
    """Block-sparse attention backward (mask constant).  Returns (dq, dk, dv), fp32.
    ``layout``: token order of every tensor argument (reordered, or natural)."""
    if scale is None:
        scale = 1.0 / math.sqrt(shape.D)
    o_dtype = NABLA_F32 if o.dtype == torch.float32 else NABLA_BF16
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dv is None else dv
    if workspace is None:
        workspace = torch.zeros(nabla_bwd_workspace_bytes(shape), dtype=torch.uint8, device=q.device)
    _check(load_library().nabla_attn_bwd(_ptr(q), _ptr(k), _ptr(v), dtype_code(v), _ptr(o), o_dtype,
                               _ptr(dout), _ptr(lse),
                               _ptr(row_idx), _ptr(row_cnt), _ptr(col_idx), _ptr(col_cnt),
                               shape.c(), float(scale), _ptr(dq), _ptr(dk), _ptr(dv), int(layout),
                               _ptr(workspace), workspace.numel(), _stream(stream)),
           "nabla_attn_bwd")
    return dq, dk, dv


def nabla_attn_fwd_noalloc(q, k, v, mask_bits, shape: Shape, o, lse=None, scale=None,
                           stream=None, layout=NABLA_LAYOUT_REORDERED):
    """Forward without a caller workspace, for callers that cannot allocate device memory.

    Same results as :func:`nabla_attn_fwd`; the workspace is a fixed 1 MiB array inside
    the library (looked up on the first call on a device, so make that call before any
    stream capture).  ``o`` (and ``lse``) must be given: this path allocates nothing.
    Calls that may overlap on the GPU share that array and must be serialised.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(shape.D)
    _check(load_library().nabla_attn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), dtype_code(v), _ptr(mask_bits), shape.c(),
        float(scale), _ptr(o), dtype_code(o), _ptr(lse), int(layout), _stream(stream)),
        "nabla_attn_fwd_noalloc")
    return o, lse


def nabla_attn_fwd_noalloc_status(stream=None) -> int:
    """Device status word of the last nabla_attn_fwd_noalloc call on the current device
    (0 = fine); waits for the stream and clears the word."""
    code = ctypes.c_uint32(0)
    rc = load_library().nabla_attn_fwd_noalloc_status(ctypes.byref(code), _stream(stream))
    if rc not in (NABLA_OK, NABLA_ERR_DEVICE_CHECK):
        raise NablaError(rc, "nabla_attn_fwd_noalloc_status")
    return int(code.value)


def nabla_read_device_status(workspace, stream=None) -> int:
    code = ctypes.c_uint32(0)
    rc = load_library().nabla_read_device_status(_ptr(workspace), ctypes.byref(code), _stream(stream))
    if rc not in (NABLA_OK, NABLA_ERR_DEVICE_CHECK):
        raise NablaError(rc, "nabla_read_device_status")
    return int(code.value)


def nabla_selftest_bounded_wait(workspace, stream=None):
    """Enqueue the failure-path self-test (a bounded wait that must give up); read the
    outcome with nabla_read_device_status (expected code: DEVICE_TIMEOUT_SELFTEST)."""
    _check(load_library().nabla_selftest_bounded_wait(_ptr(workspace), workspace.numel(), _stream(stream)),
           "nabla_selftest_bounded_wait")


DEVICE_TIMEOUT_SELFTEST = 0x10A


# ---------------------------------------------------------------------------------------
# Convenience: allocate outputs and run the whole path (mask -> forward [-> backward]).
# ---------------------------------------------------------------------------------------
def alloc_mask(shape: Shape, device, lists=True, cols=True, counts=True):
    """Mask outputs: bitmask, row lists (lists), row counts (lists or counts), column lists."""
    B, H, nb = shape.B, shape.H, shape.nb
    bits = torch.empty(B, H, nb, shape.nw, dtype=torch.int32, device=device)
    ridx = torch.empty(B, H, nb, nb, dtype=torch.int32, device=device) if lists else None
    rcnt = torch.empty(B, H, nb, dtype=torch.int32, device=device) if (lists or counts) else None
    cidx = torch.empty(B, H, nb, nb, dtype=torch.int32, device=device) if cols else None
    ccnt = torch.empty(B, H, nb, dtype=torch.int32, device=device) if cols else None
    return bits, ridx, rcnt, cidx, ccnt
