"""ctypes binding of librdl.so (include/rdl.h), with the same function names.

Argument marshalling only: every step of the computation runs in the CUDA library.
Tensors are torch tensors on the current CUDA device (PyTorch provides device memory and
streams); `None` passes a NULL pointer.  Importing this module loads the library and raises
ImportError when it is missing -- there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librdl.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "rdl.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m diffusion_lms_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE, ERR_DEVICE_CHECK = \
    0, -1, -2, -3, -4, -5, -6
ERR_SCRATCH_LIMIT = -7
NOALLOC_SCRATCH_BYTES = 32 << 20
BF16, F32 = 0, 1
FLAG_MEAN_SUMMARY, FLAG_CHECKS, FLAG_SPLIT_SUMMARY, FLAG_WAIT_TEST = 0x1, 0x2, 0x4, 0x8
WS_SCORE, WS_ATTN, WS_SWA = 0, 1, 2
CHUNK = 64


class rdl_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("L", ctypes.c_int), ("Lq", ctypes.c_int),
                ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("D", ctypes.c_int), ("r", ctypes.c_int), ("K", ctypes.c_int),
                ("w", ctypes.c_int), ("lambda_", ctypes.c_float), ("flags", ctypes.c_int)]


class RdlError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} ({status})")
        self.status = status


_vp, _ll, _sz, _int = ctypes.c_void_p, ctypes.c_longlong, ctypes.c_size_t, ctypes.c_int
_P = ctypes.POINTER(rdl_dims)
_SIGS = {
    "rdl_summary_pool": (_int, [_vp, _ll, _ll, _vp, _vp, _P, _int, _vp, _vp, _vp, _vp]),
    "rdl_route_score_topk": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _P, _int, _vp, _vp, _vp,
                                    _sz, _vp]),
    "rdl_route_attn": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _P, _int, _vp, _vp, _vp, _sz, _vp]),
    "rdl_route_attn_noalloc": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _P, _int, _vp, _vp, _vp]),
    "rdl_swa_attn": (_int, [_vp, _vp, _vp, _vp, _P, _int, _vp, _vp, _vp, _sz, _vp]),
    "rdl_workspace_bytes": (_sz, [_int, _P, _int]),
    "rdl_last_device_status": (_int, [_vp]),
    "rdl_status_string": (ctypes.c_char_p, [_int]),
    "rdl_version": (ctypes.c_char_p, []),
    "rdl_launch_count": (ctypes.c_ulonglong, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


def declared_functions(header: str = HEADER):
    """Names of the functions include/rdl.h declares."""
    src = open(header).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(rdl_\w+)\s*\(", src, re.M)))


def exported(name: str) -> bool:
    return hasattr(_lib, name)


def status_string(s: int) -> str:
    return _lib.rdl_status_string(int(s)).decode()


def version() -> str:
    return _lib.rdl_version().decode()


def launch_count() -> int:
    return int(_lib.rdl_launch_count())


@dataclass
class Dims:
    B: int
    L: int
    Lq: int
    Hq: int
    Hkv: int
    d: int
    D: int = 0
    r: int = 0
    K: int = 1
    w: int = -1
    lam: float = 0.1
    flags: int = 0

    def c(self) -> rdl_dims:
        return rdl_dims(self.B, self.L, self.Lq, self.Hq, self.Hkv, self.d, self.D, self.r,
                        self.K, self.w, self.lam, self.flags)

    @classmethod
    def of(cls, d) -> "Dims":
        """From any object with the workload fields (e.g. workloads.Dims)."""
        return cls(d.B, d.L, d.Lq, d.Hq, d.Hkv, d.d, d.D, d.r, d.K, d.w, d.lam,
                   getattr(d, "flags", 0))


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dt(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    return {"bf16": BF16, "f32": F32}[dtype]


def _check(fn: str, status: int, raise_on_error: bool) -> int:
    if status != OK and raise_on_error:
        raise RdlError(fn, status)
    return status


def workspace_bytes(which: int, dims: Dims, dtype) -> int:
    return int(_lib.rdl_workspace_bytes(which, ctypes.byref(dims.c()), _dt(dtype)))


def rdl_summary_pool(q_mask, q_chunk_stride: int, q_batch_stride: int, k, v, dims: Dims, dtype,
                     summary, entropy, o_mask=None, stream=None, raise_on_error=True) -> int:
    s = _lib.rdl_summary_pool(_p(q_mask), q_chunk_stride, q_batch_stride, _p(k), _p(v),
                              ctypes.byref(dims.c()), _dt(dtype), _p(summary), _p(entropy),
                              _p(o_mask), _stream(stream))
    return _check("rdl_summary_pool", s, raise_on_error)


def rdl_route_score_topk(q, q_pos, x, w_down, w_up, summary, entropy, dims: Dims, dtype, idx,
                         z_sel, workspace, ws_bytes: Optional[int] = None, stream=None,
                         raise_on_error=True) -> int:
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    s = _lib.rdl_route_score_topk(_p(q), _p(q_pos), _p(x), _p(w_down), _p(w_up), _p(summary),
                                  _p(entropy), ctypes.byref(dims.c()), _dt(dtype), _p(idx),
                                  _p(z_sel), _p(workspace), ws_bytes, _stream(stream))
    return _check("rdl_route_score_topk", s, raise_on_error)


def rdl_route_attn(q, q_pos, k, v, idx, z_sel, dims: Dims, dtype, o, lse=None, workspace=None,
                   ws_bytes: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    s = _lib.rdl_route_attn(_p(q), _p(q_pos), _p(k), _p(v), _p(idx), _p(z_sel),
                            ctypes.byref(dims.c()), _dt(dtype), _p(o), _p(lse), _p(workspace),
                            ws_bytes, _stream(stream))
    return _check("rdl_route_attn", s, raise_on_error)


def rdl_route_attn_noalloc(q, q_pos, k, v, idx, z_sel, dims: Dims, dtype, o, lse=None,
                           stream=None, raise_on_error=True) -> int:
    """rdl_route_attn without a workspace argument: for hosts that cannot allocate device
    memory at call time; librdl uses its own static device scratch of
    NOALLOC_SCRATCH_BYTES per device."""
    s = _lib.rdl_route_attn_noalloc(_p(q), _p(q_pos), _p(k), _p(v), _p(idx), _p(z_sel),
                                    ctypes.byref(dims.c()), _dt(dtype), _p(o), _p(lse),
                                    _stream(stream))
    return _check("rdl_route_attn_noalloc", s, raise_on_error)


def rdl_swa_attn(q, q_pos, k, v, dims: Dims, dtype, o, lse=None, workspace=None,
                 ws_bytes: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    s = _lib.rdl_swa_attn(_p(q), _p(q_pos), _p(k), _p(v), ctypes.byref(dims.c()), _dt(dtype),
                          _p(o), _p(lse), _p(workspace), ws_bytes, _stream(stream))
    return _check("rdl_swa_attn", s, raise_on_error)


def rdl_last_device_status(stream=None) -> int:
    return int(_lib.rdl_last_device_status(_stream(stream)))
