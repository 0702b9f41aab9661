"""ctypes mirror of include/ssmscan.h and the loader of libssmscan.so.

The loader fails loudly: there is no fallback of any kind when the library is
missing or cannot be loaded.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libssmscan.so")
HEADER = os.path.join(ROOT, "include", "ssmscan.h")

SSM_F32, SSM_BF16 = 0, 1
STATUS = {0: "SSM_OK", 1: "SSM_ERR_INVALID_ARG", 2: "SSM_ERR_UNSUPPORTED", 3: "SSM_ERR_ALIGNMENT",
          4: "SSM_ERR_CUDA", 5: "SSM_ERR_WORKSPACE"}

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_fp = ctypes.c_void_p  # float* passed as an address


class ScanArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("dim", _i64), ("dstate", _i64), ("seqlen", _i64),
                ("dtype", ctypes.c_int),
                ("u", _vp), ("delta", _vp), ("A", _fp), ("B", _vp), ("C", _vp), ("D", _fp),
                ("z", _vp), ("delta_bias", _fp), ("delta_softplus", ctypes.c_int),
                ("h0", _fp), ("y", _vp), ("h_last", _fp),
                ("u_stride", _i64 * 2), ("delta_stride", _i64 * 2), ("z_stride", _i64 * 2),
                ("y_stride", _i64 * 2), ("B_stride", _i64 * 2), ("C_stride", _i64 * 2),
                ("ngroups", _i64), ("B_group_stride", _i64), ("C_group_stride", _i64)]


class ConvArgs(ctypes.Structure):
    _fields_ = [("width", _i64), ("weight", _fp), ("bias", _fp), ("x_prev", _fp)]


class ScanGrads(ctypes.Structure):
    _fields_ = [(k, _fp) for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias",
                                   "dh0")]


class StepArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("dim", _i64), ("dstate", _i64), ("dtype", ctypes.c_int),
                ("u", _vp), ("delta", _vp), ("z", _vp), ("B", _vp), ("C", _vp),
                ("A", _fp), ("D", _fp), ("delta_bias", _fp), ("delta_softplus", ctypes.c_int),
                ("state", _fp), ("y", _vp)]


class SsdArgs(ctypes.Structure):
    _fields_ = [("batch", _i64), ("seqlen", _i64), ("nheads", _i64), ("headdim", _i64),
                ("dstate", _i64), ("chunk", _i64), ("dtype", ctypes.c_int),
                ("x", _vp), ("delta", _vp), ("A", _fp), ("B", _vp), ("C", _vp), ("D", _fp),
                ("delta_bias", _fp), ("delta_softplus", ctypes.c_int), ("z", _vp),
                ("h0", _fp), ("y", _vp), ("h_last", _fp)]


_lib = None


def header_functions() -> list[str]:
    """Names of the functions include/ssmscan.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\**\s+\**(ssm_[a-z0-9_]+)\s*\(",
                      text, flags=re.M)


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libssmscan.so (built in-tree by ``build.py``)."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libssmscan.so not found at {p}: build it with "
                           "`python -m selective_state_space_08_b200.build`")
    lib = ctypes.CDLL(p)
    lib.ssm_scan_fwd_workspace_size.argtypes = [ctypes.POINTER(ScanArgs)]
    lib.ssm_scan_fwd_workspace_size.restype = ctypes.c_size_t
    lib.ssm_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), _vp, ctypes.c_size_t, _vp]
    lib.ssm_scan_fwd.restype = ctypes.c_int
    lib.ssm_scan_fwd_conv.argtypes = [ctypes.POINTER(ScanArgs), ctypes.POINTER(ConvArgs), _vp,
                                      ctypes.c_size_t, _vp]
    lib.ssm_scan_fwd_conv.restype = ctypes.c_int
    lib.ssm_scan_fwd_varlen.argtypes = [ctypes.POINTER(ScanArgs), _vp, _i64, _vp, ctypes.c_size_t,
                                        _vp]
    lib.ssm_scan_fwd_varlen.restype = ctypes.c_int
    lib.ssm_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(ScanArgs)]
    lib.ssm_scan_bwd_workspace_size.restype = ctypes.c_size_t
    lib.ssm_scan_bwd.argtypes = [ctypes.POINTER(ScanArgs), _vp, ctypes.POINTER(ScanGrads), _vp,
                                 ctypes.c_size_t, _vp]
    lib.ssm_scan_bwd.restype = ctypes.c_int
    lib.ssm_scan_fwd_noalloc.argtypes = [ctypes.POINTER(ScanArgs), _vp]
    lib.ssm_scan_fwd_noalloc.restype = ctypes.c_int
    lib.ssm_scan_fwd_host_staging_size.argtypes = [ctypes.POINTER(ScanArgs), _i64]
    lib.ssm_scan_fwd_host_staging_size.restype = ctypes.c_size_t
    lib.ssm_scan_fwd_host.argtypes = [ctypes.POINTER(ScanArgs), _i64, _vp, ctypes.c_size_t, _vp]
    lib.ssm_scan_fwd_host.restype = ctypes.c_int
    lib.ssm_scan_step.argtypes = [ctypes.POINTER(StepArgs), _vp]
    lib.ssm_scan_step.restype = ctypes.c_int
    lib.ssm_scan_fwd_chunked_workspace_size.argtypes = [ctypes.POINTER(SsdArgs)]
    lib.ssm_scan_fwd_chunked_workspace_size.restype = ctypes.c_size_t
    lib.ssm_scan_fwd_chunked.argtypes = [ctypes.POINTER(SsdArgs), _vp, ctypes.c_size_t, _vp]
    lib.ssm_scan_fwd_chunked.restype = ctypes.c_int
    lib.ssm_status_string.argtypes = [ctypes.c_int]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_version.argtypes = []
    lib.ssm_version.restype = ctypes.c_int
    lib.ssm_last_error_string.argtypes = []
    lib.ssm_last_error_string.restype = ctypes.c_char_p
    if path is None:
        _lib = lib
    return lib


class SsmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def check(status: int, where: str) -> None:
    if status != 0:
        detail = ""
        if status == 4 and _lib is not None:
            detail = " -- " + _lib.ssm_last_error_string().decode(errors="replace")
        raise SsmError(status, where + detail)
