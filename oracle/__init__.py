"""CPU oracle for the selective scan -- TEST INFRASTRUCTURE ONLY.

Plain sequential double-precision C (``ssm_oracle.c``) behind ctypes.  Only
the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the library's own path never does,
and this package imports nothing from the library.

Functions (all take and return numpy arrays; inputs are widened to float64
exactly, outputs are float64):

* ``scan_fwd``      -- the Mamba-1 selective scan over a whole sequence;
* ``scan_step``     -- one decode step with the state updated in place;
* ``ssd_fwd``       -- the Mamba-2 scalar-decay scan, sequential in time;
* ``conv_silu``     -- the causal depthwise convolution and SiLU in front of
  the scan;
* ``scan_fwd_conv`` -- that stage followed by the scan;
* ``scan_bwd``      -- the gradients of the scan for a given dy.

Each follows the passages cited in ``ssm_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE double throughout)."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-o", out, src,
           "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return out


def load(path: str | None = None):
    """Load (building first if missing or older than its source) the oracle library."""
    global _lib
    with _lock:
        if path is not None:
            return _bind(ctypes.CDLL(path))
        if _lib is None:
            if (not os.path.exists(_LIB_PATH)
                    or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
        return _lib


def _bind(lib):
    lib.oracle_scan_fwd.argtypes = [_i64] * 4 + [_dp] * 8 + [ctypes.c_int, _dp, _dp, _dp,
                                                             ctypes.c_int]
    lib.oracle_scan_fwd.restype = ctypes.c_int
    lib.oracle_scan_step.argtypes = [_i64] * 3 + [_dp] * 8 + [ctypes.c_int, _dp, _dp]
    lib.oracle_scan_step.restype = ctypes.c_int
    lib.oracle_ssd_fwd.argtypes = [_i64] * 5 + [_dp] * 8 + [ctypes.c_int, _dp, _dp, _dp,
                                                            ctypes.c_int]
    lib.oracle_ssd_fwd.restype = ctypes.c_int
    lib.oracle_scan_bwd.argtypes = ([_i64] * 4 + [_dp] * 8 + [ctypes.c_int] + [_dp] * 2 +
                                    [_dp] * 9)
    lib.oracle_scan_bwd.restype = ctypes.c_int
    lib.oracle_conv_silu.argtypes = [_i64] * 4 + [_dp] * 5 + [ctypes.c_int]
    lib.oracle_conv_silu.restype = ctypes.c_int
    return lib


def _f64(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {a.shape}")
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(_dp)


def default_threads() -> int:
    return os.cpu_count() or 1


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
             h0=None, nthreads=None, lib=None):
    """Selective scan.  u, delta, z: (batch, dim, L); B, C: (batch, N, L);
    A: (dim, N); D, delta_bias: (dim); h0: (batch, dim, N).
    Returns (y (batch, dim, L), h_last (batch, dim, N)) in float64."""
    u = _f64(u)
    batch, dim, L = u.shape
    N = np.asarray(A).shape[1]
    delta = _f64(delta, u.shape)
    A = _f64(A, (dim, N))
    B = _f64(B, (batch, N, L))
    C = _f64(C, (batch, N, L))
    D = _f64(D, (dim,))
    z = _f64(z, u.shape)
    delta_bias = _f64(delta_bias, (dim,))
    h0 = _f64(h0, (batch, dim, N))
    y = np.empty((batch, dim, L), dtype=np.float64)
    h_last = np.empty((batch, dim, N), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_scan_fwd(batch, dim, N, L, _p(u), _p(delta), _p(A), _p(B), _p(C), _p(D),
                             _p(z), _p(delta_bias), int(bool(delta_softplus)), _p(h0), _p(y),
                             _p(h_last), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_scan_fwd failed ({rc})")
    return y, h_last


def scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, delta_softplus=True,
             h0=None, lib=None):
    """Gradients of sum(y * dy) for the selective scan.  Shapes as in
    ``scan_fwd``; dy like y.  Returns a dict of float64 arrays: du, ddelta,
    dA, dB, dC, and (when the matching input is given) dD, dz, ddelta_bias,
    dh0."""
    u = _f64(u)
    batch, dim, L = u.shape
    N = np.asarray(A).shape[1]
    delta = _f64(delta, u.shape)
    A = _f64(A, (dim, N))
    B = _f64(B, (batch, N, L))
    C = _f64(C, (batch, N, L))
    D = _f64(D, (dim,))
    z = _f64(z, u.shape)
    delta_bias = _f64(delta_bias, (dim,))
    h0 = _f64(h0, (batch, dim, N))
    dy = _f64(dy, u.shape)
    out = {"du": np.zeros(u.shape), "ddelta": np.zeros(u.shape), "dA": np.zeros((dim, N)),
           "dB": np.zeros((batch, N, L)), "dC": np.zeros((batch, N, L))}
    if D is not None:
        out["dD"] = np.zeros(dim)
    if z is not None:
        out["dz"] = np.zeros(u.shape)
    if delta_bias is not None:
        out["ddelta_bias"] = np.zeros(dim)
    if h0 is not None:
        out["dh0"] = np.zeros((batch, dim, N))
    lib = lib or load()
    g = lambda k: _p(out.get(k))
    rc = lib.oracle_scan_bwd(batch, dim, N, L, _p(u), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(z),
                             _p(delta_bias), int(bool(delta_softplus)), _p(h0), _p(dy), g("du"),
                             g("ddelta"), g("dA"), g("dB"), g("dC"), g("dD"), g("dz"),
                             g("ddelta_bias"), g("dh0"))
    if rc != 0:
        raise RuntimeError(f"oracle_scan_bwd failed ({rc})")
    return out


def conv_silu(x, w, bias=None, x_prev=None, nthreads=None, lib=None):
    """Causal depthwise convolution over time, then SiLU (the input stage of
    the scan).  x: (batch, dim, L); w: (dim, width); bias: (dim);
    x_prev: (batch, dim, width - 1), the inputs just before step 0 in time
    order (zeros when None).  Returns u (batch, dim, L) in float64."""
    x = _f64(x)
    batch, dim, L = x.shape
    w = _f64(w)
    if w.ndim != 2 or w.shape[0] != dim or w.shape[1] < 1:
        raise ValueError(f"w must be (dim, width), got {w.shape}")
    K = w.shape[1]
    bias = _f64(bias, (dim,))
    x_prev = _f64(x_prev, (batch, dim, K - 1))
    u = np.zeros((batch, dim, L), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_conv_silu(batch, dim, L, K, _p(x), _p(w), _p(bias), _p(x_prev), _p(u),
                              int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_conv_silu failed ({rc})")
    return u


def scan_fwd_conv(x, conv_w, conv_bias, x_prev, delta, A, B, C, D=None, z=None,
                  delta_bias=None, delta_softplus=True, h0=None, nthreads=None, lib=None):
    """The scan fed by the convolution stage: u = conv_silu(x, ...), then
    scan_fwd(u, ...).  Returns (y, h_last) in float64."""
    u = conv_silu(x, conv_w, conv_bias, x_prev, nthreads=nthreads, lib=lib)
    return scan_fwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, nthreads=nthreads,
                    lib=lib)


def scan_step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
              lib=None):
    """One decode step.  state: (batch, dim, N) -- a new array is returned, the
    argument is not modified; u, delta, z: (batch, dim); B, C: (batch, N).
    Returns (y (batch, dim), new_state)."""
    st = _f64(state).copy()
    batch, dim, N = st.shape
    u = _f64(u, (batch, dim))
    delta = _f64(delta, (batch, dim))
    A = _f64(A, (dim, N))
    B = _f64(B, (batch, N))
    C = _f64(C, (batch, N))
    D = _f64(D, (dim,))
    z = _f64(z, (batch, dim))
    delta_bias = _f64(delta_bias, (dim,))
    y = np.empty((batch, dim), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_scan_step(batch, dim, N, _p(u), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(z),
                              _p(delta_bias), int(bool(delta_softplus)), _p(st), _p(y))
    if rc != 0:
        raise RuntimeError(f"oracle_scan_step failed ({rc})")
    return y, st


def ssd_fwd(x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True, h0=None,
            nthreads=None, lib=None):
    """Mamba-2 scalar-decay scan.  x, z: (batch, L, H, P); delta: (batch, L, H);
    B, C: (batch, L, N); A, D, delta_bias: (H); h0: (batch, H, P, N).
    Returns (y (batch, L, H, P), h_last (batch, H, P, N)) in float64."""
    x = _f64(x)
    batch, L, H, P = x.shape
    N = np.asarray(B).shape[2]
    delta = _f64(delta, (batch, L, H))
    A = _f64(A, (H,))
    B = _f64(B, (batch, L, N))
    C = _f64(C, (batch, L, N))
    D = _f64(D, (H,))
    z = _f64(z, x.shape)
    delta_bias = _f64(delta_bias, (H,))
    h0 = _f64(h0, (batch, H, P, N))
    y = np.empty(x.shape, dtype=np.float64)
    h_last = np.empty((batch, H, P, N), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_ssd_fwd(batch, L, H, P, N, _p(x), _p(delta), _p(A), _p(B), _p(C), _p(D),
                            _p(z), _p(delta_bias), int(bool(delta_softplus)), _p(h0), _p(y),
                            _p(h_last), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_ssd_fwd failed ({rc})")
    return y, h_last
