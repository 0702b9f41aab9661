"""Python binding of libssmscan over torch CUDA tensors.

Argument marshalling only: the functions check devices, dtypes and layouts,
allocate outputs (and scratch) with torch when the caller passes none, and
call the C ABI on the current torch stream.  Every step of the computation
runs in the library's CUDA kernels; nothing here computes.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi

_DT = {torch.float32: _abi.SSM_F32, torch.bfloat16: _abi.SSM_BF16}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _one_device(named):
    """The CUDA device of the given tensors, which must all be on it (the
    library reads every operand on the device it launches on)."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {dev}")
    return dev


def _stream(stream, device):
    """The stream to launch on: ``stream``, which must belong to ``device``,
    or the current torch stream of ``device``."""
    s = stream if stream is not None else torch.cuda.current_stream(device)
    if s.device != device:
        raise ValueError(f"stream is on {s.device}, the tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(name, t, dtype=None, dims=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions")
    return t


def _host(name, t, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise ValueError(f"{name} must be a CPU tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _seq_strides(name, t):
    """(batch stride, row stride) of a (batch, rows, L) tensor with unit stride along L."""
    if t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name} must be contiguous along the sequence")
    return (t.stride(0), t.stride(1))


def _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, y, h_last, host=False):
    """ScanArgs for device tensors, or (host=True) for contiguous CPU tensors,
    whose strides are left at 0 (the contiguous default)."""
    check = _host if host else _cuda
    dt = u.dtype
    if dt not in _DT:
        raise ValueError("u must be float32 or bfloat16")
    batch, dim, L = u.shape
    N = A.shape[1]
    for name, t in (("delta", delta), ("z", z), ("y", y)):
        if t is not None and (t.dtype != dt or tuple(t.shape) != (batch, dim, L)):
            raise ValueError(f"{name} must be {dt} of shape {(batch, dim, L)}")
    # B and C: (batch, N, L), or grouped (batch, groups, N, L)
    G = B.shape[1] if B.dim() == 4 else 0
    bc_shape = (batch, G, N, L) if G else (batch, N, L)
    for name, t in (("B", B), ("C", C)):
        if t.dtype != dt or tuple(t.shape) != bc_shape:
            raise ValueError(f"{name} must be {dt} of shape {bc_shape}")
    for name, t, shape in (("A", A, (dim, N)), ("D", D, (dim,)), ("delta_bias", delta_bias, (dim,)),
                           ("h0", h0, (batch, dim, N)), ("h_last", h_last, (batch, dim, N))):
        if t is not None:
            check(name, t, torch.float32)
            if tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous float32 of shape {shape}")
    a = _abi.ScanArgs()
    a.batch, a.dim, a.dstate, a.seqlen = batch, dim, N, L
    a.dtype = _DT[dt]
    a.u, a.delta, a.A, a.B, a.C = _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C)
    a.D, a.z, a.delta_bias = _ptr(D), _ptr(z), _ptr(delta_bias)
    a.delta_softplus = 1 if delta_softplus else 0
    a.h0, a.y, a.h_last = _ptr(h0), _ptr(y), _ptr(h_last)
    for field, name, t in (("u_stride", "u", u), ("delta_stride", "delta", delta), ("z_stride", "z", z),
                           ("y_stride", "y", y), ("B_stride", "B", B), ("C_stride", "C", C)):
        if t is not None and not host:
            if t.dim() == 4:  # grouped: (batch, groups, N, L)
                if t.shape[-1] > 1 and t.stride(-1) != 1:
                    raise ValueError(f"{name} must be contiguous along the sequence")
                getattr(a, field)[0] = t.stride(0)
                getattr(a, field)[1] = t.stride(2)
                setattr(a, f"{name}_group_stride", t.stride(1))
            else:
                sb, sr = _seq_strides(name, t)
                getattr(a, field)[0] = sb
                getattr(a, field)[1] = sr
    a.ngroups = G
    return a


def scan_fwd_workspace_size(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                            delta_softplus=True, h0=None) -> int:
    """Bytes of scratch ``scan_fwd`` needs for these tensors."""
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, None, None)
    n = _abi.load().ssm_scan_fwd_workspace_size(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    return int(n)


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True, h0=None,
             *, y=None, h_last=None, return_last_state=True, workspace=None, stream=None):
    """Selective scan (Mamba-1 forward) on CUDA tensors.

    u, delta, z: (batch, dim, L) float32 or bfloat16, unit stride along L;
    B, C: (batch, N, L) same dtype; A: (dim, N) float32; D, delta_bias: (dim,)
    float32; h0: (batch, dim, N) float32.  Returns (y, h_last)."""
    named = (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
             ("delta_bias", delta_bias), ("h0", h0), ("y", y), ("h_last", h_last),
             ("workspace", workspace))
    for name, t in named:
        _cuda(name, t)
    dev = _one_device(named)
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, L)")
    if y is None:
        y = torch.empty(u.shape, dtype=u.dtype, device=u.device)
    if h_last is None and return_last_state:
        h_last = torch.empty((u.shape[0], u.shape[1], A.shape[1]), dtype=torch.float32,
                             device=u.device)
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, y, h_last)
    lib = _abi.load()
    need = lib.ssm_scan_fwd_workspace_size(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(int(need), dtype=torch.uint8, device=u.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _abi.check(lib.ssm_scan_fwd(ctypes.byref(a), _ptr(workspace), ws_bytes,
                                    _stream(stream, dev)), "ssm_scan_fwd")
    return y, h_last


def scan_fwd_conv(x, conv_weight, conv_bias, x_prev, delta, A, B, C, D=None, z=None,
                  delta_bias=None, delta_softplus=True, h0=None, *, y=None, h_last=None,
                  return_last_state=True, workspace=None, stream=None):
    """The scan with the convolution stage in front, in one kernel: u =
    silu(conv_bias + causal depthwise conv(x)) feeds the scan and the skip
    term.  x: (batch, dim, L) like ``scan_fwd``'s u; conv_weight: (dim,
    width) float32, width 1..4; conv_bias: (dim,) float32 or None; x_prev:
    (batch, dim, width - 1) float32 or None (inputs before step 0).
    Returns (y, h_last)."""
    named = (("x", x), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
             ("delta_bias", delta_bias), ("h0", h0), ("y", y), ("h_last", h_last),
             ("conv_weight", conv_weight), ("conv_bias", conv_bias), ("x_prev", x_prev),
             ("workspace", workspace))
    for name, t in named:
        _cuda(name, t)
    dev = _one_device(named)
    if x.dim() != 3:
        raise ValueError("x must be (batch, dim, L)")
    batch, dim, _ = x.shape
    _cuda("conv_weight", conv_weight, torch.float32, 2)
    width = conv_weight.shape[1]
    if tuple(conv_weight.shape) != (dim, width) or not conv_weight.is_contiguous():
        raise ValueError("conv_weight must be contiguous float32 of shape (dim, width)")
    for name, t, shape in (("conv_bias", conv_bias, (dim,)),
                           ("x_prev", x_prev, (batch, dim, width - 1))):
        if t is not None:
            _cuda(name, t, torch.float32)
            if tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous float32 of shape {shape}")
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    if h_last is None and return_last_state:
        h_last = torch.empty((batch, dim, A.shape[1]), dtype=torch.float32, device=x.device)
    a = _scan_args(x, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, y, h_last)
    c = _abi.ConvArgs()
    c.width, c.weight, c.bias, c.x_prev = width, _ptr(conv_weight), _ptr(conv_bias), _ptr(x_prev)
    lib = _abi.load()
    need = lib.ssm_scan_fwd_workspace_size(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(int(need), dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _abi.check(lib.ssm_scan_fwd_conv(ctypes.byref(a), ctypes.byref(c), _ptr(workspace),
                                         ws_bytes, _stream(stream, dev)), "ssm_scan_fwd_conv")
    return y, h_last


def scan_fwd_varlen(u, delta, A, B, C, cu_seqlens, D=None, z=None, delta_bias=None,
                    delta_softplus=True, *, y=None, h_last=None, return_last_state=True,
                    workspace=None, stream=None):
    """Selective scan over a packed variable-length batch: u, delta, z are
    (1, dim, L) and B, C (1, N, L) (or grouped), holding the sequences end to
    end; cu_seqlens: int32 CUDA tensor (nseq + 1) of sequence offsets.  Each
    sequence starts from a zero state.  Returns (y, h_last (nseq, dim, N))."""
    named = (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
             ("delta_bias", delta_bias), ("y", y), ("h_last", h_last), ("cu_seqlens", cu_seqlens),
             ("workspace", workspace))
    for name, t in named:
        _cuda(name, t)
    _cuda("cu_seqlens", cu_seqlens, torch.int32, 1)
    dev = _one_device(named)
    if not cu_seqlens.is_contiguous() or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a contiguous int32 vector of nseq + 1 offsets")
    if u.dim() != 3 or u.shape[0] != 1:
        raise ValueError("u must be (1, dim, L)")
    nseq = cu_seqlens.numel() - 1
    dim, N = u.shape[1], A.shape[1]
    if y is None:
        y = torch.empty(u.shape, dtype=u.dtype, device=u.device)
    if h_last is None and return_last_state:
        h_last = torch.empty((nseq, dim, N), dtype=torch.float32, device=u.device)
    if h_last is not None and (h_last.dtype != torch.float32 or tuple(h_last.shape) != (nseq, dim, N)
                               or not h_last.is_contiguous()):
        raise ValueError(f"h_last must be contiguous float32 of shape {(nseq, dim, N)}")
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, None, y, None)
    a.h_last = _ptr(h_last)
    lib = _abi.load()
    need = lib.ssm_scan_fwd_workspace_size(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(int(need), dtype=torch.uint8, device=u.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _abi.check(lib.ssm_scan_fwd_varlen(ctypes.byref(a), _ptr(cu_seqlens), nseq,
                                           _ptr(workspace), ws_bytes, _stream(stream, dev)),
                   "ssm_scan_fwd_varlen")
    return y, h_last


def scan_bwd_workspace_size(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                            delta_softplus=True, h0=None) -> int:
    """Bytes of scratch ``scan_bwd`` needs for these tensors (state checkpoints)."""
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, None, None)
    for f in ("u_stride", "delta_stride", "z_stride", "y_stride", "B_stride", "C_stride"):
        getattr(a, f)[0] = 0
        getattr(a, f)[1] = 0
    n = _abi.load().ssm_scan_bwd_workspace_size(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    return int(n)


def scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, delta_softplus=True,
             h0=None, *, workspace=None, stream=None):
    """Gradients of the selective scan for a loss with gradient ``dy``
    (batch, dim, L) float32 with respect to y.  Inputs as for ``scan_fwd``
    (contiguous).  Returns a dict of float32 tensors: du, ddelta, dA, dB, dC,
    and dD, dz, ddelta_bias, dh0 for the inputs that are given."""
    named = (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("dy", dy), ("D", D),
             ("z", z), ("delta_bias", delta_bias), ("h0", h0))
    for name, t in named:
        _cuda(name, t)
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    _cuda("dy", dy, torch.float32)
    _cuda("workspace", workspace)
    dev = _one_device(named + (("workspace", workspace),))
    if tuple(dy.shape) != tuple(u.shape):
        raise ValueError("dy must have the shape of u")
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, None, None)
    for f in ("u_stride", "delta_stride", "z_stride", "y_stride", "B_stride", "C_stride"):
        getattr(a, f)[0] = 0
        getattr(a, f)[1] = 0
    batch, dim, L = u.shape
    N = A.shape[1]
    f32 = lambda *shape: torch.empty(shape, dtype=torch.float32, device=u.device)
    out = {"du": f32(batch, dim, L), "ddelta": f32(batch, dim, L), "dA": f32(dim, N),
           "dB": f32(batch, N, L), "dC": f32(batch, N, L)}
    if D is not None:
        out["dD"] = f32(dim)
    if z is not None:
        out["dz"] = f32(batch, dim, L)
    if delta_bias is not None:
        out["ddelta_bias"] = f32(dim)
    if h0 is not None:
        out["dh0"] = f32(batch, dim, N)
    g = _abi.ScanGrads()
    for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dh0"):
        setattr(g, k, _ptr(out.get(k)))
    lib = _abi.load()
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(int(need), dtype=torch.uint8, device=u.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _abi.check(lib.ssm_scan_bwd(ctypes.byref(a), _ptr(dy), ctypes.byref(g), _ptr(workspace),
                                    ws_bytes, _stream(stream, dev)), "ssm_scan_bwd")
    return out


def scan_fwd_noalloc(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                     h0=None, *, y, h_last=None, stream=None):
    """``scan_fwd`` for callers that cannot allocate device memory: ``y`` (and
    ``h_last`` if wanted) must be passed in, and the scratch comes from the
    library's static 4 MiB device array (see ssm_scan_fwd_noalloc in
    include/ssmscan.h: first call on a device before any stream capture;
    overlapping calls race on the shared array)."""
    named = (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
             ("delta_bias", delta_bias), ("h0", h0), ("y", y), ("h_last", h_last))
    for name, t in named:
        _cuda(name, t)
    dev = _one_device(named)
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, y, h_last)
    with torch.cuda.device(dev):
        _abi.check(_abi.load().ssm_scan_fwd_noalloc(ctypes.byref(a), _stream(stream, dev)),
                   "ssm_scan_fwd_noalloc")
    return y, h_last


def scan_fwd_host_staging_size(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                               delta_softplus=True, h0=None, *, slice_batch=1,
                               return_last_state=True) -> int:
    """Bytes of device staging ``scan_fwd_host`` needs for these CPU tensors."""
    for name, t in (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
                    ("delta_bias", delta_bias), ("h0", h0)):
        _host(name, t)
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, None, None, host=True)
    # The outputs' presence (not their address) enters the size: stand-ins.
    a.y = ctypes.c_void_p(4096)
    if return_last_state:
        a.h_last = ctypes.c_void_p(4096)
    n = _abi.load().ssm_scan_fwd_host_staging_size(ctypes.byref(a), int(slice_batch))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    return int(n)


def scan_fwd_host(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                  h0=None, *, y=None, h_last=None, return_last_state=True, slice_batch=1,
                  staging=None, stream=None, synchronize=True):
    """Selective scan on contiguous CPU tensors (page-locked ones let the
    copies overlap): the batch moves through device staging in slices of
    ``slice_batch`` sequences, copies in, scans and copies out overlapping.
    Outputs are CPU tensors (page-locked when allocated here); with
    ``synchronize=False`` they are complete only once ``stream`` (default:
    the current torch stream) has finished.  Returns (y, h_last)."""
    for name, t in (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
                    ("delta_bias", delta_bias), ("h0", h0), ("y", y), ("h_last", h_last)):
        _host(name, t)
    if u.dim() != 3:
        raise ValueError("u must be (batch, dim, L)")
    if y is None:
        y = torch.empty(u.shape, dtype=u.dtype, pin_memory=True)
    if h_last is None and return_last_state:
        h_last = torch.empty((u.shape[0], u.shape[1], A.shape[1]), dtype=torch.float32,
                             pin_memory=True)
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, y, h_last, host=True)
    lib = _abi.load()
    need = lib.ssm_scan_fwd_host_staging_size(ctypes.byref(a), int(slice_batch))
    if need == ctypes.c_size_t(-1).value:
        raise ValueError("invalid arguments")
    _cuda("staging", staging)
    dev = staging.device if staging is not None else (
        stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device()))
    if staging is None or staging.numel() * staging.element_size() < need:
        staging = torch.empty(max(int(need), 1), dtype=torch.uint8, device=dev)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        _abi.check(lib.ssm_scan_fwd_host(ctypes.byref(a), int(slice_batch), _ptr(staging),
                                         staging.numel() * staging.element_size(),
                                         _stream(s, dev)), "ssm_scan_fwd_host")
    if synchronize:
        s.synchronize()
    return y, h_last


def scan_step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
              *, y=None, stream=None):
    """One decode step; ``state`` (batch, dim, N) float32 is updated in place.
    u, delta, z: (batch, dim); B, C: (batch, N).  Returns y (batch, dim)."""
    named = (("state", state), ("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C),
             ("D", D), ("z", z), ("delta_bias", delta_bias), ("y", y))
    for name, t in named:
        _cuda(name, t)
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    dev = _one_device(named)
    if u.dtype not in _DT:
        raise ValueError("u must be float32 or bfloat16")
    batch, dim = u.shape
    N = A.shape[1]
    if state.dtype != torch.float32 or tuple(state.shape) != (batch, dim, N):
        raise ValueError("state must be float32 (batch, dim, N)")
    for name, t, shape, dtype in (("delta", delta, (batch, dim), u.dtype),
                                  ("z", z, (batch, dim), u.dtype), ("B", B, (batch, N), u.dtype),
                                  ("C", C, (batch, N), u.dtype), ("A", A, (dim, N), torch.float32),
                                  ("D", D, (dim,), torch.float32),
                                  ("delta_bias", delta_bias, (dim,), torch.float32)):
        if t is not None and (tuple(t.shape) != shape or t.dtype != dtype):
            raise ValueError(f"{name} must be {dtype} of shape {shape}")
    if y is None:
        y = torch.empty((batch, dim), dtype=u.dtype, device=u.device)
    a = _abi.StepArgs()
    a.batch, a.dim, a.dstate, a.dtype = batch, dim, N, _DT[u.dtype]
    a.u, a.delta, a.z, a.B, a.C = _ptr(u), _ptr(delta), _ptr(z), _ptr(B), _ptr(C)
    a.A, a.D, a.delta_bias = _ptr(A), _ptr(D), _ptr(delta_bias)
    a.delta_softplus = 1 if delta_softplus else 0
    a.state, a.y = _ptr(state), _ptr(y)
    with torch.cuda.device(dev):
        _abi.check(_abi.load().ssm_scan_step(ctypes.byref(a), _stream(stream, dev)),
                   "ssm_scan_step")
    return y


def ssd_workspace_size(batch, seqlen, nheads, headdim, dstate, chunk) -> int:
    a = _abi.SsdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.chunk = (batch, seqlen, nheads, headdim,
                                                                  dstate, chunk)
    a.dtype = _abi.SSM_BF16
    n = _abi.load().ssm_scan_fwd_chunked_workspace_size(ctypes.byref(a))
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("unsupported or invalid sizes")
    return int(n)


def ssd_fwd(x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True, h0=None, *,
            chunk=256, y=None, h_last=None, return_last_state=True, workspace=None, stream=None,
            check_status=False):
    """Mamba-2 scalar-decay scan, chunked (tensor cores).

    x, z: (batch, L, H, P) bfloat16; delta: (batch, L, H) bfloat16; B, C:
    (batch, L, N) bfloat16; A, D, delta_bias: (H,) float32; h0: (batch, H, P, N)
    float32.  Returns (y, h_last).  With ``check_status`` the call waits for the
    GPU and raises if a tensor-core wait inside the kernels gave up."""
    named = (("x", x), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
             ("delta_bias", delta_bias), ("h0", h0), ("y", y), ("h_last", h_last))
    for name, t in named:
        _cuda(name, t)
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    _cuda("workspace", workspace)
    dev = _one_device(named + (("workspace", workspace),))
    batch, L, H, P = x.shape
    N = B.shape[-1]
    for name, t, shape, dtype in (("x", x, (batch, L, H, P), torch.bfloat16),
                                  ("delta", delta, (batch, L, H), torch.bfloat16),
                                  ("B", B, (batch, L, N), torch.bfloat16),
                                  ("C", C, (batch, L, N), torch.bfloat16),
                                  ("z", z, (batch, L, H, P), torch.bfloat16),
                                  ("A", A, (H,), torch.float32), ("D", D, (H,), torch.float32),
                                  ("delta_bias", delta_bias, (H,), torch.float32),
                                  ("h0", h0, (batch, H, P, N), torch.float32),
                                  ("h_last", h_last, (batch, H, P, N), torch.float32)):
        if t is not None and (tuple(t.shape) != shape or t.dtype != dtype):
            raise ValueError(f"{name} must be {dtype} of shape {shape}")
    if y is None:
        y = torch.empty_like(x)
    if h_last is None and return_last_state:
        h_last = torch.empty((batch, H, P, N), dtype=torch.float32, device=x.device)
    a = _abi.SsdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.chunk = batch, L, H, P, N, chunk
    a.dtype = _abi.SSM_BF16
    a.x, a.delta, a.A, a.B, a.C, a.D = _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D)
    a.delta_bias, a.delta_softplus, a.z = _ptr(delta_bias), 1 if delta_softplus else 0, _ptr(z)
    a.h0, a.y, a.h_last = _ptr(h0), _ptr(y), _ptr(h_last)
    lib = _abi.load()
    need = lib.ssm_scan_fwd_chunked_workspace_size(ctypes.byref(a))
    if need == ctypes.c_size_t(-1).value:
        raise ValueError("unsupported or invalid arguments")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(int(need), dtype=torch.uint8, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _abi.check(lib.ssm_scan_fwd_chunked(ctypes.byref(a), _ptr(workspace), ws_bytes,
                                            _stream(stream, dev)), "ssm_scan_fwd_chunked")
    if check_status:
        torch.cuda.synchronize(x.device)
        status = int(workspace[:4].view(torch.int32).item())
        if status != 0:
            raise RuntimeError(f"ssm_scan_fwd_chunked: device status {status} "
                               "(a tensor-core wait gave up)")
    return y, h_last
