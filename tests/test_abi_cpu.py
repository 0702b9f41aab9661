"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import subprocess

import pytest

from selective_state_space_08_b200 import _abi, build

NULL = None


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def test_library_exports_every_declared_function(lib):
    names = _abi.header_functions()
    assert set(names) >= {"ssm_scan_fwd", "ssm_scan_fwd_workspace_size", "ssm_scan_step",
                          "ssm_scan_fwd_chunked", "ssm_scan_fwd_chunked_workspace_size",
                          "ssm_status_string", "ssm_version", "ssm_last_error_string",
                          "ssm_scan_fwd_noalloc"}
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True,
                         text=True).stdout
    for n in names:
        assert f" T {n}" in out, n


def test_status_strings(lib):
    for code in range(6):
        assert lib.ssm_status_string(code)
    assert lib.ssm_version() >= 100


def _args(**kw):
    a = _abi.ScanArgs()
    a.batch, a.dim, a.dstate, a.seqlen = 2, 40, 16, 100
    a.dtype = _abi.SSM_BF16
    fake = 0x10000  # never dereferenced: every case below fails on the host
    for f in ("u", "delta", "A", "B", "C", "y"):
        setattr(a, f, fake)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(dstate=0), 2), (dict(dstate=17), 2), (dict(batch=-1), 1), (dict(seqlen=-3), 1),
    (dict(dtype=7), 1), (dict(u=None), 1), (dict(A=None), 1), (dict(y=None), 1),
    (dict(u=0x10001), 3), (dict(A=0x10002), 3), (dict(batch=70000), 2),
])
def test_scan_fwd_rejects_bad_arguments(lib, kw, status):
    a = _args(**kw)
    assert lib.ssm_scan_fwd(ctypes.byref(a), None, 0, None) == status


def test_scan_fwd_null_args(lib):
    assert lib.ssm_scan_fwd(None, None, 0, None) == 1
    assert lib.ssm_scan_fwd_workspace_size(None) == ctypes.c_size_t(-1).value


def test_workspace_required_for_long_sequences(lib):
    a = _args(batch=1, dim=64, seqlen=1 << 20)
    need = lib.ssm_scan_fwd_workspace_size(ctypes.byref(a))
    assert 0 < need < (1 << 30)
    assert lib.ssm_scan_fwd(ctypes.byref(a), None, 0, None) == 5
    assert lib.ssm_scan_fwd(ctypes.byref(a), 0x10000, need - 1, None) == 5
    assert lib.ssm_scan_fwd(ctypes.byref(a), 0x10008, need, None) == 3


def test_workspace_query_ignores_pointers(lib):
    a = _args(batch=1, dim=64, seqlen=1 << 20, u=None, delta=None, A=None, B=None, C=None, y=None)
    assert 0 < lib.ssm_scan_fwd_workspace_size(ctypes.byref(a)) < (1 << 30)


def test_no_workspace_when_channels_fill_the_gpu(lib):
    a = _args(batch=8, dim=1536, seqlen=2048)
    assert lib.ssm_scan_fwd_workspace_size(ctypes.byref(a)) == 0


def test_empty_problems_are_no_ops(lib):
    a = _args(batch=0)
    assert lib.ssm_scan_fwd(ctypes.byref(a), None, 0, None) == 0
    a = _args(dim=0)
    assert lib.ssm_scan_fwd(ctypes.byref(a), None, 0, None) == 0


def test_host_scan_staging_and_host_side_errors(lib):
    """ssm_scan_fwd_host: staging grows with the slice up to the whole batch;
    bad slices and strided layouts are refused; missing or short staging is
    reported before anything touches a GPU."""
    a = _args(batch=5, dim=64, seqlen=300)
    size = [lib.ssm_scan_fwd_host_staging_size(ctypes.byref(a), sb) for sb in (1, 2, 5, 9)]
    assert 0 < size[0] < size[1] < size[2] == size[3]
    bad = ctypes.c_size_t(-1).value
    assert lib.ssm_scan_fwd_host_staging_size(ctypes.byref(a), 0) == bad
    assert lib.ssm_scan_fwd_host_staging_size(None, 1) == bad
    s = _args(batch=5, dim=64, seqlen=300)
    s.u_stride[1] = 512
    assert lib.ssm_scan_fwd_host_staging_size(ctypes.byref(s), 1) == bad
    assert lib.ssm_scan_fwd_host(ctypes.byref(s), 1, 0x10000, 1 << 30, None) == 2
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), 0, 0x10000, 1 << 30, None) == 1
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), 2, None, 0, None) == 5
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), 2, 0x10000, size[1] - 1, None) == 5
    assert lib.ssm_scan_fwd_host(ctypes.byref(a), 2, 0x10010, size[1], None) == 3
    assert lib.ssm_scan_fwd_host(ctypes.byref(_args(batch=0)), 1, None, 0, None) == 0


def test_grouped_bc_arguments(lib):
    """Groups must hold whole 32-channel blocks; a negative count is invalid."""
    ok = _args(dim=64, ngroups=2)
    assert lib.ssm_scan_fwd_workspace_size(ctypes.byref(ok)) != ctypes.c_size_t(-1).value
    assert lib.ssm_scan_fwd(ctypes.byref(_args(dim=40, ngroups=2)), None, 0, None) == 2
    assert lib.ssm_scan_fwd(ctypes.byref(_args(dim=96, ngroups=2)), None, 0, None) == 2
    assert lib.ssm_scan_fwd(ctypes.byref(_args(ngroups=-1)), None, 0, None) == 1


def test_varlen_scan_host_checks(lib):
    cu = 0x10000  # never dereferenced: every case below fails on the host
    a = _args(batch=1)
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(a), None, 2, None, 0, None) == 1
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(a), cu, 0, None, 0, None) == 1
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(_args(batch=2)), cu, 2, None, 0, None) == 2
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(_args(batch=1, h0=0x10000)), cu, 2, None, 0,
                                   None) == 2
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(a), 0x10002, 2, None, 0, None) == 3


def test_backward_host_checks(lib):
    a = _args(batch=2, dim=40, seqlen=100)
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(a))
    # checkpoints (16 states x ceil(100 / 16) blocks) and per-channel-block dB / dC partials
    assert need == (2 * 40 * 16 * 7 + 2 * 2 * 2 * 16 * 100) * 4
    g = _abi.ScanGrads()
    assert lib.ssm_scan_bwd(ctypes.byref(a), 0x10000, None, None, 0, None) == 1
    assert lib.ssm_scan_bwd(ctypes.byref(a), 0x10000, ctypes.byref(g), None, 0, None) == 1
    g.dA, g.dB, g.dC = 0x10000, 0x10000, 0x10000
    assert lib.ssm_scan_bwd(ctypes.byref(a), 0x10000, ctypes.byref(g), None, 0, None) == 5
    a.y = None  # the forward output plays no part in the gradients
    assert lib.ssm_scan_bwd(ctypes.byref(a), 0x10000, ctypes.byref(g), None, 0, None) == 5
    a.u = None
    assert lib.ssm_scan_bwd(ctypes.byref(a), 0x10000, ctypes.byref(g), None, 0, None) == 1
    s = _args(batch=2, dim=40, seqlen=100)
    s.u_stride[1] = 128
    assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(s)) == ctypes.c_size_t(-1).value


def test_conv_scan_rejects_bad_stage_arguments(lib):
    a = _args()
    c = _abi.ConvArgs()
    c.width, c.weight = 4, 0x10000
    assert lib.ssm_scan_fwd_conv(ctypes.byref(a), None, None, 0, None) == 1
    for width in (0, 5):
        c.width = width
        assert lib.ssm_scan_fwd_conv(ctypes.byref(a), ctypes.byref(c), None, 0, None) == 2
    c.width, c.weight = 4, None
    assert lib.ssm_scan_fwd_conv(ctypes.byref(a), ctypes.byref(c), None, 0, None) == 1
    c.weight, c.bias = 0x10000, 0x10002
    assert lib.ssm_scan_fwd_conv(ctypes.byref(a), ctypes.byref(c), None, 0, None) == 3
    c.bias = None
    assert lib.ssm_scan_fwd_conv(ctypes.byref(_args(dim=0)), ctypes.byref(c), None, 0, None) == 0


def _ssd_args(**kw):
    a = _abi.SsdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.chunk = 2, 1000, 8, 64, 128, 256
    a.dtype = _abi.SSM_BF16
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_chunked_scan_sizes_and_limits(lib):
    """The chunked scan's workspace query accepts the implemented sizes and
    refuses the others, including sizes past the 32-bit TMA coordinates."""
    bad = ctypes.c_size_t(-1).value
    ok = lib.ssm_scan_fwd_chunked_workspace_size(ctypes.byref(_ssd_args()))
    assert 0 < ok < (1 << 30)
    assert lib.ssm_scan_fwd_chunked_workspace_size(ctypes.byref(_ssd_args(chunk=128))) > ok
    for kw in (dict(headdim=32), dict(dstate=64), dict(chunk=64), dict(dtype=_abi.SSM_F32),
               dict(batch=-1), dict(seqlen=(1 << 31)),
               dict(batch=4096, nheads=4096, seqlen=1024)):  # 4096*4096*4 chunks * 64 rows
        assert lib.ssm_scan_fwd_chunked_workspace_size(ctypes.byref(_ssd_args(**kw))) == bad, kw
    assert lib.ssm_scan_fwd_chunked(ctypes.byref(_ssd_args()), None, 0, None) == 1  # null pointers
    assert lib.ssm_scan_fwd_chunked(ctypes.byref(_ssd_args(batch=0)), None, 0, None) == 0


def test_step_rejects_bad_arguments(lib):
    s = _abi.StepArgs()
    s.batch, s.dim, s.dstate, s.dtype = 2, 3, 16, 0
    assert lib.ssm_scan_step(ctypes.byref(s), None) == 1  # null pointers
    s.dstate = 17
    assert lib.ssm_scan_step(ctypes.byref(s), None) == 2
    assert lib.ssm_scan_step(None, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    from selective_state_space_08_b200 import api
    x = torch.zeros(1, 2, 3)
    with pytest.raises(ValueError):
        api.scan_fwd(x, x, torch.zeros(2, 4), torch.zeros(1, 4, 3), torch.zeros(1, 4, 3))
