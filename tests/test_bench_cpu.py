"""The bench's roofline arithmetic, checked on the CPU: algorithmic bytes per
scan against the per-configuration byte counts of the workloads, and the ALU
bound's balanced split of the exponentials between the MUFU and FMA pipes."""
import pytest

import bench
from selective_state_space_08_b200 import synth


@pytest.mark.parametrize("name,gate,mbytes", [
    ("mamba130m_layer", True, 203.3),   # 8.08 B per element
    ("mamba2p8b_layer", True, 673.8),
    ("mamba2p8b_layer", False, 506.0),
    ("long_seq", True, 8660.0),
])
def test_scan_bytes_match_the_workload_byte_counts(name, gate, mbytes):
    c = synth.CONFIGS[name]
    got = bench.scan_bytes(c["batch"], c["dim"], c["dstate"], c["seqlen"], 2, gate)
    assert abs(got / 1e6 - mbytes) <= 0.0006 * mbytes


def test_scan_bytes_count_each_tensor_once():
    # one channel, one state, one step, fp32: u, delta, z, y, B, C, A, D, bias, h_last
    assert bench.scan_bytes(1, 1, 1, 1, 4, gate=True) == 10 * 4
    assert bench.scan_bytes(1, 1, 1, 1, 4, gate=False) == 9 * 4
    assert bench.scan_bytes(1, 1, 1, 1, 4, gate=False, h_last=False) == 8 * 4


@pytest.mark.parametrize("dstate", [1, 4, 16])
@pytest.mark.parametrize("gate", [True, False])
def test_alu_bound_balances_the_two_pipes(dstate, gate):
    n_tr = dstate + 2 + (2 if gate else 0)
    n_fma = 4 * dstate + 4
    c = bench.EXP_POLY_LANE_OPS
    mufu, fp32 = bench.MUFU_LANES_PER_SM, bench.FP32_LANES_PER_SM
    cyc = bench.alu_cycles_per_elem(dstate, gate)
    # no split beats it: every share s of exponentials on MUFU costs at least as much
    for k in range(101):
        s = k / 100
        assert cyc <= max(s * n_tr / mufu, (n_fma + (1 - s) * n_tr * c) / fp32) + 1e-12
    # and it is attained: both extremes bracket it
    assert cyc >= n_fma / fp32 and cyc >= (n_fma + n_tr * c) / (fp32 + mufu * c) - 1e-12


def test_alu_peak_of_the_bench_workload():
    assert bench.alu_cycles_per_elem(16, True) == pytest.approx(0.8906, abs=5e-5)
    assert bench.alu_peak_elems(16, True) / 1e9 == pytest.approx(326.5, abs=0.05)
