"""Host-side logic of bench.py that needs no GPU: the launch count it claims,
the clock-sample filter, the step plan and the algorithmic byte count."""
import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import torch  # noqa: E402
from calibration_free_weight_b200 import synth  # noqa: E402


def test_solver_launches_follow_the_schedules():
    # group stop, axis 1: one launch of the one-pass kernel
    assert bench.solver_launches(0, 20) == 1 and bench.solver_launches(0, 20, 16) == 1
    # axis 0: passes of 2 and 3 evaluations, then the rest
    assert bench.solver_launches(0, 20, axis=0) == 3
    assert bench.solver_launches(0, 5, axis=0) == 2 and bench.solver_launches(0, 6, axis=0) == 3
    assert bench.solver_launches(0, 2, axis=0) == 1 and bench.solver_launches(0, 1, axis=0) == 1
    # no stop: one pass
    assert bench.solver_launches(2, 20) == 1
    # tensor stop, g <= 16: chunks [0,2) [2,6) [6,10) [10,14) [14,18) [18,20) + the writing launch
    assert bench.solver_launches(1, 20, 16) == 7
    assert bench.solver_launches(1, 2, 16) == 2 and bench.solver_launches(1, 3, 16) == 3
    assert bench.solver_launches(1, 6, 16) == 3 and bench.solver_launches(1, 7, 16) == 4
    # g >= 32: chunks [0,2) [2,10) [10,20) (a last chunk shorter than 4 merged) + the writing launch
    assert bench.solver_launches(1, 20, 64) == 4 and bench.solver_launches(1, 20, 32) == 4
    assert bench.solver_launches(1, 10, 128) == 3 and bench.solver_launches(1, 11, 128) == 3
    assert bench.solver_launches(1, 14, 128) == 4 and bench.solver_launches(1, 13, 128) == 3


def test_clock_samples_outside_the_timed_region_are_dropped():
    c = bench.Clocks(0)
    c.lines = ["2026/12/02 12:30:51.900, 1000, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active",
               "2026/12/02 12:30:52.123, 1965, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Active",
               "2026/12/02 12:30:52.800, 1905, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Not Active",
               "2026/12/02 12:30:53.500, 1200, 1965, 900.0, 0x8, Active, Not Active, Not Active, Not Active"]
    c.t0 = datetime.datetime(2026, 12, 2, 12, 30, 52).timestamp()
    c.t1 = datetime.datetime(2026, 12, 2, 12, 30, 53).timestamp()
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == (1965 + 1905) / 2
    assert s["reasons"] == ["sw_power_cap"]  # the hw_slowdown sample lies after the region


def test_plan_and_bytes():
    calls = bench.plan()
    assert len(calls) == 30
    assert sum(r * c for _, r, c, *_ in calls) == 1352663040
    # b4 g64 on 4096x4096: 2 B read + 0.5 B codes + 4/64 B scale/zero per weight
    assert bench.algorithmic_bytes(4096, 4096, 4, 64) == 4096 * 4096 * 2.5625
    # consecutive calls never reuse the previous call's matrix
    assert all(a[0] != b[0] for a, b in zip(calls, calls[1:]))


def test_oracle_model_rate_extrapolates_from_its_sample():
    """The streamed workloads' CPU baseline: the oracle on the first rows of one
    layer's matrices, with each matrix's settings, extrapolated to the model."""
    import bench
    Ws = [synth.weight(32, 256, seed=1, dtype=torch.float16), synth.weight(32, 512, seed=2, dtype=torch.float16)]
    sets = [dict(nbits=4, group_size=64, stop_mode=1, zero_nbits=16),
            dict(nbits=2, group_size=32, stop_mode=0, zero_nbits=8)]
    cb = bench.oracle_model_rate(Ws, sets, 1e9, rows=16, nthreads=1)
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
    assert abs(cb["extrapolated_model_s"] - 1e9 / (cb["value"] * 1e9)) < 1e-6 * cb["extrapolated_model_s"]
    assert "first 16 rows" in cb["sample"]


def test_llama70_plan():
    """The default workload: 80 layers x 7 matrices at two settings = 1120
    calls and 136.9 G weights per step; layers split across ranks cover every
    layer exactly once."""
    calls = bench.model70_calls(range(80))
    assert len(calls) == 1120
    assert sum(r * c for _, _, r, c, _, _ in calls) == 2 * 80 * synth.LLAMA2_70B.weights_per_layer()
    assert 2 * 80 * synth.LLAMA2_70B.weights_per_layer() == 136_902_082_560
    assert {(nb, g) for *_, nb, g in calls} == {(2, 16), (4, 128)}
    for world in (1, 2, 4, 8):
        got = sorted(l for r in range(world) for l in bench.rank_layers(80, world, r))
        assert got == list(range(80))
    cfg = bench.config70(1, 80)
    assert cfg["workload"] == "llama2-70b" and cfg["calls_per_step"] == 1120
    assert cfg["weights_per_step"] == 136_902_082_560


def test_llama70_host_plan():
    GB = 1 << 30
    assert bench.host_plan70(400 * GB, 2 * GB, 1 * GB, 80) == (80, True)
    assert bench.host_plan70(170 * GB, 2 * GB, 1 * GB, 80) == (80, False)
    assert bench.host_plan70(41 * GB, 2 * GB, 1 * GB, 80) == (20, False)
    assert bench.host_plan70(0, 2 * GB, 1 * GB, 80) == (1, False)
