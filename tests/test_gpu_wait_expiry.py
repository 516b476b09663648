"""The library's bounded waits: a wait that runs out must end, be reported, and leave the device usable.

Every mbarrier wait in the kernels gives up after about one second of device time (or 2^22 polls) and
records the expiry in a device flag that kda_device_status reports. kda_selftest_wait_expiry launches one
single-thread kernel that waits on an mbarrier nothing ever arrives on, so its wait runs out by design: no
fault, no trap, no unbounded loop. The test checks the report, the reset, and that a prefill right after it
still matches the fp64 oracle (bf16 bound of the parity suite: rms(err) <= 2e-2 rms(ref)).
"""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_bounded_b200 import build
    build.build()
    import gated_delta_rule_bounded_b200 as m
    m.load_library()
    return m


def test_expired_wait_is_reported_and_the_context_stays_usable(kda):
    assert not kda.device_status(), "a wait expired before the test"
    t0 = time.perf_counter()
    kda.selftest_wait_expiry()
    flagged = kda.device_status()  # synchronises, reads and resets the flags
    dt = time.perf_counter() - t0
    assert flagged, "the expired wait was not reported"
    assert dt < 30.0, f"the wait took {dt:.1f} s to give up"
    assert not kda.device_status(), "the flag was not reset"

    d = W.random_scan_case(1, 130, 2, 128, 128, seed=9, dtype="bf16", z_std=2.0, init_std=0.1)
    g = {n: (x.to("cuda") if isinstance(x, torch.Tensor) else x) for n, x in d.items()}
    alpha = kda.bounded_decay(g["z"], g["A_log"], d["g_min"])
    o, sf = kda.prefill(g["q"], g["k"], g["v"], alpha, g["beta"], g["initial_state"])
    torch.cuda.synchronize()
    assert not kda.device_status()
    ref_alpha = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"])
    ro, rs = oracle.scan(d["q"], d["k"], d["v"], ref_alpha, d["beta"], d["initial_state"])
    for got, ref in ((o, ro), (sf, rs)):
        got = got.double().cpu().numpy()
        rms = float(np.sqrt(np.mean(ref ** 2)))
        assert float(np.sqrt(np.mean((got - ref) ** 2))) <= 2e-2 * rms
