"""Failure detection on the GPU, in the form that faults nothing: a bounded
device-side wait that nothing completes gives up after a short limit, the kernel
returns, the host reads LATTICE_ERR_TIMEOUT from lattice_get_device_status, and
the same CUDA context then runs a scan that still matches the oracle."""
import numpy as np
import pytest

import lattice_inputs as LI
import oracle
from helpers import dev_inputs, s_err, y_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import orthogonal_update_recurrent_b200 as L
    from orthogonal_update_recurrent_b200 import build
    build.build()
    return L


def test_wait_that_runs_out_is_reported_and_the_context_stays_usable(L):
    L.device_status()  # clean start
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    L.selftest_bounded_wait(1_000_000)  # 1 ms
    t1.record()
    with pytest.raises(L.LatticeError) as ei:
        L.device_status()
    assert ei.value.code == L.ERR_TIMEOUT
    assert t0.elapsed_time(t1) >= 0.9  # the wait lasted its limit
    L.device_status()  # the status word was cleared by the read
    # the context still runs the tensor-core path correctly
    w = LI.Workload("t", B=1, T=150, H=2, m=64, d=64, seed=31)
    inp = LI.make_inputs(w)
    t = dev_inputs(inp)
    y, S = L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], chunk=64)
    L.device_status()
    yo, So, _ = oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], chunk=64)
    assert y_err(y.cpu().numpy(), yo) <= 2e-2
    assert s_err(S.cpu().numpy(), So) <= 2e-2
