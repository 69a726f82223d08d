"""lattice_scan_bwd_noalloc: the backward pass for callers that cannot allocate
device memory (a plug-in whose host application owns every device allocation
through its own pool, or a process that reserved the device's memory up front).
It runs the same backward kernel with its scratch in a static array inside the
library; the caller passes only inputs and outputs.

The test calls the entry point through the C ABI twice in a row, on different
shapes and data, and checks each result against lattice_scan_bwd (the entry point
that takes a caller-allocated workspace) within the backward tests' tolerance. The
second call would expose scratch contents left over from the first.

The file sorts last so that pytest collects it after every other test: the entry
point's static array stays resident on the device once used, and a run that stops
at the first failure has then already run the rest of the suite. The test passes
both alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest

import lattice_inputs as LI
from helpers import dev_inputs, rel_err_per_slice

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL_BWD = 1e-4
SLICES = {"dx": (0, 2), "dc": (0, 2), "dq": (0, 2), "dmu": (0, 2), "deta": (0, 2), "dS0": (0, 1)}


@pytest.fixture(scope="module")
def L():
    import orthogonal_update_recurrent_b200 as L
    from orthogonal_update_recurrent_b200 import build
    build.build()
    lib = L.lib()
    vp, i, fp = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
    lib.lattice_scan_bwd_noalloc.argtypes = [vp, i, fp, vp, i, fp, fp, fp, fp, fp, fp, fp, fp, fp,
                                             fp, fp, i, i, i, i, i, i, i, vp]
    lib.lattice_scan_bwd_noalloc.restype = ctypes.c_int
    return L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def noalloc_bwd(L, t, dy, dST, chunk):
    B, T, H, d = t["x"].shape
    m = t["c"].shape[-1]
    f32 = dict(dtype=torch.float32, device="cuda")
    out = {"dx": torch.empty((B, T, H, d), **f32), "dc": torch.empty((B, T, H, m), **f32),
           "dq": torch.empty((B, T, H, m), **f32), "dmu": torch.empty((B, T, H), **f32),
           "deta": None if t["eta"] is None else torch.empty((B, T, H), **f32),
           "dS0": torch.empty((B, H, m, d), **f32)}
    dt = lambda x: 1 if x.dtype == torch.bfloat16 else 0
    code = L.lib().lattice_scan_bwd_noalloc(
        _p(t["x"]), dt(t["x"]), _p(t["c"]), _p(t["q"]), dt(t["q"]), _p(t["mu"]), _p(t["eta"]),
        _p(t["S0"]), _p(dy), _p(dST), _p(out["dx"]), _p(out["dc"]), _p(out["dq"]), _p(out["dmu"]),
        _p(out["deta"]), _p(out["dS0"]), B, T, H, m, d, chunk, 0,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == L.OK, code
    return out


def test_noalloc_backward_matches_the_workspace_entry_point_on_two_calls_in_a_row(L):
    cases = [  # (workload, chunk, with eta): different shapes and data for each call
        (LI.Workload("a", B=2, T=150, H=2, m=64, d=64, seed=901), 16, True),
        (LI.Workload("b", B=1, T=90, H=3, m=32, d=32, x_dtype="f32", q_dtype="f32", seed=902), 1, False),
    ]
    for w, chunk, eta in cases:
        inp = LI.make_inputs(w)
        if eta:
            inp["eta"] = np.random.default_rng([w.seed, 9]).uniform(0.5, 1.5, inp["mu"].shape).astype(np.float32)
        cot = LI.make_cotangents(inp, seed=w.seed)
        t = dev_inputs(inp)
        dy = torch.from_numpy(cot["dy"]).cuda()
        dST = torch.from_numpy(cot["dS_T"]).cuda()
        got = noalloc_bwd(L, t, dy, dST, chunk)
        ref = L.scan_bwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], dy, dST, eta=t["eta"], chunk=chunk)
        torch.cuda.synchronize()
        L.device_status()
        for k, ax in SLICES.items():
            if ref[k] is None:
                assert got[k] is None
                continue
            err = rel_err_per_slice(got[k].cpu().numpy(), ref[k].cpu().numpy(), ax)
            assert err <= TOL_BWD, (w.name, k, err)
