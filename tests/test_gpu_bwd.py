"""Parity of the CUDA backward pass (through the C ABI) with the fp64 oracle's
adjoint (oracle.scan_bwd, itself pinned by finite differences of the forward).

The loss is L = sum_t dy_t . y_t + dS_T . S_T with seeded cotangents from
lattice_inputs.make_cotangents. Every gradient (dx, dc, dq, dmu, deta, dS0) is
compared element by element with the per-(b,h)-slice relative error of the
forward tests. Tolerance: 1e-4 (fp32 arithmetic, exactly representable inputs)
on sequences of up to a few hundred tokens; the full small training shape uses
the chunked form's 2e-2 for the bf16-input chunked scan and 1e-3 for the exact
recurrence, whose adjoint accumulates fp32 rounding over 2048 tokens.
"""
import numpy as np
import pytest

import lattice_inputs as LI
import oracle
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
    return L


def with_eta(inp, seed):
    rng = np.random.default_rng([seed, 9])
    out = dict(inp)
    out["eta"] = rng.uniform(0.5, 1.5, inp["mu"].shape).astype(np.float32)
    return out


def run_gpu_bwd(L, inp, cot, chunk, seg=0):
    t = dev_inputs(inp)
    dy = torch.from_numpy(cot["dy"]).cuda()
    dST = None if cot["dS_T"] is None else torch.from_numpy(cot["dS_T"]).cuda()
    g = L.scan_bwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], dy, dST, eta=t["eta"], chunk=chunk, seg=seg)
    torch.cuda.synchronize()
    L.device_status()
    return {k: (None if v is None else v.cpu().numpy()) for k, v in g.items()}


def run_oracle_bwd(inp, cot, chunk):
    return oracle.scan_bwd(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], cot["dy"],
                           cot["dS_T"], eta=inp["eta"], chunk=chunk)


def errors(gg, go):
    out = {}
    for k, ax in SLICES.items():
        if go[k] is None:
            assert gg[k] is None
            continue
        out[k] = rel_err_per_slice(gg[k], go[k], ax)
    return out


def check(gg, go, tol):
    e = errors(gg, go)
    bad = {k: v for k, v in e.items() if not v <= tol}
    assert not bad, f"gradient errors above {tol}: {bad} (all: {e})"


@pytest.mark.parametrize("m,d", [(16, 32), (5, 32), (64, 64), (128, 128), (64, 128), (48, 16)])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_bwd_exact_shapes(L, m, d, dt):
    """Exact recurrence, three segments of 64 tokens (the last one ragged), eta given."""
    w = LI.Workload("t", B=2, T=150, H=2, m=m, d=d, x_dtype=dt, q_dtype=dt, chunk=1, seed=800 + m + d)
    inp = with_eta(LI.make_inputs(w), 800)
    cot = LI.make_cotangents(inp, seed=800 + m)
    check(run_gpu_bwd(L, inp, cot, 1), run_oracle_bwd(inp, cot, 1), TOL_BWD)


@pytest.mark.parametrize("m,d,C", [(16, 32, 4), (64, 64, 16), (64, 64, 64), (128, 128, 64),
                                   (48, 16, 8), (64, 128, 32)])
def test_bwd_chunked_shapes(L, m, d, C):
    """Eq. 17: several chunks and segments, a ragged last chunk, bf16 x/q."""
    T = max(2 * C + C // 2 + 3, 150)
    w = LI.Workload("t", B=2, T=T, H=2, m=m, d=d, seed=820 + m + d + C)
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=820 + C)
    check(run_gpu_bwd(L, inp, cot, C), run_oracle_bwd(inp, cot, C), TOL_BWD)


@pytest.mark.parametrize("m,d,C", [(64, 64, 1), (64, 64, 16), (128, 64, 1), (128, 32, 8)])
def test_bwd_batch_filling_the_device(L, m, d, C):
    """80 sequences (more than half the SMs): one CTA per sequence instead of a
    cluster, including the two-slots-per-octet layout at m = 128."""
    w = LI.Workload("t", B=10, T=40, H=8, m=m, d=d, seed=830 + m + d + C)
    inp = with_eta(LI.make_inputs(w), 830)
    cot = LI.make_cotangents(inp, seed=830 + C)
    check(run_gpu_bwd(L, inp, cot, C), run_oracle_bwd(inp, cot, C), TOL_BWD)


def test_bwd_without_eta_and_final_state_gradient(L):
    w = LI.Workload("t", B=1, T=70, H=3, m=32, d=64, seed=840)
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=840, with_dS_T=False)
    for C in (1, 16):
        gg = run_gpu_bwd(L, inp, cot, C)
        assert gg["deta"] is None
        check(gg, run_oracle_bwd(inp, cot, C), TOL_BWD)


@pytest.mark.parametrize("C", [1, 8])
def test_bwd_segment_length_does_not_change_the_result(L, C):
    """States are recomputed from checkpoints with the same arithmetic, so the
    gradients are bit-identical for any segment length (one chunk per segment, the
    default, and one segment holding the whole sequence)."""
    w = LI.Workload("t", B=2, T=100, H=2, m=16, d=32, seed=850 + C)
    inp = with_eta(LI.make_inputs(w), 850)
    cot = LI.make_cotangents(inp, seed=850)
    ref = run_gpu_bwd(L, inp, cot, C)
    for seg in (C, 8 * C, 104 if C == 8 else 100):
        g = run_gpu_bwd(L, inp, cot, C, seg=seg)
        for k in ref:
            assert (ref[k] is None) == (g[k] is None)
            if ref[k] is not None:
                assert np.array_equal(ref[k], g[k]), (seg, k)


@pytest.mark.parametrize("m,d,C", [(64, 64, 16), (128, 64, 32), (100, 128, 64)])
def test_bwd_is_deterministic(L, m, d, C):
    """Run to run bit-identity, including the sums over a cluster's CTAs (4, 8 and 7 CTAs)."""
    w = LI.Workload("t", B=2, T=90, H=2, m=m, d=d, seed=860)
    inp = with_eta(LI.make_inputs(w), 860)
    cot = LI.make_cotangents(inp, seed=860)
    a = run_gpu_bwd(L, inp, cot, C)
    b = run_gpu_bwd(L, inp, cot, C)
    for k in a:
        if a[k] is not None:
            assert np.array_equal(a[k], b[k]), k


def test_bwd_empty_sequence_passes_the_state_gradient_through(L):
    w = LI.Workload("t", B=2, T=0, H=2, m=8, d=16, seed=870)
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=870)
    for C in (1, 4):
        g = run_gpu_bwd(L, inp, cot, C)
        assert np.array_equal(g["dS0"], cot["dS_T"])


@pytest.mark.parametrize("m,d,C,T", [(5, 32, 8, 70), (40, 64, 12, 100), (128, 64, 2, 37),
                                     (16, 128, 64, 50), (100, 128, 24, 130)])
def test_bwd_chunk_parallel_edges(L, m, d, C, T):
    """The chunk-parallel kernel (chunks of 2..64, d >= 32): slot counts that leave the
    last CTA of a sequence partly empty (m = 5, 40, 100), chunk sizes that are not a
    multiple of 8 (12, 24, 2), a single ragged chunk shorter than C (T = 50 < 64),
    clusters of 1 to 8 CTAs, eta given."""
    w = LI.Workload("t", B=2, T=T, H=2, m=m, d=d, seed=900 + m + d + C)
    inp = with_eta(LI.make_inputs(w), 900 + C)
    cot = LI.make_cotangents(inp, seed=900 + T)
    check(run_gpu_bwd(L, inp, cot, C), run_oracle_bwd(inp, cot, C), TOL_BWD)


@pytest.mark.parametrize("m,d,C,T,xd,qd", [(64, 64, 64, 150, "f32", "f32"), (40, 128, 16, 90, "f32", "f32"),
                                           (16, 32, 8, 61, "f32", "f32"), (64, 64, 32, 100, "bf16", "f32"),
                                           (48, 128, 64, 70, "f32", "bf16")])
def test_bwd_chunk_parallel_input_dtypes(L, m, d, C, T, xd, qd):
    """The chunk-parallel kernel with fp32 x and/or q (16-byte vector loads of fp32 x,
    fp32 q), eta given, a ragged last chunk."""
    w = LI.Workload("t", B=2, T=T, H=2, m=m, d=d, x_dtype=xd, q_dtype=qd, seed=950 + m + d + C)
    inp = with_eta(LI.make_inputs(w), 950 + C)
    cot = LI.make_cotangents(inp, seed=950 + T)
    check(run_gpu_bwd(L, inp, cot, C), run_oracle_bwd(inp, cot, C), TOL_BWD)


def test_bwd_chunk_parallel_empty_sequence(L):
    w = LI.Workload("t", B=2, T=0, H=3, m=40, d=64, seed=910)
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=910)
    g = run_gpu_bwd(L, inp, cot, 16)
    assert np.array_equal(g["dS0"], cot["dS_T"])


def test_bwd_unaligned_x_falls_back_to_the_token_kernel(L):
    """x that does not start on a 16-byte boundary cannot take the chunk-parallel
    kernel's vector loads; the call runs the token-by-token kernel instead, on the same
    definition, and agrees with the oracle (and, within rounding, with the aligned call)."""
    w = LI.Workload("t", B=1, T=90, H=2, m=32, d=64, seed=920)
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=920)
    t = dev_inputs(inp)
    flat = torch.empty(t["x"].numel() + 1, dtype=t["x"].dtype, device="cuda")
    xs = flat[1:].view(t["x"].shape)
    xs.copy_(t["x"])
    assert xs.data_ptr() % 16 != 0
    dy = torch.from_numpy(cot["dy"]).cuda()
    dST = torch.from_numpy(cot["dS_T"]).cuda()
    gu = L.scan_bwd(xs, t["c"], t["q"], t["mu"], t["S0"], dy, dST, chunk=16)
    ga = L.scan_bwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], dy, dST, chunk=16)
    torch.cuda.synchronize()
    L.device_status()
    go = run_oracle_bwd(inp, cot, 16)
    for g in (gu, ga):
        check({k: (None if v is None else v.cpu().numpy()) for k, v in g.items()}, go, TOL_BWD)


def test_bwd_mid_layer_full_size_sampled(L):
    """The mid-size layer at full size (B=8, H=16, T=4096, m=d=128, 10% duplicate
    tokens): clusters of 8 CTAs, 64 chunks; two sampled sequences against the oracle."""
    w = LI.WORKLOADS["mid_layer"]
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=930)
    gg = run_gpu_bwd(L, inp, cot, w.chunk)
    pairs = [(0, 0), (7, 15)]
    sub = LI.sample_heads(inp, pairs)
    bs, hs = [p[0] for p in pairs], [p[1] for p in pairs]
    sub_cot = dict(dy=np.ascontiguousarray(cot["dy"][bs, :, hs][:, :, None, :]),
                   dS_T=np.ascontiguousarray(cot["dS_T"][bs, hs][:, None]))
    go = run_oracle_bwd(sub, sub_cot, w.chunk)
    gsub = {"dx": gg["dx"][bs, :, hs][:, :, None, :], "dc": gg["dc"][bs, :, hs][:, :, None, :],
            "dq": gg["dq"][bs, :, hs][:, :, None, :], "dmu": gg["dmu"][bs, :, hs][:, :, None],
            "deta": None, "dS0": gg["dS0"][bs, hs][:, None]}
    check(gsub, go, 2e-2)
    for k in ("dx", "dc", "dq", "dmu", "dS0"):
        assert np.isfinite(gg[k]).all()


def test_bwd_long_context_slice_sampled(L):
    """The long-context shape's first 8192 tokens (B=1, H=16, m=64, d=128, chunk 64,
    mu = sigmoid(N(4, 0.5))): 128 chunks on 4-CTA clusters; two sampled heads against the
    oracle (the whole 65536 tokens would need 4 GB of oracle states per head)."""
    w = LI.WORKLOADS["long_ctx"]
    inp = LI.make_inputs(w, T=8192)
    cot = LI.make_cotangents(inp, seed=940)
    gg = run_gpu_bwd(L, inp, cot, w.chunk)
    pairs = [(0, 3), (0, 12)]
    sub = LI.sample_heads(inp, pairs)
    bs, hs = [p[0] for p in pairs], [p[1] for p in pairs]
    sub_cot = dict(dy=np.ascontiguousarray(cot["dy"][bs, :, hs][:, :, None, :]),
                   dS_T=np.ascontiguousarray(cot["dS_T"][bs, hs][:, None]))
    go = run_oracle_bwd(sub, sub_cot, w.chunk)
    gsub = {"dx": gg["dx"][bs, :, hs][:, :, None, :], "dc": gg["dc"][bs, :, hs][:, :, None, :],
            "dq": gg["dq"][bs, :, hs][:, :, None, :], "dmu": gg["dmu"][bs, :, hs][:, :, None],
            "deta": None, "dS0": gg["dS0"][bs, hs][:, None]}
    check(gsub, go, 2e-2)


def test_bwd_rejects_unsupported_shapes(L):
    w = LI.Workload("t", B=1, T=8, H=1, m=130, d=32, seed=880)
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=880)
    with pytest.raises(L.LatticeError):
        run_gpu_bwd(L, inp, cot, 1)
    w = LI.Workload("t", B=1, T=8, H=1, m=16, d=32, seed=881)
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=881)
    with pytest.raises(L.LatticeError):
        run_gpu_bwd(L, inp, cot, 4, seg=6)  # segment not a multiple of the chunk


@pytest.mark.parametrize("chunk,tol", [(64, 2e-2), (1, 1e-3)])
def test_bwd_small_train_full_size_sampled(L, chunk, tol):
    """The small training shape at full size (B=4, H=8, T=2048, m=d=64, bf16 x/q)
    on the GPU; four sampled (b,h) sequences are checked against the oracle
    (sequences are independent, so the sample is exact for them)."""
    w = LI.WORKLOADS["small_train"]
    inp = LI.make_inputs(w)
    cot = LI.make_cotangents(inp, seed=890)
    gg = run_gpu_bwd(L, inp, cot, chunk)
    pairs = [(0, 0), (1, 5), (2, 3), (3, 7)]
    sub = LI.sample_heads(inp, pairs)
    bs, hs = [p[0] for p in pairs], [p[1] for p in pairs]
    sub_cot = dict(dy=np.ascontiguousarray(cot["dy"][bs, :, hs][:, :, None, :]),
                   dS_T=np.ascontiguousarray(cot["dS_T"][bs, hs][:, None]))
    go = run_oracle_bwd(sub, sub_cot, chunk)
    gsub = {"dx": gg["dx"][bs, :, hs][:, :, None, :], "dc": gg["dc"][bs, :, hs][:, :, None, :],
            "dq": gg["dq"][bs, :, hs][:, :, None, :], "dmu": gg["dmu"][bs, :, hs][:, :, None],
            "deta": None, "dS0": gg["dS0"][bs, hs][:, None]}
    check(gsub, go, tol)
    for k in ("dx", "dc", "dq", "dmu", "dS0"):
        assert np.isfinite(gg[k]).all()
