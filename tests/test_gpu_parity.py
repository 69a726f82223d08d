"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Inputs come from lattice_inputs (seeded, shared with the oracle). The error
metric is per (b,h) slice max|gpu - ref| / max|ref|, then the max over slices.
Tolerances: 1e-4 for fp32 arithmetic on short sequences and for the exact
recurrence at every size (exact recurrence, decode step, read-out, CUDA-core
chunked form on short sequences) - the inputs are exactly representable, so
the error is the kernel's fp32 rounding; 2e-2 for the bf16-input chunked form
at full workload sizes (both kernels): the chunked recurrence carries each
slot's norm from chunk to chunk, so fp32 rounding accumulates there (a plain
fp32 evaluation drifts to about 3e-4 over 65536 tokens), and the tensor-core
kernel's matrix operands are bf16 (hi+lo pairs where they carry the state).
"""
import numpy as np
import pytest

import lattice_inputs as LI
import oracle
from helpers import dev_inputs, s_err, y_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_TC = 2e-2


@pytest.fixture(scope="module")
def L():
    import orthogonal_update_recurrent_b200 as L
    from orthogonal_update_recurrent_b200 import build
    build.build()
    return L


def run_gpu(L, inp, chunk, impl="auto", eta=None, mode="sim", lin=2, norm="token"):
    t = dev_inputs(inp)
    y, S = L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], eta=t["eta"] if eta is None else eta,
                      chunk=chunk, impl=impl, mode=mode, lin=lin, norm=norm)
    torch.cuda.synchronize()
    L.device_status()
    return y.cpu().numpy(), S.cpu().numpy()


def run_oracle(inp, chunk, mode="sim", lin=2, norm="token"):
    y, S, _ = oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], eta=inp["eta"],
                          chunk=chunk, mode=mode, lin=lin, norm=norm)
    return y, S


def small(name, **kw):
    return LI.WORKLOADS[name].with_(**kw)


# ----------------------------------------------------------- exact recurrence

def test_exact_tiny_f32_full(L):
    """The tiny fp32 workload at full size: B=1,H=1,T=256,m=16,d=32."""
    w = LI.WORKLOADS["tiny_f32"]
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, 1)
    yo, So = run_oracle(inp, 1)
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32
    np.testing.assert_allclose(np.linalg.norm(Sg, axis=-1), 1.0, atol=1e-5)


@pytest.mark.parametrize("m,d", [(16, 16), (5, 32), (64, 64), (128, 128), (64, 128), (200, 64),
                                 (256, 128)])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_exact_shapes(L, m, d, dt):
    w = LI.Workload("t", B=2, T=37, H=3, m=m, d=d, x_dtype=dt, q_dtype=dt, seed=m * 7 + d)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, 1)
    yo, So = run_oracle(inp, 1)
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


def test_exact_with_eta_and_edge_gates(L):
    """eta given; mu = 0 and mu = 1 tokens; a zero-intensity token; duplicates."""
    w = LI.Workload("t", B=2, T=41, H=2, m=32, d=64, x_dtype="f32", q_dtype="bf16",
                    dup_frac=0.2, seed=5)
    inp = LI.make_inputs(w)
    rng = np.random.default_rng(0)
    inp["eta"] = rng.uniform(0.2, 1.5, inp["mu"].shape).astype(np.float32)
    inp["mu"][:, 3] = 0.0
    inp["mu"][:, 4] = 1.0
    inp["c"][:, 5] = 0.0
    yg, Sg = run_gpu(L, inp, 1)
    yo, So = run_oracle(inp, 1)
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


def test_exact_identity_and_in_place(L):
    """mu = 1, c = 0: the state does not move; S_out == S0 updates in place."""
    w = LI.Workload("t", B=1, T=20, H=2, m=16, d=32, seed=9)
    inp = LI.make_inputs(w)
    inp["mu"][:] = 1.0
    inp["c"][:] = 0.0
    t = dev_inputs(inp)
    S = t["S0"].clone()
    y, S2 = L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], S, S_out=S)
    torch.cuda.synchronize()
    assert S2.data_ptr() == S.data_ptr()
    np.testing.assert_allclose(S.cpu().numpy(), inp["S0"], atol=2e-7)
    yref = np.einsum("bthm,bhmd->bthd", inp["q"].astype(np.float64), inp["S0"].astype(np.float64))
    assert y_err(y.cpu().numpy(), yref) <= TOL_F32


def test_empty_sequence_copies_state(L):
    w = LI.Workload("t", B=2, T=0, H=2, m=16, d=32, seed=1)
    inp = LI.make_inputs(w)
    t = dev_inputs(inp)
    y, S = L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], t["S0"])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(S.cpu().numpy(), inp["S0"])
    assert y.numel() == 0


@pytest.mark.parametrize("chunk,T1,impl", [(1, 13, "simt"), (64, 128, "simt"), (64, 128, "tcgen05"),
                                           (64, 128, "tcgen05_split"), (64, 128, "split_reg"),
                                           (64, 128, "split_reg8")])
def test_resume(L, chunk, T1, impl):
    """scan(T1) then scan(T2) from the carried state equals scan(T1 + T2):
    bitwise on CUDA cores; within the bf16 tolerance on tensor cores, which
    round the state operand afresh from the fp32 state handed over."""
    w = LI.Workload("t", B=2, T=200, H=2, m=64, d=64, seed=3)
    inp = LI.make_inputs(w)
    t = dev_inputs(inp)
    y, S = L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], chunk=chunk, impl=impl)
    sl = lambda a, s: a[:, s].contiguous()
    ya, Sa = L.scan_fwd(sl(t["x"], slice(0, T1)), sl(t["c"], slice(0, T1)), sl(t["q"], slice(0, T1)),
                        sl(t["mu"], slice(0, T1)), t["S0"], chunk=chunk, impl=impl)
    yb, Sb = L.scan_fwd(sl(t["x"], slice(T1, None)), sl(t["c"], slice(T1, None)),
                        sl(t["q"], slice(T1, None)), sl(t["mu"], slice(T1, None)), Sa, chunk=chunk,
                        impl=impl)
    torch.cuda.synchronize()
    yab = torch.cat([ya, yb], 1)
    if impl == "simt":
        assert torch.equal(yab, y)
        assert torch.equal(Sb, S)
    else:
        assert y_err(yab.cpu().numpy(), y.cpu().numpy()) <= TOL_TC
        assert s_err(Sb.cpu().numpy(), S.cpu().numpy()) <= TOL_TC


@pytest.mark.parametrize("m,chunk,impl", [(128, 1, "auto"), (128, 64, "tcgen05"), (64, 64, "tcgen05_split"),
                                          (64, 64, "split_reg"), (64, 64, "split_reg8")])
def test_deterministic(L, m, chunk, impl):
    """Repeated calls give bitwise-equal results (every reduction has a fixed order,
    the cluster read-out reduction included)."""
    w = LI.Workload("t", B=2, T=100, H=4, m=m, d=128, seed=4)
    t = dev_inputs(LI.make_inputs(w))
    y1, S1 = L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], chunk=chunk, impl=impl)
    y2, S2 = L.scan_fwd(t["x"], t["c"], t["q"], t["mu"], t["S0"], chunk=chunk, impl=impl)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(S1, S2)


# -------------------------------------------------- chunked (Eq. 17) CUDA cores

@pytest.mark.parametrize("m,d,C", [(16, 32, 4), (64, 64, 64), (128, 128, 64), (64, 128, 16),
                                   (48, 16, 8)])
def test_chunked_simt(L, m, d, C):
    w = LI.Workload("t", B=2, T=2 * C + C // 2 + 3, H=2, m=m, d=d, seed=m + d + C)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, C, impl="simt")
    yo, So = run_oracle(inp, C)
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


# ------------------------------------------- chunked (Eq. 17) tensor cores

@pytest.mark.parametrize("m,d", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [64, 2 * 64 + 37, 5 * 64])
def test_chunked_tcgen05(L, m, d, T):
    """tcgen05 kernel vs the oracle's Eq. 17 chunked form: several chunks and a
    ragged tail; bf16 x/q, fp32 state."""
    w = LI.Workload("t", B=2, T=T, H=3, m=m, d=d, seed=1000 + m + d + T)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, 64, impl="tcgen05")
    yo, So = run_oracle(inp, 64)
    assert y_err(yg, yo) <= TOL_TC
    assert s_err(Sg, So) <= TOL_TC


@pytest.mark.parametrize("m,impl", [(128, "tcgen05"), (64, "tcgen05_split"), (64, "split_reg"),
                                    (64, "split_reg8")])
def test_chunked_tcgen05_eta_and_gate_edges(L, m, impl):
    """eta given, mu = 1 and mu = 0 tokens, a token with mu = 0 and no write (a
    zero-norm update keeps every slot), zero intensities, duplicates."""
    w = LI.Workload("t", B=2, T=150, H=2, m=m, d=128, dup_frac=0.1, seed=77)
    inp = LI.make_inputs(w)
    rng = np.random.default_rng(1)
    inp["eta"] = rng.uniform(0.3, 1.5, inp["mu"].shape).astype(np.float32)
    inp["mu"][:, 10] = 1.0
    inp["mu"][:, 70] = 0.0
    inp["c"][:, 20] = 0.0
    inp["mu"][:, 100] = 0.0
    inp["c"][:, 100] = 0.0
    yg, Sg = run_gpu(L, inp, 64, impl=impl)
    yo, So = run_oracle(inp, 64)
    assert y_err(yg, yo) <= TOL_TC
    assert s_err(Sg, So) <= TOL_TC


@pytest.mark.parametrize("impl", ["split_reg", "split_reg8"])
@pytest.mark.parametrize("d", [64, 128])
def test_chunked_reg_chunk16_eta_and_gate_edges(L, d, impl):
    """Chunk 16 on the register-chain kernels with eta given (per-token inputs staged with
    each 64-token stage), mu = 1 and mu = 0 tokens, a zero-norm update, zero
    intensities, duplicates and a ragged last stage."""
    w = LI.Workload("t", B=2, T=150, H=2, m=64, d=d, dup_frac=0.1, seed=78 + d)
    inp = LI.make_inputs(w)
    rng = np.random.default_rng(2)
    inp["eta"] = rng.uniform(0.3, 1.5, inp["mu"].shape).astype(np.float32)
    inp["mu"][:, 10] = 1.0
    inp["mu"][:, 70] = 0.0
    inp["c"][:, 20] = 0.0
    inp["mu"][:, 100] = 0.0
    inp["c"][:, 100] = 0.0
    yg, Sg = run_gpu(L, inp, 16, impl=impl)
    yo, So = run_oracle(inp, 16)
    assert y_err(yg, yo) <= TOL_TC
    assert s_err(Sg, So) <= TOL_TC


# ------------------------------- chunked (Eq. 17), slots split over a cluster

@pytest.mark.parametrize("impl", ["tcgen05_split", "split_reg", "split_reg8"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 64, 2 * 64 + 37, 5 * 64])
def test_chunked_tcgen05_split(L, d, T, impl):
    """Cluster kernels (16 slots per CTA, read-out reduced across the 4 CTAs) vs the
    oracle's Eq. 17 chunked form: one token, several chunks and a ragged tail."""
    w = LI.Workload("t", B=2, T=T, H=3, m=64, d=d, seed=2000 + d + T)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, 64, impl=impl)
    yo, So = run_oracle(inp, 64)
    assert y_err(yg, yo) <= TOL_TC
    assert s_err(Sg, So) <= TOL_TC


@pytest.mark.parametrize("impl", ["split_reg", "split_reg8"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 16, 37, 64 + 16 + 5, 5 * 64 + 9])
def test_chunked_reg_chunk16(L, d, T, impl):
    """Chunk size 16 on the register-chain kernels (four chunks per 64-token read-out
    round) vs the oracle's Eq. 17 chunked form with C = 16: partial chunks and stages."""
    w = LI.Workload("t", B=2, T=T, H=3, m=64, d=d, seed=2100 + d + T)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, 16, impl=impl)
    yo, So = run_oracle(inp, 16)
    assert y_err(yg, yo) <= TOL_TC
    assert s_err(Sg, So) <= TOL_TC


@pytest.mark.parametrize("impl", ["tcgen05_split", "split_reg", "split_reg8"])
def test_chunked_split_and_wide_agree(L, impl):
    """The tensor-core kernels compute the same chunked form."""
    w = LI.Workload("t", B=3, T=700, H=2, m=64, d=128, seed=12)
    inp = LI.make_inputs(w)
    y1, S1 = run_gpu(L, inp, 64, impl="tcgen05")
    y2, S2 = run_gpu(L, inp, 64, impl=impl)
    assert y_err(y2, y1) <= 1e-2
    assert s_err(S2, S1) <= 1e-3


def test_chunked_automatic_choice(L):
    import torch as _t
    assert L.chunk_impl(4, 8, 64, 64, 64) == "split_reg"          # 32 sequences: 32 clusters of 4 CTAs
    assert L.chunk_impl(1, 16, 64, 128, 64) == "split_reg"
    assert L.chunk_impl(4, 8, 64, 64, 16) == "split_reg"          # chunk 16 on tensor cores too
    assert L.chunk_impl(8, 16, 64, 64, 64) == "tcgen05"           # 128 sequences fill the SMs
    assert L.chunk_impl(8, 16, 64, 64, 16) == "simt"
    assert L.chunk_impl(8, 16, 128, 128, 64) == "tcgen05"
    assert L.chunk_impl(1, 1, 128, 128, 64) == "tcgen05"          # the split kernel is for m = 64
    assert L.chunk_impl(4, 8, 128, 128, 32) == "simt"
    assert L.chunk_impl(4, 8, 64, 64, 64, x_dtype=_t.float32) == "simt"
    assert L.chunk_impl(4, 8, 32, 128, 64) == "simt"


# ------------------------------------------------------------- decode step

@pytest.mark.parametrize("m,d", [(128, 128), (64, 64), (16, 32), (7, 16), (200, 128)])
def test_step_matches_oracle_over_steps(L, m, d):
    w = LI.WORKLOADS["decode"].with_(m=m, d=d)
    B, H, n = 3, 5, 6
    S0 = LI.make_decode_state(w, B=B, H=H)
    st = LI.make_decode_steps(w, n, B=B, H=H)
    S = torch.from_numpy(S0.copy()).cuda()
    So = S0.astype(np.float64)
    for k in range(n):
        one = {key: st[key][k] for key in ("x", "q", "c", "mu")}
        one["x_bits"] = None if st["x_bits"] is None else st["x_bits"][k]
        one["q_bits"] = None if st["q_bits"] is None else st["q_bits"][k]
        one["eta"] = None
        t = dev_inputs(one)
        y = L.step(S, t["x"], t["c"], t["q"], t["mu"])
        yo, So, _ = oracle.step(So, one["x"], one["c"], one["q"], one["mu"])
        torch.cuda.synchronize()
        assert y_err(y.cpu().numpy()[:, None], yo[:, None]) <= TOL_F32
    assert s_err(S.cpu().numpy(), So) <= TOL_F32


def test_readout(L):
    rng = np.random.default_rng(2)
    for m, d in ((128, 128), (5, 16), (64, 32)):
        S = rng.standard_normal((3, 4, m, d)).astype(np.float32)
        q = rng.standard_normal((3, 4, m)).astype(np.float32)
        y = L.readout(torch.from_numpy(S).cuda(), torch.from_numpy(q).cuda())
        yo = oracle.readout(S, q)
        torch.cuda.synchronize()
        assert y_err(y.cpu().numpy()[:, None], yo[:, None]) <= TOL_F32


# ---------------------------------------------- full-size workloads, every head
#
# The launches the benchmark times, compared head by head with the oracle over every
# (b, h) sequence of the workload (the oracle runs each sequence on a host thread).

FULL = ["small_train", "mid_layer", "long_ctx"]
# a few sequences of each workload, for the paths that are checked on samples
FULL_PAIRS = {"small_train": [(0, 0), (3, 7), (2, 4)], "mid_layer": [(0, 0), (7, 15), (4, 9)],
              "long_ctx": [(0, 0), (0, 11)]}


def every_head(w):
    return [(b, h) for b in range(w.B) for h in range(w.H)]


def oracle_every_head(inp, w, chunk, **kw):
    """The oracle over every sequence of a full workload, as [B, T, H, d] / [B, H, m, d]."""
    pairs = every_head(w)
    yo, So = run_oracle(LI.sample_heads(inp, pairs), chunk, **kw)
    yo = yo[:, :, 0].reshape(w.B, w.H, w.T, w.d).transpose(0, 2, 1, 3)
    So = So[:, 0].reshape(w.B, w.H, w.m, w.d)
    return yo, So


@pytest.mark.parametrize("name", FULL)
def test_full_size_exact_every_head(L, name):
    """Full-size workload, exact recurrence, every sequence against the oracle."""
    w = LI.WORKLOADS[name]
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, 1)
    yo, So = oracle_every_head(inp, w, 1)
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


@pytest.mark.parametrize("name", FULL)
def test_full_size_chunked_every_head(L, name):
    """Full-size workload, chunk 64, every sequence against the oracle's Eq. 17 chunked
    form, for every kernel that runs the shape (the automatic choice included)."""
    w = LI.WORKLOADS[name]
    inp = LI.make_inputs(w)
    yo, So = oracle_every_head(inp, w, w.chunk)
    impls = ["auto", "simt", "tcgen05"] + (["tcgen05_split", "split_reg", "split_reg8"] if w.m == 64 else [])
    for impl in impls:
        yg, Sg = run_gpu(L, inp, w.chunk, impl=impl)
        assert y_err(yg, yo) <= TOL_TC, impl
        assert s_err(Sg, So) <= TOL_TC, impl
        del yg, Sg


# ------------------------------------------- reconstruction objective (DEC)
#
# Under the reconstruction objective each token writes the residual
# x - sum_i (c_i/|s_i|) s_i, which on these inputs has norm ~4 against unit slots:
# every token turns every slot by a large angle, and the slots are coupled through
# the residual. The map is chaotic. A correctly rounded fp32 evaluation leaves the
# fp64 oracle by 1e-4 within 8-12 tokens (m = d = 128), and decorrelates by a few
# hundred. Parity is therefore checked where fp32 can hold it:
#   - on short sequences;
#   - on long sequences re-synchronised to the oracle's state (rounded to fp32) every
#     few tokens or every chunk, so every kernel path runs on every token while the
#     error never compounds beyond a segment;
#   - at full size, by the invariants that hold at any length (finite values, unit
#     slots for the exact recurrence) and by the prefix before the divergence.

DEC_SHAPES = [(16, 32, "f32"), (64, 64, "bf16"), (128, 128, "bf16"), (7, 16, "f32"), (200, 128, "bf16")]


def _dec_segments(L, inp, chunk, seg):
    """Run the GPU and the oracle segment by segment from the same (fp32) state."""
    T = inp["x"].shape[1]
    S = inp["S0"].astype(np.float32)
    worst_y = worst_s = 0.0
    for t0 in range(0, T, seg):
        sub = {k: (v[:, t0:t0 + seg] if isinstance(v, np.ndarray) and v.ndim >= 3 and k != "S0" else v)
               for k, v in inp.items()}
        for k in ("x_bits", "q_bits"):
            if inp.get(k) is not None:
                sub[k] = inp[k][:, t0:t0 + seg]
        sub["S0"] = S
        yg, Sg = run_gpu(L, sub, chunk, mode="dec")
        yo, So = run_oracle(sub, chunk, mode="dec")
        worst_y = max(worst_y, y_err(yg, yo))
        worst_s = max(worst_s, s_err(Sg, So))
        S = So.astype(np.float32)
    return worst_y, worst_s


@pytest.mark.parametrize("m,d,dt", DEC_SHAPES)
def test_dec_exact_short(L, m, d, dt):
    """Exact recurrence under the reconstruction objective, a few tokens, vs the oracle
    (3 for 200 slots, whose residual is larger and diverges sooner: a correctly
    rounded fp32 evaluation is 7e-5 off after 4 tokens there)."""
    T = 4 if m <= 128 else 3
    w = LI.Workload("t", B=2, T=T, H=3, m=m, d=d, x_dtype=dt, q_dtype=dt, seed=300 + m + d)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, 1, mode="dec")
    yo, So = run_oracle(inp, 1, mode="dec")
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


@pytest.mark.parametrize("m,d,dt", DEC_SHAPES[:3])
def test_dec_exact_resynchronised(L, m, d, dt):
    """69 tokens in segments of 4, each from the oracle's state: every token's path
    (residual reduction, projection, write, normaliser, read-out) at 1e-4."""
    w = LI.Workload("t", B=2, T=69, H=2, m=m, d=d, x_dtype=dt, q_dtype=dt, seed=310 + m + d)
    wy, ws = _dec_segments(L, LI.make_inputs(w), 1, 4)
    assert wy <= TOL_F32 and ws <= TOL_F32


# The chunked form under the reconstruction objective compounds the chunk-start
# residual's gates over the chunk. With the configs' intensities c = sigmoid(N(0,1))
# its slot norms grow without bound, even in the fp64 oracle: 1e11 to 1e56 after two
# chunks of 64. With c = sigmoid(N(-4,1)) they stay O(1) (1.8-2.4 after 2048 tokens),
# so the chunked DEC cases draw their intensities from that distribution.
DEC_CHUNK_C_LOC = -4.0


@pytest.mark.parametrize("m,d,C", [(16, 32, 4), (64, 64, 64), (128, 128, 64), (48, 16, 8)])
def test_dec_chunked_resynchronised(L, m, d, C):
    """Eq. 17 under the reconstruction objective (residual from the chunk-start
    state), chunk by chunk from the oracle's state, ragged tail included."""
    w = LI.Workload("t", B=2, T=3 * C + C // 2 + 3, H=2, m=m, d=d, seed=400 + m + d + C,
                    c_loc=DEC_CHUNK_C_LOC)
    wy, ws = _dec_segments(L, LI.make_inputs(w), C, C)
    assert wy <= TOL_F32 and ws <= TOL_F32


@pytest.mark.parametrize("m,d,C", [(64, 64, 16), (48, 32, 32), (64, 64, 64)])
def test_dec_chunked_split_several_chunks_per_call(L, m, d, C):
    """The chunked reconstruction objective on the cluster kernel (few sequences, chunks
    of whole 16-token blocks, d <= 64): three chunks per call, so the chunk-start state
    is taken again inside a call, with the block's reconstructions summed over the
    cluster; resynchronised with the oracle every three chunks, eta given."""
    w = LI.Workload("t", B=2, T=7 * C + 5, H=2, m=m, d=d, seed=470 + m + d + C, c_loc=DEC_CHUNK_C_LOC)
    inp = LI.make_inputs(w)
    inp["eta"] = np.random.default_rng(7).uniform(0.5, 1.5, inp["mu"].shape).astype(np.float32)
    wy, ws = _dec_segments(L, inp, C, 3 * C)
    assert wy <= TOL_F32 and ws <= TOL_F32


def test_dec_with_eta_and_gate_edges(L):
    w = LI.Workload("t", B=2, T=40, H=2, m=32, d=64, seed=500)
    inp = LI.make_inputs(w)
    rng = np.random.default_rng(5)
    inp["eta"] = rng.uniform(0.3, 1.5, inp["mu"].shape).astype(np.float32)
    inp["mu"][:, 1] = 1.0
    inp["mu"][:, 6] = 0.0
    inp["c"][:, 2] = 0.0
    inp["mu"][:, 21] = 0.0
    inp["c"][:, 21] = 0.0
    wy, ws = _dec_segments(L, inp, 1, 4)
    assert wy <= TOL_F32 and ws <= TOL_F32
    inp["c"] *= 0.05  # the chunked form wants small intensities (see above)
    wy, ws = _dec_segments(L, inp, 8, 8)
    assert wy <= TOL_F32 and ws <= TOL_F32


@pytest.mark.parametrize("m,d", [(128, 128), (64, 64), (7, 16)])
def test_dec_step_resynchronised(L, m, d):
    """Decode steps under the reconstruction objective, each from the oracle's state."""
    w = LI.WORKLOADS["decode"].with_(m=m, d=d)
    B, H, n = 3, 5, 6
    So = LI.make_decode_state(w, B=B, H=H).astype(np.float64)
    st = LI.make_decode_steps(w, n, B=B, H=H)
    for k in range(n):
        one = {key: st[key][k] for key in ("x", "q", "c", "mu")}
        one["x_bits"] = None if st["x_bits"] is None else st["x_bits"][k]
        one["q_bits"] = None if st["q_bits"] is None else st["q_bits"][k]
        one["eta"] = None
        t = dev_inputs(one)
        S32 = So.astype(np.float32)
        S = torch.from_numpy(S32.copy()).cuda()
        y = L.step(S, t["x"], t["c"], t["q"], t["mu"], mode="dec")
        yo, So, _ = oracle.step(S32, one["x"], one["c"], one["q"], one["mu"], mode="dec")
        torch.cuda.synchronize()
        assert y_err(y.cpu().numpy()[:, None], yo[:, None]) <= TOL_F32
        assert s_err(S.cpu().numpy(), So) <= TOL_F32


def test_dec_tensor_core_choices_are_unsupported(L):
    w = LI.Workload("t", B=1, T=4, H=1, m=64, d=64, seed=1)
    inp = LI.make_inputs(w)
    for impl in ("tcgen05", "tcgen05_split", "split_reg", "split_reg8"):
        with pytest.raises(L.LatticeError):
            run_gpu(L, inp, 64, impl=impl, mode="dec")
    yg, _ = run_gpu(L, inp, 64, mode="dec")  # AUTO takes the CUDA-core kernel
    yo, _ = run_oracle(inp, 64, mode="dec")
    assert y_err(yg, yo) <= TOL_F32


@pytest.mark.parametrize("name", FULL[:2])
@pytest.mark.parametrize("chunk", [1, 64])
def test_dec_full_size(L, name, chunk):
    """Full-size workload under the reconstruction objective (the launch bench.py
    times): finite everywhere, unit slots after the exact recurrence, and the
    sampled sequences' first 4 tokens equal to the oracle's."""
    w = LI.WORKLOADS[name]
    if chunk > 1:
        w = w.with_(c_loc=DEC_CHUNK_C_LOC)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, chunk, mode="dec")
    assert np.isfinite(yg).all() and np.isfinite(Sg).all()
    if chunk == 1:
        # each step renormalises in fp32: the norm error random-walks (1.3e-5 seen after 4096)
        np.testing.assert_allclose(np.linalg.norm(Sg, axis=-1), 1.0, atol=TOL_F32)
    pairs = FULL_PAIRS[name]
    sub = LI.sample_heads(inp, pairs)
    sub = {k: (v[:, :4] if isinstance(v, np.ndarray) and v.ndim >= 3 and k != "S0" else v)
           for k, v in sub.items()}
    yo, _ = run_oracle(sub, chunk, mode="dec")
    bs = [p[0] for p in pairs]
    hs = [p[1] for p in pairs]
    assert y_err(yg[bs, :4, hs][:, :, None], yo) <= TOL_F32


# ------------------------------------- chunk linearisation 1 (recurrence_linear1)

@pytest.mark.parametrize("m,d,C", [(16, 32, 4), (64, 64, 64), (128, 128, 64), (64, 128, 16), (48, 16, 8)])
def test_lin1_chunked(L, m, d, C):
    """eq. recurrence_linear1 on the CUDA-core kernel vs the oracle: several chunks
    and a ragged tail."""
    w = LI.Workload("t", B=2, T=2 * C + C // 2 + 3, H=2, m=m, d=d, seed=600 + m + d + C)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, C, lin=1)
    yo, So = run_oracle(inp, C, lin=1)
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


def test_lin1_dec_resynchronised(L):
    w = LI.Workload("t", B=2, T=3 * 16 + 5, H=2, m=32, d=64, seed=610, c_loc=DEC_CHUNK_C_LOC)
    inp = LI.make_inputs(w)
    T = inp["x"].shape[1]
    S = inp["S0"].astype(np.float32)
    for t0 in range(0, T, 16):
        sub = {k: (v[:, t0:t0 + 16] if isinstance(v, np.ndarray) and v.ndim >= 3 and k != "S0" else v)
               for k, v in inp.items()}
        sub["S0"] = S
        yg, Sg = run_gpu(L, sub, 16, mode="dec", lin=1)
        yo, So = run_oracle(sub, 16, mode="dec", lin=1)
        assert y_err(yg, yo) <= TOL_F32 and s_err(Sg, So) <= TOL_F32
        S = So.astype(np.float32)


def test_lin1_tensor_core_choices_are_unsupported(L):
    w = LI.Workload("t", B=1, T=64, H=1, m=64, d=64, seed=1)
    inp = LI.make_inputs(w)
    for impl in ("tcgen05", "tcgen05_split", "split_reg", "split_reg8"):
        with pytest.raises(L.LatticeError):
            run_gpu(L, inp, 64, impl=impl, lin=1)


@pytest.mark.parametrize("name", FULL[:1])
def test_lin1_full_size_sampled(L, name):
    w = LI.WORKLOADS[name]
    pairs = FULL_PAIRS[name]
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, w.chunk, lin=1)
    sub = LI.sample_heads(inp, pairs)
    yo, So = run_oracle(sub, w.chunk, lin=1)
    bs = [p[0] for p in pairs]
    hs = [p[1] for p in pairs]
    assert y_err(yg[bs, :, hs][:, :, None], yo) <= TOL_TC
    assert s_err(Sg[bs, hs][:, None], So) <= TOL_TC


# --------------------------------- normalisation at chunk boundaries (ablation)

@pytest.mark.parametrize("lin", [1, 2])
@pytest.mark.parametrize("m,d,C", [(16, 32, 4), (64, 64, 16), (128, 128, 64), (48, 16, 8)])
def test_chunk_norm(L, lin, m, d, C):
    """No per-token normaliser inside a chunk, unit slots after each chunk (Appendix C
    ablation), either linearisation, vs the oracle; ragged tail included."""
    w = LI.Workload("t", B=2, T=2 * C + C // 2 + 3, H=2, m=m, d=d, seed=700 + m + d + C + lin)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, C, lin=lin, norm="chunk")
    yo, So = run_oracle(inp, C, lin=lin, norm="chunk")
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


def test_chunk_norm_chunk_one_is_exact_and_tensor_cores_refuse(L):
    w = LI.Workload("t", B=1, T=40, H=2, m=64, d=64, seed=710)
    inp = LI.make_inputs(w)
    y1, S1 = run_gpu(L, inp, 1, norm="chunk")
    ye, Se = run_oracle(inp, 1)
    assert y_err(y1, ye) <= TOL_F32 and s_err(S1, Se) <= TOL_F32
    for impl in ("tcgen05", "tcgen05_split", "split_reg", "split_reg8"):
        with pytest.raises(L.LatticeError):
            run_gpu(L, inp, 64, impl=impl, norm="chunk")


# ------------------------------------------- batches that fill the device

@pytest.mark.parametrize("m,d,C,lin,norm", [(64, 64, 1, 2, "token"), (64, 32, 16, 2, "token"),
                                            (128, 64, 1, 2, "token"), (48, 64, 8, 1, "token"),
                                            (64, 64, 16, 2, "chunk")])
def test_cuda_core_scan_batch_filling_the_device(L, m, d, C, lin, norm):
    """80 sequences (more than half the SMs): one CTA per sequence instead of a
    cluster per sequence, for the exact recurrence and the CUDA-core chunked forms."""
    w = LI.Workload("t", B=10, T=37, H=8, m=m, d=d, x_dtype="f32", q_dtype="f32",
                    seed=950 + m + d + C + lin)
    inp = LI.make_inputs(w)
    yg, Sg = run_gpu(L, inp, C, impl="simt" if C > 1 else "auto", lin=lin, norm=norm)
    yo, So = run_oracle(inp, C, lin=lin, norm=norm)
    assert y_err(yg, yo) <= TOL_F32
    assert s_err(Sg, So) <= TOL_F32


def test_decode_workload_full_size_1000_steps(L):
    """The decode workload at full size (B=256, H=32, m=d=128, fp32 state of 512 MiB),
    1000 consecutive steps in place, inputs cycling through a ring of 40 pre-drawn
    steps: every head against the oracle for the first 3 steps, then 64 sampled heads
    at every step and their final state."""
    w = LI.WORKLOADS["decode"]
    ring = 40
    S0 = LI.make_decode_state(w)
    st = LI.make_decode_steps(w, ring)
    S = torch.from_numpy(S0).cuda()
    dev = {k: dev_inputs({"x": st["x"][k], "q": st["q"][k], "c": st["c"][k], "mu": st["mu"][k],
                          "x_bits": st["x_bits"][k], "q_bits": st["q_bits"][k], "eta": None})
           for k in range(ring)}
    rng = np.random.default_rng(5)
    flat = rng.choice(w.B * w.H, size=64, replace=False)
    bs, hs = flat // w.H, flat % w.H
    So = S0.astype(np.float64)
    for k in range(1000):
        r = k % ring
        t = dev[r]
        y = L.step(S, t["x"], t["c"], t["q"], t["mu"])
        if k < 3:  # every head
            yo, So, _ = oracle.step(So, st["x"][r], st["c"][r], st["q"][r], st["mu"][r])
            torch.cuda.synchronize()
            assert y_err(y.cpu().numpy()[:, None], yo[:, None]) <= TOL_F32, k
            if k == 2:
                So = np.ascontiguousarray(So[bs, hs][:, None])  # keep the sampled heads
        else:
            sub = lambda a: np.ascontiguousarray(a[bs, hs][:, None])
            yo, So, _ = oracle.step(So, sub(st["x"][r]), sub(st["c"][r]), sub(st["q"][r]), sub(st["mu"][r]))
            yg = y[torch.from_numpy(bs).cuda(), torch.from_numpy(hs).cuda()].cpu().numpy()
            assert y_err(yg[:, None, None], yo[:, None]) <= TOL_F32, k
    L.device_status()
    Sg = S[torch.from_numpy(bs).cuda(), torch.from_numpy(hs).cuda()].cpu().numpy()[:, None]
    assert s_err(Sg, So) <= TOL_F32
    np.testing.assert_allclose(np.linalg.norm(Sg, axis=-1), 1.0, atol=1e-5)


@pytest.mark.parametrize("mode", ["sim", "dec"])
@pytest.mark.parametrize("m,d,xq_f32", [(128, 128, False), (64, 64, True), (7, 16, False), (256, 64, True)])
def test_step_persistent_many_heads_per_cta(L, m, d, xq_f32, mode):
    """4096 heads: the persistent decode kernel takes several heads per CTA, each
    head's state (and x, c, mu, eta) copied in while the CTA computes the one before.
    With eta, fp32 or bf16 x and q, two consecutive steps on the same state."""
    w = LI.WORKLOADS["decode"].with_(m=m, d=d)
    B, H, n = 64, 64, 2
    So = LI.make_decode_state(w, B=B, H=H).astype(np.float64)
    st = LI.make_decode_steps(w, n, B=B, H=H)
    rng = np.random.default_rng([m, d, 17])
    S = torch.from_numpy(So.astype(np.float32)).cuda()
    for k in range(n):
        one = {key: st[key][k] for key in ("x", "q", "c", "mu")}
        one["x_bits"] = None if xq_f32 else st["x_bits"][k]
        one["q_bits"] = None if xq_f32 else st["q_bits"][k]
        one["eta"] = rng.uniform(0.5, 1.5, size=(B, H)).astype(np.float32)
        t = dev_inputs(one)
        S32 = S.cpu().numpy()
        y = L.step(S, t["x"], t["c"], t["q"], t["mu"], eta=t["eta"], mode=mode)
        yo, So, _ = oracle.step(S32, one["x"], one["c"], one["q"], one["mu"], eta=one["eta"], mode=mode)
        torch.cuda.synchronize()
        L.device_status()
        assert y_err(y.cpu().numpy()[:, None], yo[:, None]) <= TOL_F32
        assert s_err(S.cpu().numpy(), So) <= TOL_F32


@pytest.mark.parametrize("mode", ["sim", "dec"])
@pytest.mark.parametrize("m,d", [(128, 128), (64, 64), (16, 32), (7, 16), (256, 64)])
def test_step_many_heads(L, m, d, mode):
    """320 heads, several waves of CTAs, for either objective; each step starts from
    the oracle's state rounded to fp32. At m = 256 the reconstruction objective's
    write direction becomes long and nearly parallel to some slots (|x|^2 ~ 1.5e4,
    |x_perp|^2 ~ 4), which needs |x_perp|^2 summed directly rather than by
    Pythagoras."""
    w = LI.WORKLOADS["decode"].with_(m=m, d=d)
    B, H, n = 40, 8, 3
    So = LI.make_decode_state(w, B=B, H=H).astype(np.float64)
    st = LI.make_decode_steps(w, n, B=B, H=H)
    for k in range(n):
        one = {key: st[key][k] for key in ("x", "q", "c", "mu")}
        one["x_bits"] = st["x_bits"][k]
        one["q_bits"] = st["q_bits"][k]
        one["eta"] = None
        t = dev_inputs(one)
        S32 = So.astype(np.float32)
        S = torch.from_numpy(S32.copy()).cuda()
        y = L.step(S, t["x"], t["c"], t["q"], t["mu"], mode=mode)
        yo, So, _ = oracle.step(S32, one["x"], one["c"], one["q"], one["mu"], mode=mode)
        torch.cuda.synchronize()
        L.device_status()
        assert y_err(y.cpu().numpy()[:, None], yo[:, None]) <= TOL_F32
        assert s_err(S.cpu().numpy(), So) <= TOL_F32
