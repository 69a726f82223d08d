"""Pins of the fp64 oracle to facts fixed by the paper and by the mathematics.

Paper: "Lattice: Learning to Efficiently Compress the Memory" (arXiv 2504.05646).
Each test names the passage or property it checks. None of these tests re-types
the oracle's formula: they use printed values (Figure 1), independent
constructions (explicit d x d projection matrices, finite differences of the
loss, the d = 2 rotation angle) or invariants.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_inputs(rng, B, T, H, m, d, unit=True, mu_range=(0.3, 1.0), xs=1.0):
    x = rng.standard_normal((B, T, H, d)) * xs
    q = rng.standard_normal((B, T, H, m))
    c = rng.uniform(0.05, 1.0, (B, T, H, m))
    mu = rng.uniform(*mu_range, (B, T, H))
    S0 = rng.standard_normal((B, H, m, d))
    if unit:
        S0 /= np.linalg.norm(S0, axis=-1, keepdims=True)
    else:
        S0 *= rng.uniform(0.5, 2.0, (B, H, m, 1))
    return x, c, q, mu, S0


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = np.array([float(t) for t in v])
    return vals


# ---------------------------------------------------------------- Figure 1 ---

def test_fig1_worked_example():
    """Figure 1 (a),(b): P(s)h = (1.2,-0.6); s + alpha P(s)h = (2.2,1.4) at alpha = 1.
    The oracle's write carries intensity c/|s|, so c = |s| gives alpha = 1."""
    g = _read_golden("fig1_orthogonal_update.txt")
    s, h = g["s"], g["h"]
    n = math.sqrt(float(s @ s))
    w, n2 = oracle.osr_write(s, h, c=n * g["alpha"][0], mu=1.0, eta=1.0)
    assert n2 == pytest.approx(5.0, abs=1e-15)
    np.testing.assert_allclose(w, g["s_next"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(w - s, g["h_perp"], rtol=0, atol=1e-14)
    # the orthogonal write is not the linear-attention superposition
    assert np.abs(w - g["s_hat_linear_attention"]).max() > 0.5
    # other intensities and gates scale the same orthogonal direction
    w2, _ = oracle.osr_write(s, h, c=0.7, mu=0.3, eta=0.5)
    np.testing.assert_allclose(w2 - 0.3 * s, 0.5 * (0.7 / n) * g["h_perp"], atol=1e-14)


# ------------------------------------------------------ §3.1.1 / §3.2 facts ---

@pytest.mark.parametrize("d", [2, 7, 64])
def test_write_is_orthogonal_and_pythagorean(d):
    """§3.1.1: only the part orthogonal to the slot is written; §3.2:
    |s + Delta|^2 = |s|^2 + |Delta|^2."""
    rng = _rng(d)
    for _ in range(20):
        s = rng.standard_normal(d) * rng.uniform(0.2, 3.0)
        x = rng.standard_normal(d)
        mu, c, eta = rng.uniform(0, 1), rng.uniform(0, 2), rng.uniform(0.1, 2)
        w, _ = oracle.osr_write(s, x, c, mu, eta)
        delta = w - mu * s
        assert abs(delta @ s) <= 1e-12 * np.linalg.norm(delta) * np.linalg.norm(s) + 1e-15
        w1, _ = oracle.osr_write(s, x, c, 1.0, eta)
        assert (w1 @ w1) == pytest.approx(s @ s + (w1 - s) @ (w1 - s), rel=1e-12)


def test_write_is_negative_ogd_gradient_of_similarity_loss():
    """§3.1.1 eq. (similarity_obj_stateNorm) and eq. (OSR), OGD step of eq. (OGD):
    with mu = 1 the write equals -eta * dL/ds_i for L(S) = -<phi(S) c, x>,
    phi normalising each slot. Checked by central finite differences at |s| != 1."""
    rng = _rng(11)
    m, d = 3, 5
    S = rng.standard_normal((m, d)) * rng.uniform(0.5, 2.0, (m, 1))
    x = rng.standard_normal(d)
    c = rng.uniform(0.1, 1.0, m)
    eta = 0.37

    def loss(Sm):
        phi = Sm / np.linalg.norm(Sm, axis=1, keepdims=True)
        return -float((phi.T @ c) @ x)

    eps = 1e-6
    for i in range(m):
        grad = np.zeros(d)
        for k in range(d):
            Sp, Sn = S.copy(), S.copy()
            Sp[i, k] += eps
            Sn[i, k] -= eps
            grad[k] = (loss(Sp) - loss(Sn)) / (2 * eps)
        w, _ = oracle.osr_write(S[i], x, c[i], 1.0, eta)
        np.testing.assert_allclose(w - S[i], -eta * grad, rtol=1e-7, atol=1e-9)


def test_unit_norm_after_every_exact_step():
    """§3.2 eq. (normalized_recurrence): every slot is on the unit sphere after
    each step, also when the initial slots are not."""
    rng = _rng(3)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 12, 2, 5, 6, unit=False)
    S = S0
    for t in range(12):
        y, S, deg = oracle.step(S, x[:, t], c[:, t], q[:, t], mu[:, t])
        assert deg == 0
        np.testing.assert_allclose(np.linalg.norm(S, axis=-1), 1.0, rtol=0, atol=1e-12)


def test_identity_when_gate_one_and_no_write():
    """§3.3 eq. (dacay_recurrence) with mu = 1 and zero intensity: the state is
    unchanged and the read-out is q . S0 at every step."""
    rng = _rng(4)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 9, 3, 4, 8)
    c[:] = 0.0
    mu[:] = 1.0
    y, S, deg = oracle.scan(x, c, q, mu, S0)
    np.testing.assert_allclose(S, S0, atol=1e-15)
    y_ref = np.einsum("bthm,bhmd->bthd", q, S0)
    np.testing.assert_allclose(y, y_ref, atol=1e-13)
    # the same holds for the chunked form
    y2, S2, _ = oracle.scan(x, c, q, mu, S0, chunk=4)
    np.testing.assert_allclose(S2, S0, atol=1e-15)
    np.testing.assert_allclose(y2, y_ref, atol=1e-13)


def test_redundant_input_leaves_slot_unchanged():
    """§3.1.1 (highlight box): an input already aligned with a slot carries no
    new information for it, so with mu = 1 that slot does not move."""
    rng = _rng(5)
    m, d = 4, 6
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 1, 1, m, d)
    x[0, 0, 0] = -2.5 * S0[0, 0, 1]
    mu[:] = 1.0
    _, S, _ = oracle.scan(x, c, q, mu, S0)
    np.testing.assert_allclose(S[0, 0, 1], S0[0, 0, 1], atol=1e-15)
    assert np.abs(S[0, 0, 0] - S0[0, 0, 0]).max() > 1e-3


def test_zero_norm_update_is_kept_and_counted():
    """mu = 0 with an input parallel to the slot: the update is the zero vector,
    whose projection onto the sphere is undefined; the slot is kept."""
    rng = _rng(6)
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 1, 1, 3, 5)
    x[0, 0, 0] = 0.8 * S0[0, 0, 2]
    mu[:] = 0.0
    _, S, deg = oracle.scan(x, c, q, mu, S0)
    assert deg == 1
    np.testing.assert_allclose(S[0, 0, 2], S0[0, 0, 2], atol=0)
    _, S2, deg2 = oracle.scan(x, c, q, mu, S0, chunk=4)
    assert deg2 == 1
    np.testing.assert_allclose(S2[0, 0, 2], S0[0, 0, 2], atol=0)


def test_closed_form_rotation_in_the_plane():
    """d = 2, m = 1: a unit slot is an angle theta; the write adds eta c (x.t)
    along the tangent t and mu along s, so theta' = theta + atan2(eta c (x.t), mu)."""
    rng = _rng(7)
    T = 6
    for mu0 in (None, 0.0):
        theta = rng.uniform(-np.pi, np.pi)
        S0 = np.array([np.cos(theta), np.sin(theta)]).reshape(1, 1, 1, 2)
        x = rng.standard_normal((1, T, 1, 2))
        c = rng.uniform(0.1, 2.0, (1, T, 1, 1))
        mu = rng.uniform(0.0, 1.0, (1, T, 1)) if mu0 is None else np.full((1, T, 1), mu0)
        eta = rng.uniform(0.2, 1.5, (1, T, 1))
        _, S, _ = oracle.scan(x, c, np.ones((1, T, 1, 1)), mu, S0, eta=eta)
        th = theta
        for t in range(T):
            tang = np.array([-np.sin(th), np.cos(th)])
            th = th + math.atan2(eta[0, t, 0] * c[0, t, 0, 0] * float(x[0, t, 0] @ tang),
                                 mu[0, t, 0])
        np.testing.assert_allclose(S[0, 0, 0], [np.cos(th), np.sin(th)], atol=1e-12)


def test_brute_force_projection_matrices():
    """eq. (OSR) evaluated literally: stack the Jacobians P(s_i)/|s_i| into a
    d x d x m tensor, contract h^T with it (einsum 'd1, d1 d m -> d m'), scale
    by the intensities, add mu S (General Form), project each slot onto the unit
    sphere (§3.2) and read out with the updated state. Paper layout S is d x m."""
    rng = _rng(8)
    B, T, H, m, d = 2, 8, 2, 3, 5
    x, c, q, mu, S0 = _rand_inputs(rng, B, T, H, m, d, unit=False)
    eta = rng.uniform(0.2, 1.2, (B, T, H))
    y_o, S_o, _ = oracle.scan(x, c, q, mu, S0, eta=eta)
    for b in range(B):
        for hh in range(H):
            Sdm = S0[b, hh].T.copy()  # d x m, slots are columns
            for t in range(T):
                P = np.zeros((d, d, m))
                for i in range(m):
                    s = Sdm[:, i]
                    P[:, :, i] = (np.eye(d) - np.outer(s, s) / (s @ s)) / np.linalg.norm(s)
                h = -x[b, t, hh]
                grad = np.einsum("a,adm->dm", h, P) * c[b, t, hh][None, :]
                Snew = mu[b, t, hh] * Sdm - eta[b, t, hh] * grad
                Sdm = Snew / np.linalg.norm(Snew, axis=0, keepdims=True)
                np.testing.assert_allclose(y_o[b, t, hh], Sdm @ q[b, t, hh], atol=1e-12)
            np.testing.assert_allclose(S_o[b, hh], Sdm.T, atol=1e-12)


# ------------------------------------------------------ chunked form (Eq. 17) ---

def test_chunk_size_one_is_the_exact_recurrence():
    """Appendix C / Appendix D: chunk size 1 is the exact recurrence. With the
    mu^2 reading of the chunk normaliser the two forms agree to rounding for
    unit-norm initial slots (every state the exact recurrence produces)."""
    rng = _rng(9)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 17, 3, 6, 7, unit=True)
    eta = rng.uniform(0.2, 1.2, mu.shape)
    y1, S1, _ = oracle.scan(x, c, q, mu, S0, eta=eta, chunk=1)
    y2, S2, _ = oracle.scan(x, c, q, mu, S0, eta=eta, chunk=1, form="matrix")
    # chunk=1 via the chunked code path (token form) too
    y3, S3, _ = oracle.scan(x, c, q, mu, S0, eta=eta, chunk=1, form="token")
    from oracle import _load, _f64, _p
    lib = _load()
    y4 = np.zeros_like(y1)
    S4 = np.zeros_like(S1)
    B, T, H, d = x.shape
    m = c.shape[-1]
    lib.oracle_chunked_scan(B, T, H, m, d, 1, _p(_f64(x)), _p(_f64(c)), _p(_f64(q)),
                            _p(_f64(mu)), _p(_f64(eta)), _p(_f64(S0)), _p(S4), _p(y4), 1)
    for y, S in ((y2, S2), (y3, S3), (y4, S4)):
        np.testing.assert_allclose(y, y1, atol=1e-12)
        np.testing.assert_allclose(S, S1, atol=1e-12)


def test_chunk_normaliser_keeps_the_chunk_start_norm():
    """Appendix D listing (compress_chunk): the normaliser carries the
    chunk-start norm, so the first token of a chunk - where Eq. 17 is exact -
    leaves each slot with its chunk-start norm, unit or not; the exact
    recurrence (§3.2) projects onto the unit sphere instead."""
    rng = _rng(10)
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 1, 2, 5, 6, unit=False)
    _, Sc, _ = oracle.scan(x, c, q, mu, S0, chunk=4)
    np.testing.assert_allclose(np.linalg.norm(Sc, axis=-1), np.linalg.norm(S0, axis=-1), rtol=1e-12)
    _, Se, _ = oracle.scan(x, c, q, mu, S0, chunk=1)
    np.testing.assert_allclose(np.linalg.norm(Se, axis=-1), 1.0, rtol=1e-12)
    # direction after the first token is the same in both forms
    np.testing.assert_allclose(Sc / np.linalg.norm(Sc, axis=-1, keepdims=True), Se, atol=1e-12)


def test_chunked_form_stays_bounded_on_the_training_shape():
    """The chunk-normaliser reading keeps the chunked recurrence stable over a
    whole small-training-shape sequence (2048 tokens, 32 chunks of 64): slot
    norms stay O(1). The unit-sphere reading (1/sqrt(mu^2 n^2 + |Delta|^2))
    overflows within a few chunks on the same inputs."""
    import lattice_inputs as LI
    inp = LI.make_inputs(LI.WORKLOADS["small_train"].with_(B=1, H=2))
    y, S, deg = oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], chunk=64)
    assert np.isfinite(y).all() and deg == 0
    n = np.linalg.norm(S, axis=-1)
    assert 0.1 < n.min() and n.max() < 10.0


@pytest.mark.parametrize("C", [2, 4, 16, 64])
def test_chunk_closed_form_equals_token_form(C):
    """§3.4.1 / Appendix B.1: the chunk-level matrix form (cumulative gates,
    causal score matrix, chunk-end state) equals the token-wise linear
    recurrence of Eq. 17. Ragged final chunk included."""
    rng = _rng(100 + C)
    T = 2 * C + C // 2 + 1
    x, c, q, mu, S0 = _rand_inputs(rng, 1, T, 2, 5, 4, unit=False, mu_range=(0.6, 1.0))
    y1, S1, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="token")
    y2, S2, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="matrix")
    np.testing.assert_allclose(y2, y1, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-10)


def test_chunk_first_token_matches_exact_step_and_later_tokens_differ():
    """Eq. 17 is exact for the first token of each chunk (the chunk-start state
    is the current state) and an approximation afterwards."""
    rng = _rng(12)
    C = 8
    x, c, q, mu, S0 = _rand_inputs(rng, 1, C, 1, 4, 6)
    ye, Se, _ = oracle.scan(x, c, q, mu, S0, chunk=1)
    yc, Sc, _ = oracle.scan(x, c, q, mu, S0, chunk=C)
    np.testing.assert_allclose(yc[:, 0], ye[:, 0], atol=1e-13)
    assert np.abs(yc[:, -1] - ye[:, -1]).max() > 1e-6


def test_beta_matrix_form_equals_materialised_update_norm():
    """Appendix B.1 eq. (beta_chunk): |Delta s_i|^2 from the closed form (with
    the minus sign and clip at 0) equals the squared norm of the materialised
    update Delta s_i = -khat_i P(s0_i) h, built here from an explicit projection
    matrix; the printed '+' would not."""
    rng = _rng(13)
    m, d = 6, 9
    S0 = rng.standard_normal((m, d)) * rng.uniform(0.5, 2.0, (m, 1))
    for _ in range(10):
        x = rng.standard_normal(d)
        c = rng.uniform(0.0, 1.5, m)
        eta = rng.uniform(0.2, 2.0)
        g, kt, dsq, _ = oracle.chunk_token_gates(S0, x, c, mu=0.8, eta=eta)
        h = -x
        for i in range(m):
            s = S0[i]
            P = np.eye(d) - np.outer(s, s) / (s @ s)
            delta = -(c[i] / np.linalg.norm(s)) * (P @ h)
            assert dsq[i] == pytest.approx(eta ** 2 * (delta @ delta), rel=1e-10, abs=1e-14)
            khat = c[i] / np.linalg.norm(s)
            hhat = (h @ s) / (s @ s)
            plus = eta ** 2 * (khat ** 2 * (h @ h) + (s @ s) * hhat ** 2 * khat ** 2)
            if abs(hhat) > 1e-3 and c[i] > 1e-3:
                assert abs(plus - dsq[i]) > 1e-8


# ------------------------------------------------------------ composition ---

def test_resume_composes():
    """The state is the whole carry: scan(T1) then scan(T2) from S_T1 equals
    scan(T1+T2) (exact: any split; chunked: T1 a multiple of C)."""
    rng = _rng(14)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 24, 2, 4, 5)
    for chunk, T1 in ((1, 7), (8, 16)):
        y, S, _ = oracle.scan(x, c, q, mu, S0, chunk=chunk)
        ya, Sa, _ = oracle.scan(x[:, :T1], c[:, :T1], q[:, :T1], mu[:, :T1], S0, chunk=chunk)
        yb, Sb, _ = oracle.scan(x[:, T1:], c[:, T1:], q[:, T1:], mu[:, T1:], Sa, chunk=chunk)
        np.testing.assert_array_equal(np.concatenate([ya, yb], 1), y)
        np.testing.assert_array_equal(Sb, S)


def test_readout_definition():
    """Appendix D listing y = q @ S: y = sum_i q_i s_i, checked entrywise."""
    rng = _rng(15)
    S = rng.standard_normal((2, 3, 5, 7))
    q = rng.standard_normal((2, 3, 5))
    y = oracle.readout(S, q)
    for b in range(2):
        for h in range(3):
            ref = sum(q[b, h, i] * S[b, h, i] for i in range(5))
            np.testing.assert_allclose(y[b, h], ref, atol=1e-13)


def test_threads_do_not_change_results():
    rng = _rng(16)
    x, c, q, mu, S0 = _rand_inputs(rng, 3, 10, 3, 4, 5)
    for chunk in (1, 4):
        y1, S1, _ = oracle.scan(x, c, q, mu, S0, chunk=chunk, nthreads=1)
        y8, S8, _ = oracle.scan(x, c, q, mu, S0, chunk=chunk, nthreads=8)
        np.testing.assert_array_equal(y1, y8)
        np.testing.assert_array_equal(S1, S8)


# --------------------------------------------- reconstruction objective (DEC) ---

def test_dec_write_is_negative_half_gradient_of_reconstruction_loss():
    """§3.1.1 eq. (decoding_stateNorm_loss), eq. (decoding_recurrence) and eq. (OSR)
    with h = e: with mu = 1 the write is -eta (c_i/|s_i|) P(s_i) e, the gradient
    as printed, which is half the gradient of L(S) = |phi(S) c - x|^2 (phi
    normalises each slot). Checked by central finite differences at |s| != 1."""
    rng = _rng(21)
    m, d = 4, 6
    S = rng.standard_normal((m, d)) * rng.uniform(0.5, 2.0, (m, 1))
    x = rng.standard_normal(d)
    c = rng.uniform(0.1, 1.0, m)
    eta = 0.41

    def loss(Sm):
        phi = Sm / np.linalg.norm(Sm, axis=1, keepdims=True)
        e = phi.T @ c - x
        return float(e @ e)

    x_eff = oracle.write_input(S, c, x, mode="dec")
    eps = 1e-6
    for i in range(m):
        grad = np.zeros(d)
        for k in range(d):
            Sp, Sn = S.copy(), S.copy()
            Sp[i, k] += eps
            Sn[i, k] -= eps
            grad[k] = (loss(Sp) - loss(Sn)) / (2 * eps)
        w, _ = oracle.osr_write(S[i], x_eff, c[i], 1.0, eta)
        np.testing.assert_allclose(w - S[i], -eta * grad / 2, rtol=1e-7, atol=1e-9)


@pytest.mark.parametrize("chunk", [1, 4])
def test_dec_perfect_reconstruction_leaves_the_state(chunk):
    """With x_t = phi(S0)^T c_t the reconstruction error is zero, so eq. (OSR)
    writes nothing; the forget gate and the normaliser then leave every slot
    unchanged (§3.2, §3.3), and y_t = q_t S0 at every step, in both forms."""
    rng = _rng(22)
    B, T, H, m, d = 1, 9, 2, 5, 6
    x, c, q, mu, S0 = _rand_inputs(rng, B, T, H, m, d, unit=True)
    for b in range(B):
        for h in range(H):
            phi = S0[b, h] / np.linalg.norm(S0[b, h], axis=1, keepdims=True)
            for t in range(T):
                x[b, t, h] = phi.T @ c[b, t, h]
    y, S, deg = oracle.scan(x, c, q, mu, S0, chunk=chunk, mode="dec")
    assert deg == 0
    np.testing.assert_allclose(S, S0, atol=1e-12)
    np.testing.assert_allclose(y, np.einsum("bthm,bhmd->bthd", q, S0), atol=1e-12)


def test_dec_brute_force_projection_matrices():
    """eq. (OSR) with h = e evaluated literally in the paper's d x m layout: the
    error e = Phi c - x from the current state, the stacked Jacobians
    P(s_i)/|s_i|, the General Form mu S - eta grad, the unit-sphere projection
    (§3.2) and the read-out with the updated state."""
    rng = _rng(23)
    B, T, H, m, d = 2, 8, 2, 3, 5
    x, c, q, mu, S0 = _rand_inputs(rng, B, T, H, m, d, unit=False)
    eta = rng.uniform(0.2, 1.2, (B, T, H))
    y_o, S_o, _ = oracle.scan(x, c, q, mu, S0, eta=eta, mode="dec")
    for b in range(B):
        for hh in range(H):
            Sdm = S0[b, hh].T.copy()  # d x m, slots are columns
            for t in range(T):
                Phi = Sdm / np.linalg.norm(Sdm, axis=0, keepdims=True)
                e = Phi @ c[b, t, hh] - x[b, t, hh]
                P = np.zeros((d, d, m))
                for i in range(m):
                    s = Sdm[:, i]
                    P[:, :, i] = (np.eye(d) - np.outer(s, s) / (s @ s)) / np.linalg.norm(s)
                grad = np.einsum("a,adm->dm", e, P) * c[b, t, hh][None, :]
                Snew = mu[b, t, hh] * Sdm - eta[b, t, hh] * grad
                Sdm = Snew / np.linalg.norm(Snew, axis=0, keepdims=True)
                np.testing.assert_allclose(y_o[b, t, hh], Sdm @ q[b, t, hh], atol=1e-12)
            np.testing.assert_allclose(S_o[b, hh], Sdm.T, atol=1e-12)


def test_dec_chunk_size_one_is_the_exact_recurrence():
    """Appendix D: chunk size 1 is the exact recurrence under the reconstruction
    objective too (the chunk-start state is the current state)."""
    rng = _rng(24)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 13, 2, 6, 7, unit=True)
    y1, S1, _ = oracle.scan(x, c, q, mu, S0, chunk=1, mode="dec")
    from oracle import _load, _f64, _p
    lib = _load()
    B, T, H, d = x.shape
    m = c.shape[-1]
    y2, S2 = np.zeros_like(y1), np.zeros_like(S1)
    lib.oracle_chunked_scan_mode(1, B, T, H, m, d, 1, _p(_f64(x)), _p(_f64(c)), _p(_f64(q)),
                                 _p(_f64(mu)), None, _p(_f64(S0)), _p(S2), _p(y2), 1)
    np.testing.assert_allclose(y2, y1, atol=1e-12)
    np.testing.assert_allclose(S2, S1, atol=1e-12)


@pytest.mark.parametrize("C", [4, 16])
def test_dec_chunk_closed_form_equals_token_form(C):
    """§3.4.1 / Appendix B.1 with H = K Phi - V (Appendix D, compress_chunk): the
    chunk-level matrix form equals the token-wise Eq. 17 recurrence."""
    rng = _rng(200 + C)
    T = 2 * C + 3
    x, c, q, mu, S0 = _rand_inputs(rng, 1, T, 2, 5, 4, unit=False, mu_range=(0.6, 1.0))
    y1, S1, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="token", mode="dec")
    y2, S2, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="matrix", mode="dec")
    np.testing.assert_allclose(y2, y1, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-10)


def test_dec_differs_from_sim():
    """The two objectives write different things (guards against a mode flag
    that is ignored)."""
    rng = _rng(25)
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 4, 1, 3, 5)
    ys, _, _ = oracle.scan(x, c, q, mu, S0, mode="sim")
    yd, _, _ = oracle.scan(x, c, q, mu, S0, mode="dec")
    assert np.abs(ys - yd).max() > 1e-3


# ------------------------------------------- linearisation 1 (recurrence_linear1) ---

def test_lin1_chunk_size_one_is_the_exact_recurrence():
    """§3.4.1: with chunk size 1 the chunk-start state is the current state, so
    eq. (recurrence_linear1) is the exact recurrence."""
    rng = _rng(31)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 11, 2, 5, 6, unit=True)
    y1, S1, _ = oracle.scan(x, c, q, mu, S0, chunk=1)
    from oracle import _load, _f64, _p
    lib = _load()
    B, T, H, d = x.shape
    m = c.shape[-1]
    y2, S2 = np.zeros_like(y1), np.zeros_like(S1)
    lib.oracle_chunked_scan_lin(1, 0, 1, B, T, H, m, d, 1, _p(_f64(x)), _p(_f64(c)), _p(_f64(q)),
                                _p(_f64(mu)), None, _p(_f64(S0)), _p(S2), _p(y2), 1)
    np.testing.assert_allclose(y2, y1, atol=1e-12)
    np.testing.assert_allclose(S2, S1, atol=1e-12)


@pytest.mark.parametrize("C", [4, 16])
@pytest.mark.parametrize("mode", ["sim", "dec"])
def test_lin1_chunk_closed_form_equals_token_form(C, mode):
    """eq. (chunkwise_OSR): the chunk-level form of recurrence_linear1 - gates
    a_tau = prod beta mu, the f / F terms carrying h~ k^ on the chunk-start state,
    the causal score matrix - equals the token-wise recurrence."""
    rng = _rng(300 + C)
    T = 2 * C + 5
    x, c, q, mu, S0 = _rand_inputs(rng, 1, T, 2, 5, 4, unit=False, mu_range=(0.6, 1.0))
    if mode == "dec":
        c *= 0.1
    y1, S1, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="token", lin=1, mode=mode)
    y2, S2, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="matrix", lin=1, mode=mode)
    np.testing.assert_allclose(y2, y1, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-10)


def test_lin1_first_token_is_exact_and_differs_from_eq17_later():
    """Both linearisations are exact on the first token of a chunk; afterwards
    recurrence_linear1 (h~ k^ on the chunk-start slot) and Eq. 17 (on the running
    slot) differ."""
    rng = _rng(32)
    C = 8
    x, c, q, mu, S0 = _rand_inputs(rng, 1, C, 1, 4, 6)
    ye, _, _ = oracle.scan(x, c, q, mu, S0, chunk=1)
    y1, _, _ = oracle.scan(x, c, q, mu, S0, chunk=C, lin=1)
    y2, _, _ = oracle.scan(x, c, q, mu, S0, chunk=C, lin=2)
    np.testing.assert_allclose(y1[:, 0], ye[:, 0], atol=1e-13)
    assert np.abs(y1[:, -1] - y2[:, -1]).max() > 1e-6


def test_lin1_on_the_training_shape_stays_bounded():
    import lattice_inputs as LI
    inp = LI.make_inputs(LI.WORKLOADS["small_train"].with_(B=1, H=2))
    y, S, deg = oracle.scan(inp["x"], inp["c"], inp["q"], inp["mu"], inp["S0"], chunk=64, lin=1)
    assert np.isfinite(y).all() and deg == 0
    n = np.linalg.norm(S, axis=-1)
    assert 0.05 < n.min() and n.max() < 20.0


# --------------------------------- normalisation at chunk boundaries (ablation) ---

@pytest.mark.parametrize("lin", [1, 2])
def test_chunk_norm_with_chunk_size_one_is_the_exact_recurrence(lin):
    """Appendix C, "Per-token vs. Per-chunk Normalization": with no normaliser inside
    a chunk and the unit-sphere projection after each chunk, chunk size 1 writes the
    unnormalised OSR update and projects it: the exact recurrence (§3.2), for either
    linearisation."""
    rng = _rng(41 + lin)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 9, 2, 5, 6, unit=False)
    ye, Se, _ = oracle.scan(x, c, q, mu, S0, chunk=1)
    yc, Sc, _ = oracle.scan(x, c, q, mu, S0, chunk=1, lin=lin, norm="chunk")
    np.testing.assert_allclose(Sc, Se, atol=1e-12)
    # the read-out of a chunk precedes its boundary projection: y_t = q (|w| s_t)
    np.testing.assert_allclose(np.linalg.norm(Sc, axis=-1), 1.0, atol=1e-12)
    assert np.isfinite(yc).all()


@pytest.mark.parametrize("lin", [1, 2])
@pytest.mark.parametrize("C", [4, 16])
def test_chunk_norm_closed_form_equals_token_form(lin, C):
    rng = _rng(400 + C + lin)
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 2 * C + 3, 2, 5, 4, unit=True, mu_range=(0.6, 1.0))
    y1, S1, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="token", lin=lin, norm="chunk")
    y2, S2, _ = oracle.scan(x, c, q, mu, S0, chunk=C, form="matrix", lin=lin, norm="chunk")
    np.testing.assert_allclose(y2, y1, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-10)


def test_chunk_norm_carried_state_is_on_the_sphere_and_differs_from_per_token():
    rng = _rng(43)
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 3 * 8, 2, 5, 6, unit=True)
    yc, Sc, _ = oracle.scan(x, c, q, mu, S0, chunk=8, norm="chunk")
    yt, St, _ = oracle.scan(x, c, q, mu, S0, chunk=8)
    np.testing.assert_allclose(np.linalg.norm(Sc, axis=-1), 1.0, atol=1e-12)
    assert np.abs(yc - yt).max() > 1e-6


@pytest.mark.parametrize("lin", [1, 2])
def test_chunk_norm_zero_write_decays_inside_the_chunk_and_returns_at_the_boundary(lin):
    """With c = 0 nothing is written: inside a chunk the slots are only scaled by the
    running product of mu (no normaliser, beta = 1), each read-out sees that decayed
    state, and the projection after the chunk brings unit slots back to where they
    started. The read-out of a chunk's last token sees the state before the
    projection."""
    rng = _rng(44 + lin)
    C, B, T, H, m, d = 4, 1, 2 * 4 + 3, 2, 3, 5
    x, c, q, mu, S0 = _rand_inputs(rng, B, T, H, m, d, unit=True)
    c[:] = 0.0
    y, S, _ = oracle.scan(x, c, q, mu, S0, chunk=C, lin=lin, norm="chunk")
    for t in range(T):
        t0 = (t // C) * C
        decay = np.prod(mu[:, t0:t + 1, :], axis=1)                   # [B][H]
        want = np.einsum("bhi,bhik->bhk", q[:, t], S0) * decay[..., None]
        np.testing.assert_allclose(y[:, t], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S0, atol=1e-12)


# --------------------------------------------------------------- backward pass ---

def _loss_and_grads(args, dy, dST, chunk):
    def loss(**kw):
        y, S, _ = oracle.scan(kw["x"], kw["c"], kw["q"], kw["mu"], kw["S0"], eta=kw["eta"], chunk=chunk)
        return (dy * y).sum() + (0.0 if dST is None else (dST * S).sum())
    g = oracle.scan_bwd(args["x"], args["c"], args["q"], args["mu"], args["S0"], dy, dST,
                        eta=args["eta"], chunk=chunk)
    return loss, g


@pytest.mark.parametrize("chunk", [1, 4])
@pytest.mark.parametrize("with_eta,with_dST", [(True, True), (False, False)])
def test_backward_equals_central_differences(chunk, with_eta, with_dST):
    """The paper prints no backward pass; its adjoint is fixed by the forward. Every
    gradient entry of L = sum dy.y + dS_T.S_T equals the central difference of the
    (separately pinned) forward, for the exact recurrence and for Eq. 17 with a
    ragged last chunk (T = 9, C = 4)."""
    rng = _rng(50 + chunk + 2 * with_eta)
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 9, 1, 3, 5, unit=False)
    eta = rng.uniform(0.5, 1.5, mu.shape) if with_eta else None
    dy = rng.standard_normal(x.shape)
    dST = rng.standard_normal(S0.shape) if with_dST else None
    args = dict(x=x, c=c, q=q, mu=mu, eta=eta, S0=S0)
    loss, g = _loss_and_grads(args, dy, dST, chunk)
    assert (g["deta"] is None) == (eta is None)
    h = 1e-6
    for name, a in args.items():
        if a is None:
            continue
        num = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            ap, am = a.copy(), a.copy()
            ap[idx] += h
            am[idx] -= h
            num[idx] = (loss(**{**args, name: ap}) - loss(**{**args, name: am})) / (2 * h)
        np.testing.assert_allclose(g["d" + name], num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_chunk_one_matches_exact_except_the_radial_state_gradient():
    """At chunk size 1 with unit slots the two forwards agree (§3.4.1), so every
    gradient agrees too, except the component of dS0 along each slot: the exact
    recurrence projects onto the unit sphere, Eq. 17 keeps the chunk-start norm."""
    rng = _rng(52)
    x, c, q, mu, S0 = _rand_inputs(rng, 2, 7, 2, 3, 5, unit=True)
    dy = rng.standard_normal(x.shape)
    dST = rng.standard_normal(S0.shape)
    a = oracle.scan_bwd(x, c, q, mu, S0, dy, dST, chunk=1)
    b = oracle.scan_bwd(x, c, q, mu, S0, dy, dST, chunk=1, form="chunked")
    for k in ("dx", "dc", "dq", "dmu"):
        np.testing.assert_allclose(a[k], b[k], atol=1e-12, err_msg=k)
    r = a["dS0"] - b["dS0"]
    tangential = r - (r * S0).sum(-1, keepdims=True) * S0
    np.testing.assert_allclose(tangential, 0.0, atol=1e-12)
    assert np.abs((r * S0).sum(-1)).max() > 1e-3


def test_backward_of_a_single_token_readout():
    """T = 1: dL/dq_i = dy . s_1,i with s_1 the returned final state (Appendix D
    read-out), and with dy = 0 only dS_T drives the gradients."""
    rng = _rng(53)
    x, c, q, mu, S0 = _rand_inputs(rng, 1, 1, 2, 4, 6, unit=True)
    dy = rng.standard_normal(x.shape)
    y, S, _ = oracle.scan(x, c, q, mu, S0, chunk=1)
    g = oracle.scan_bwd(x, c, q, mu, S0, dy, None, chunk=1)
    np.testing.assert_allclose(g["dq"][:, 0], np.einsum("bhd,bhid->bhi", dy[:, 0], S), atol=1e-13)
    g0 = oracle.scan_bwd(x, c, q, mu, S0, np.zeros_like(dy), None, chunk=1)
    for k in ("dx", "dc", "dq", "dmu", "dS0"):
        assert not np.any(g0[k])
