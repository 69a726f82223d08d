"""fp64 CPU oracle of the Lattice compression-layer state recurrence.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the library. The arithmetic lives in
``lattice_oracle.c`` (plain C, fp64, token by token); this module compiles it
with gcc and marshals numpy arrays. See that file's header for the paper
passages each function follows and for the readings of open points.

Parity status: every function here is pinned by tests/test_oracle_pins.py
against values and properties the paper and the mathematics fix.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lattice_oracle.c")
_LIB = os.path.join(_HERE, "liblattice_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle to oracle/liblattice_oracle.so (plain IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i, ll = ctypes.c_int, ctypes.c_longlong
        scan_args = [i, i, i, i, i, _D, _D, _D, _D, _D, _D, _D, _D, i]
        lib.oracle_exact_scan.argtypes = scan_args
        lib.oracle_exact_scan.restype = ll
        for name in ("oracle_chunked_scan", "oracle_chunked_matrix_scan"):
            f = getattr(lib, name)
            f.argtypes = [i, i, i, i, i, i, _D, _D, _D, _D, _D, _D, _D, _D, i]
            f.restype = ll
        lib.oracle_exact_scan_mode.argtypes = [i] + scan_args
        lib.oracle_exact_scan_mode.restype = ll
        for name in ("oracle_chunked_scan_mode", "oracle_chunked_matrix_scan_mode"):
            f = getattr(lib, name)
            f.argtypes = [i, i, i, i, i, i, i, _D, _D, _D, _D, _D, _D, _D, _D, i]
            f.restype = ll
        lib.oracle_chunked_scan_lin.argtypes = [i, i, i, i, i, i, i, i, i, _D, _D, _D, _D, _D, _D, _D, _D, i]
        lib.oracle_chunked_scan_lin.restype = ll
        lib.oracle_write_input.argtypes = [i, i, i, _D, _D, _D, _D]
        lib.oracle_write_input.restype = None
        lib.oracle_readout.argtypes = [i, i, i, i, _D, _D, _D]
        lib.oracle_readout.restype = None
        lib.oracle_osr_write.argtypes = [i, _D, _D, ctypes.c_double, ctypes.c_double,
                                         ctypes.c_double, _D, _D]
        lib.oracle_osr_write.restype = None
        lib.oracle_chunk_token_gates.argtypes = [i, i, _D, _D, _D, _D, ctypes.c_double,
                                                 ctypes.c_double, _D, _D, _D,
                                                 ctypes.POINTER(ll)]
        lib.oracle_chunk_token_gates.restype = None
        lib.oracle_scan_bwd.argtypes = [i, i, i, i, i, i, i] + [_D] * 14 + [i]
        lib.oracle_scan_bwd.restype = None
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(_D)


def _threads(n: Optional[int]) -> int:
    if n is not None:
        return n
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


_MODES = {"sim": 0, "dec": 1}


def scan(x, c, q, mu, S0, eta=None, chunk: int = 1, form: str = "token",
         nthreads: Optional[int] = None, mode: str = "sim", lin: int = 2, norm: str = "token"):
    """Whole-sequence forward. x[B][T][H][d], c/q[B][T][H][m], mu/eta[B][T][H],
    S0[B][H][m][d]. chunk == 1: exact recurrence; chunk > 1: Eq. 17 chunked
    recurrence, evaluated token by token (form="token") or through the
    chunk-level closed form (form="matrix"). mode "sim": similarity objective
    (h = -x); "dec": reconstruction objective (h = phi(S) c - x). lin selects the
    chunk linearisation of §3.4.1: 2 = Eq. 17 (recurrence_linear2), 1 =
    recurrence_linear1. norm "token": the per-token normaliser; "chunk": none inside
    a chunk, every slot projected onto the unit sphere after each chunk (Appendix C
    ablation). Returns (y, S_T, n_degenerate)."""
    md = _MODES[mode]
    x, c, q, mu, S0 = map(_f64, (x, c, q, mu, S0))
    eta = None if eta is None else _f64(eta)
    B, T, H, d = x.shape
    m = c.shape[-1]
    assert c.shape == (B, T, H, m) and q.shape == (B, T, H, m) and mu.shape == (B, T, H)
    assert S0.shape == (B, H, m, d)
    y = np.zeros((B, T, H, d))
    S = np.zeros((B, H, m, d))
    lib = _load()
    nt = _threads(nthreads)
    args = (_p(x), _p(c), _p(q), _p(mu), _p(eta), _p(S0), _p(S), _p(y), nt)
    if lin not in (1, 2) or norm not in ("token", "chunk"):
        raise ValueError((lin, norm))
    if norm == "chunk" or lin == 1:
        code = lin | (4 if norm == "chunk" else 0)
        if form not in ("token", "matrix"):
            raise ValueError(form)
        deg = lib.oracle_chunked_scan_lin(1 if form == "token" else 2, md, code, B, T, H, m, d, chunk, *args)
    elif chunk == 1 and form == "token":
        deg = lib.oracle_exact_scan_mode(md, B, T, H, m, d, *args)
    elif form == "token":
        deg = lib.oracle_chunked_scan_mode(md, B, T, H, m, d, chunk, *args)
    elif form == "matrix":
        deg = lib.oracle_chunked_matrix_scan_mode(md, B, T, H, m, d, chunk, *args)
    else:
        raise ValueError(form)
    return y, S, int(deg)


def scan_bwd(x, c, q, mu, S0, dy, dS_T=None, eta=None, chunk: int = 1,
             nthreads: Optional[int] = None, form: Optional[str] = None):
    """Gradients of L = sum_t dy_t . y_t + dS_T . S_T through the similarity-objective
    scan (the exact recurrence for chunk == 1, Eq. 17 with the chunk size otherwise;
    form="chunked" forces the chunked definition at chunk 1). Returns a dict with
    dx, dc, dq, dmu, deta (None when eta is None) and dS0, in the inputs' layouts."""
    x, c, q, mu, S0, dy = map(_f64, (x, c, q, mu, S0, dy))
    eta = None if eta is None else _f64(eta)
    dS_T = None if dS_T is None else _f64(dS_T)
    B, T, H, d = x.shape
    m = c.shape[-1]
    assert c.shape == (B, T, H, m) and q.shape == (B, T, H, m) and mu.shape == (B, T, H)
    assert S0.shape == (B, H, m, d) and dy.shape == (B, T, H, d)
    if form is None:
        form = "exact" if chunk == 1 else "chunked"
    out = {"dx": np.zeros_like(x), "dc": np.zeros_like(c), "dq": np.zeros_like(q),
           "dmu": np.zeros_like(mu), "deta": None if eta is None else np.zeros_like(eta),
           "dS0": np.zeros_like(S0)}
    _load().oracle_scan_bwd({"exact": 0, "chunked": 1}[form], B, T, H, m, d, chunk,
                            _p(x), _p(c), _p(q), _p(mu), _p(eta), _p(S0), _p(dy), _p(dS_T),
                            _p(out["dx"]), _p(out["dc"]), _p(out["dq"]), _p(out["dmu"]),
                            _p(out["deta"]), _p(out["dS0"]), _threads(nthreads))
    return out


def step(S, x, c, q, mu, eta=None, nthreads: Optional[int] = None, mode: str = "sim"):
    """One decode step (the exact recurrence with T = 1). S[B][H][m][d],
    x[B][H][d], c/q[B][H][m], mu/eta[B][H]. Returns (y[B][H][d], S_new, n_degenerate)."""
    x = _f64(x)[:, None]
    c = _f64(c)[:, None]
    q = _f64(q)[:, None]
    mu = _f64(mu)[:, None]
    eta = None if eta is None else _f64(eta)[:, None]
    y, S_new, deg = scan(x, c, q, mu, S, eta=eta, chunk=1, nthreads=nthreads, mode=mode)
    return y[:, 0], S_new, deg


def write_input(S, c, x, mode: str = "dec"):
    """-h of one token against the slots S[m][d] (x for "sim"; x - sum_i c_i s_i/|s_i| for "dec")."""
    S, c, x = _f64(S), _f64(c), _f64(x)
    m, d = S.shape
    out = np.zeros(d)
    _load().oracle_write_input(_MODES[mode], m, d, _p(S), _p(c), _p(x), _p(out))
    return out


def readout(S, q):
    """y[B][H][d] = sum_i q[B][H][i] S[B][H][i][:]."""
    S, q = _f64(S), _f64(q)
    B, H, m, d = S.shape
    y = np.zeros((B, H, d))
    _load().oracle_readout(B, H, m, d, _p(S), _p(q), _p(y))
    return y


def osr_write(s, x, c: float, mu: float, eta: float = 1.0):
    """Unnormalised single-slot write w = mu s + eta (c/|s|) P(s) x. Returns (w, |s|^2)."""
    s, x = _f64(s), _f64(x)
    w = np.zeros_like(s)
    n2 = ctypes.c_double(0.0)
    _load().oracle_osr_write(s.shape[0], _p(s), _p(x), c, mu, eta, _p(w), ctypes.byref(n2))
    return w, n2.value


def chunk_token_gates(S0, x, c, mu: float, eta: float = 1.0):
    """Per-slot gates of one token against a chunk-start state S0[m][d].
    Returns (g[m], kt[m], dsq[m], n_degenerate)."""
    S0, x, c = _f64(S0), _f64(x), _f64(c)
    m, d = S0.shape
    n2 = _f64((S0 * S0).sum(-1))
    g, kt, dsq = np.zeros(m), np.zeros(m), np.zeros(m)
    deg = ctypes.c_longlong(0)
    _load().oracle_chunk_token_gates(m, d, _p(S0), _p(n2), _p(x), _p(c), mu, eta, _p(g),
                                     _p(kt), _p(dsq), ctypes.byref(deg))
    return g, kt, dsq, deg.value
