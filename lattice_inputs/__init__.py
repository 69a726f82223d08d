"""Seeded synthetic inputs for the Lattice compression-layer state recurrence.

This module is shared by the fp64 oracle tests, the CUDA parity tests and the
benchmark. It holds only random-number generation and storage-format rounding;
none of the recurrence's arithmetic lives here.

The workloads stand in for the language-model activations the paper trains on
(Lattice: Learning to Efficiently Compress the Memory, §4 and Appendix C): the
datasets and trained projection weights are not available, so the recurrence's
inputs are drawn from the distributions below with the paper's head sizes
(d_head = 64, Appendix C hyper-parameter table) and chunk size 64 (Appendix C.2).

Layouts (row-major), following the listing's argument shapes in Appendix D:
    x   [B][T][H][d]   input written into the slots (the listing's V)
    c   [B][T][H][m]   per-slot writing intensity / code (the listing's K)
    q   [B][T][H][m]   read-out query
    mu  [B][T][H]      forget gate
    eta [B][T][H]      step size (None => 1)
    S0  [B][H][m][d]   initial state, one slot per row
Bf16 tensors are produced as fp32, rounded to nearest-even, and kept both as
raw uint16 bit patterns (for the device) and as the exactly representable fp32
values (for the oracle, which widens them to fp64 without loss).
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "bf16_round_bits", "bf16_bits_to_f32", "make_inputs",
    "make_decode_state", "make_decode_steps", "sample_heads", "make_cotangents",
]


def bf16_round_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-z.astype(np.float64)))).astype(np.float32)


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, storage dtypes and input distributions."""
    name: str
    B: int
    T: int
    H: int
    m: int
    d: int
    x_dtype: str = "bf16"          # "f32" or "bf16"
    q_dtype: str = "bf16"
    x_std: Optional[float] = None  # None => 1/sqrt(d)
    q_std: Optional[float] = None
    c_loc: float = 0.0             # c = sigmoid(N(c_loc, c_scale))
    c_scale: float = 1.0
    mu_loc: float = 3.0            # mu = sigmoid(N(mu_loc, mu_scale))
    mu_scale: float = 1.0
    dup_frac: float = 0.0          # fraction of positions t>=1 that copy an earlier token
    chunk: int = 64                # 1 => exact recurrence
    seed: int = 0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def sx(self) -> float:
        return self.x_std if self.x_std is not None else 1.0 / np.sqrt(self.d)

    @property
    def sq(self) -> float:
        return self.q_std if self.q_std is not None else 1.0 / np.sqrt(self.d)


# The five workloads of the hot path (names describe what each one is).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", B=1, H=1, T=256, m=16, d=32, x_dtype="f32",
                         q_dtype="f32", x_std=1.0, q_std=1.0, mu_loc=2.0, chunk=1, seed=0),
    "small_train": Workload("small_train", B=4, H=8, T=2048, m=64, d=64, seed=1),
    "mid_layer": Workload("mid_layer", B=8, H=16, T=4096, m=128, d=128, dup_frac=0.10, seed=2),
    "long_ctx": Workload("long_ctx", B=1, H=16, T=65536, m=64, d=128, mu_loc=4.0,
                         mu_scale=0.5, seed=3),
    # Decode: one token per sequence per step; T here counts distinct pre-drawn steps.
    "decode": Workload("decode", B=256, H=32, T=1, m=128, d=128, chunk=1, seed=4),
}


def _draw_vec(rng, shape, std, dtype):
    v = rng.standard_normal(shape, dtype=np.float32)
    v *= np.float32(std)
    if dtype == "bf16":
        bits = bf16_round_bits(v)
        return bf16_bits_to_f32(bits), bits
    return v, None


def _unit_rows(rng, shape):
    s = rng.standard_normal(shape, dtype=np.float32).astype(np.float64)
    s /= np.sqrt((s * s).sum(-1, keepdims=True))
    return s.astype(np.float32)


def make_inputs(w: Workload, T: Optional[int] = None, B: Optional[int] = None,
                H: Optional[int] = None) -> dict:
    """Draw one workload's inputs. Draw order: x, q, c, mu, S0, duplicates.

    Returns a dict with fp32 arrays x, q, c, mu, S0 (bf16-valued where the
    workload stores bf16), the uint16 bit patterns x_bits / q_bits (or None),
    eta=None and the list of duplicated positions.
    """
    B = w.B if B is None else B
    T = w.T if T is None else T
    H = w.H if H is None else H
    rng = np.random.default_rng(w.seed)
    x, x_bits = _draw_vec(rng, (B, T, H, w.d), w.sx, w.x_dtype)
    q, q_bits = _draw_vec(rng, (B, T, H, w.m), w.sq, w.q_dtype)
    c = _sigmoid(w.c_loc + w.c_scale * rng.standard_normal((B, T, H, w.m), dtype=np.float32))
    mu = _sigmoid(w.mu_loc + w.mu_scale * rng.standard_normal((B, T, H), dtype=np.float32))
    S0 = _unit_rows(rng, (B, H, w.m, w.d))
    dups = []
    if w.dup_frac > 0 and T > 1:
        n_dup = int(round(w.dup_frac * (T - 1)))
        for b in range(B):
            pos = np.sort(rng.choice(np.arange(1, T), size=n_dup, replace=False))
            src = (rng.random(n_dup) * pos).astype(np.int64)  # uniform in [0, t)
            for t, s in zip(pos.tolist(), src.tolist()):
                # copy the whole token (every head) from an earlier position
                x[b, t] = x[b, s]
                q[b, t] = q[b, s]
                c[b, t] = c[b, s]
                mu[b, t] = mu[b, s]
                if x_bits is not None:
                    x_bits[b, t] = x_bits[b, s]
                if q_bits is not None:
                    q_bits[b, t] = q_bits[b, s]
                dups.append((b, t, s))
    return dict(x=x, q=q, c=c, mu=mu, S0=S0, eta=None, x_bits=x_bits, q_bits=q_bits,
                dups=dups, B=B, T=T, H=H, m=w.m, d=w.d)


def make_decode_state(w: Workload, B: Optional[int] = None, H: Optional[int] = None) -> np.ndarray:
    """Initial decode state [B][H][m][d]: random unit-norm rows (fp32)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    rng = np.random.default_rng([w.seed, 1])
    return _unit_rows(rng, (B, H, w.m, w.d))


def make_decode_steps(w: Workload, n_steps: int, B: Optional[int] = None,
                      H: Optional[int] = None) -> dict:
    """Per-step decode inputs, stacked on a leading step axis:
    x [n][B][H][d], q [n][B][H][m], c [n][B][H][m], mu [n][B][H]."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    rng = np.random.default_rng([w.seed, 2])
    x, x_bits = _draw_vec(rng, (n_steps, B, H, w.d), w.sx, w.x_dtype)
    q, q_bits = _draw_vec(rng, (n_steps, B, H, w.m), w.sq, w.q_dtype)
    c = _sigmoid(w.c_loc + w.c_scale * rng.standard_normal((n_steps, B, H, w.m), dtype=np.float32))
    mu = _sigmoid(w.mu_loc + w.mu_scale * rng.standard_normal((n_steps, B, H), dtype=np.float32))
    return dict(x=x, q=q, c=c, mu=mu, eta=None, x_bits=x_bits, q_bits=q_bits,
                n=n_steps, B=B, H=H, m=w.m, d=w.d)


def sample_heads(inp: dict, pairs) -> dict:
    """Slice a make_inputs() dict down to the given (b, h) pairs, each as its own
    batch row with H=1, so the oracle can run sampled sequences one by one."""
    out = {}
    bs = [p[0] for p in pairs]
    hs = [p[1] for p in pairs]
    out["x"] = np.ascontiguousarray(inp["x"][bs, :, hs][:, :, None, :])
    out["q"] = np.ascontiguousarray(inp["q"][bs, :, hs][:, :, None, :])
    out["c"] = np.ascontiguousarray(inp["c"][bs, :, hs][:, :, None, :])
    out["mu"] = np.ascontiguousarray(inp["mu"][bs, :, hs][:, :, None])
    out["S0"] = np.ascontiguousarray(inp["S0"][bs, hs][:, None])
    out["eta"] = None if inp.get("eta") is None else np.ascontiguousarray(
        inp["eta"][bs, :, hs][:, :, None])
    out.update(B=len(pairs), T=inp["T"], H=1, m=inp["m"], d=inp["d"])
    return out


def make_cotangents(inp: dict, seed: int = 0, with_dS_T: bool = True) -> dict:
    """Upstream gradients for a backward pass over make_inputs(...) = inp:
    dy [B][T][H][d] ~ N(0, 1) and dS_T [B][H][m][d] ~ N(0, 1) (or None), fp32."""
    B, T, H, m, d = inp["B"], inp["T"], inp["H"], inp["m"], inp["d"]
    rng = np.random.default_rng([seed, 3])
    dy = rng.standard_normal((B, T, H, d), dtype=np.float32)
    dS_T = rng.standard_normal((B, H, m, d), dtype=np.float32) if with_dS_T else None
    return dict(dy=dy, dS_T=dS_T)
