"""Python binding of liblattice (B200, sm_100a): the Lattice compression-layer
state recurrence ("Lattice: Learning to Efficiently Compress the Memory",
arXiv 2504.05646, §3).

This module only marshals arguments: it checks tensor placement, dtypes and
shapes, and passes raw device pointers and the current CUDA stream to the C
ABI declared in include/lattice.h. Every step of the computation runs in the
library's CUDA kernels. There is no CPU or PyTorch fallback: without the built
library every call raises.

Tensors (row-major, contiguous, on one CUDA device):
    x   [B, T, H, d]  float32 or bfloat16      c   [B, T, H, m] float32
    q   [B, T, H, m]  float32 or bfloat16      mu  [B, T, H]    float32
    eta [B, T, H]     float32 or None (=1)     S0  [B, H, m, d] float32
Decode calls drop the T axis.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["LatticeError", "lib", "scan_fwd", "scan_bwd", "scan_bwd_workspace_bytes", "step",
           "readout", "chunk_impl", "device_status", "selftest_bounded_wait", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblattice.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = range(5)
_F32, _BF16 = 0, 1
_IMPL = {"auto": 0, "simt": 1, "tcgen05": 2, "tcgen05_split": 3, "split_reg": 4, "split_reg8": 5}
_MODE = {"sim": 0, "dec": 1}
_lib = None


class LatticeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = _lib.lattice_status_string(code).decode() if _lib is not None else str(code)
        if code == ERR_CUDA and _lib is not None:
            msg += " [" + _lib.lattice_last_cuda_error().decode() + "]"
        super().__init__(f"{what}: {msg} (status {code})")


def lib() -> ctypes.CDLL:
    """Load liblattice.so (built in-tree by orthogonal_update_recurrent_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"liblattice.so not found at {LIB_PATH}; build it with "
                "`python -m orthogonal_update_recurrent_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, fp = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
        L.lattice_scan_fwd.argtypes = [vp, i, fp, vp, i, fp, fp, fp, fp, fp, i, i, i, i, i, i, i, vp]
        L.lattice_scan_fwd_impl.argtypes = [vp, i, fp, vp, i, fp, fp, fp, fp, fp, i, i, i, i, i,
                                            i, i, i, vp]
        L.lattice_scan_fwd_ex.argtypes = [vp, i, fp, vp, i, fp, fp, fp, fp, fp, i, i, i, i, i,
                                          i, i, i, i, vp]
        L.lattice_scan_bwd.argtypes = [vp, i, fp, vp, i, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp,
                                       fp, vp, ctypes.c_size_t, i, i, i, i, i, i, i, vp]
        L.lattice_scan_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        L.lattice_scan_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.lattice_step.argtypes = [fp, vp, i, fp, vp, i, fp, fp, fp, i, i, i, i, i, vp]
        L.lattice_readout.argtypes = [fp, vp, i, fp, i, i, i, i, vp]
        L.lattice_get_device_status.argtypes = [vp]
        L.lattice_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, vp]
        L.lattice_status_string.argtypes = [i]
        L.lattice_status_string.restype = ctypes.c_char_p
        L.lattice_version.argtypes = []
        L.lattice_chunk_impl.argtypes = [i, i, i, i, i, i, i]
        L.lattice_last_cuda_error.argtypes = []
        L.lattice_last_cuda_error.restype = ctypes.c_char_p
        for f in ("lattice_scan_fwd", "lattice_scan_fwd_impl", "lattice_scan_fwd_ex", "lattice_scan_bwd",
                  "lattice_step", "lattice_readout", "lattice_selftest_bounded_wait",
                  "lattice_get_device_status", "lattice_version", "lattice_chunk_impl"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return _F32
    if t.dtype == torch.bfloat16:
        return _BF16
    raise TypeError(f"expected float32 or bfloat16, got {t.dtype}")


def _chk(t: torch.Tensor, name: str, shape, dtypes=(torch.float32,)):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must have dtype in {dtypes}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _raise(code: int, what: str):
    if code != OK:
        raise LatticeError(code, what)


_XQ = (torch.float32, torch.bfloat16)


def scan_fwd(x: torch.Tensor, c: torch.Tensor, q: torch.Tensor, mu: torch.Tensor,
             S0: torch.Tensor, eta: Optional[torch.Tensor] = None, chunk: int = 1,
             S_out: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
             impl: str = "auto", stream=None, mode: str = "sim",
             lin: int = 2, norm: str = "token") -> Tuple[torch.Tensor, torch.Tensor]:
    """Whole-sequence forward (the paper's lattice_compress, Appendix D).
    chunk == 1: exact recurrence; chunk > 1: the chunked form, Eq. 17 (lin=2) or
    eq. recurrence_linear1 (lin=1); norm "chunk" drops the per-token normaliser and
    projects the slots onto the unit sphere after each chunk. mode "sim": similarity
    objective; "dec": reconstruction objective.
    Returns (y [B,T,H,d] float32, S_T [B,H,m,d] float32). S_out may be S0."""
    B, T, H, d = x.shape
    m = c.shape[-1]
    _chk(x, "x", (B, T, H, d), _XQ)
    _chk(c, "c", (B, T, H, m))
    _chk(q, "q", (B, T, H, m), _XQ)
    _chk(mu, "mu", (B, T, H))
    _chk(S0, "S0", (B, H, m, d))
    if eta is not None:
        _chk(eta, "eta", (B, T, H))
    if S_out is None:
        S_out = torch.empty_like(S0)
    _chk(S_out, "S_out", (B, H, m, d))
    if y is None:
        y = torch.empty((B, T, H, d), dtype=torch.float32, device=x.device)
    _chk(y, "y", (B, T, H, d))
    L = lib()
    code = L.lattice_scan_fwd_ex(_ptr(x), _dt(x), _ptr(c), _ptr(q), _dt(q), _ptr(mu), _ptr(eta),
                                 _ptr(S0), _ptr(S_out), _ptr(y), B, T, H, m, d, int(chunk),
                                 _MODE[mode], {2: 0, 1: 1}[lin] | {"token": 0, "chunk": 2}[norm],
                                 _IMPL[impl], _stream(stream))
    _raise(code, "lattice_scan_fwd")
    return y, S_out


def scan_bwd_workspace_bytes(B: int, T: int, H: int, m: int, d: int, chunk: int = 1,
                             seg: int = 0) -> int:
    """Device workspace bytes scan_bwd needs (0: the shape is not supported)."""
    return int(lib().lattice_scan_bwd_workspace_bytes(B, T, H, m, d, int(chunk), int(seg)))


def scan_bwd(x: torch.Tensor, c: torch.Tensor, q: torch.Tensor, mu: torch.Tensor,
             S0: torch.Tensor, dy: torch.Tensor, dS_T: Optional[torch.Tensor] = None,
             eta: Optional[torch.Tensor] = None, chunk: int = 1, seg: int = 0,
             workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Backward pass of scan_fwd (similarity objective; exact for chunk 1, Eq. 17
    otherwise): gradients of L = sum_t dy_t . y_t + dS_T . S_T. Returns a dict with
    dx, dc, dq, dmu, deta (None when eta is None) and dS0, all float32. seg: tokens
    between state checkpoints (0: default). workspace: optional uint8 device tensor of
    at least scan_bwd_workspace_bytes(...) bytes; allocated when None."""
    B, T, H, d = x.shape
    m = c.shape[-1]
    _chk(x, "x", (B, T, H, d), _XQ)
    _chk(c, "c", (B, T, H, m))
    _chk(q, "q", (B, T, H, m), _XQ)
    _chk(mu, "mu", (B, T, H))
    _chk(S0, "S0", (B, H, m, d))
    _chk(dy, "dy", (B, T, H, d))
    if dS_T is not None:
        _chk(dS_T, "dS_T", (B, H, m, d))
    if eta is not None:
        _chk(eta, "eta", (B, T, H))
    L = lib()
    need = L.lattice_scan_bwd_workspace_bytes(B, T, H, m, d, int(chunk), int(seg))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or not workspace.is_contiguous():
        raise TypeError("workspace must be a contiguous CUDA tensor")
    f32 = dict(dtype=torch.float32, device=x.device)
    out = {"dx": torch.empty((B, T, H, d), **f32), "dc": torch.empty((B, T, H, m), **f32),
           "dq": torch.empty((B, T, H, m), **f32), "dmu": torch.empty((B, T, H), **f32),
           "deta": None if eta is None else torch.empty((B, T, H), **f32),
           "dS0": torch.empty((B, H, m, d), **f32)}
    code = L.lattice_scan_bwd(_ptr(x), _dt(x), _ptr(c), _ptr(q), _dt(q), _ptr(mu), _ptr(eta),
                              _ptr(S0), _ptr(dy), _ptr(dS_T), _ptr(out["dx"]), _ptr(out["dc"]),
                              _ptr(out["dq"]), _ptr(out["dmu"]), _ptr(out["deta"]), _ptr(out["dS0"]),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              B, T, H, m, d, int(chunk), int(seg), _stream(stream))
    _raise(code, "lattice_scan_bwd")
    return out


def step(S: torch.Tensor, x: torch.Tensor, c: torch.Tensor, q: torch.Tensor, mu: torch.Tensor,
         eta: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
         stream=None, mode: str = "sim") -> torch.Tensor:
    """One decode step, state updated in place. S [B,H,m,d], x [B,H,d], c/q [B,H,m],
    mu/eta [B,H]. Returns y [B,H,d]."""
    B, H, m, d = S.shape
    _chk(S, "S", (B, H, m, d))
    _chk(x, "x", (B, H, d), _XQ)
    _chk(c, "c", (B, H, m))
    _chk(q, "q", (B, H, m), _XQ)
    _chk(mu, "mu", (B, H))
    if eta is not None:
        _chk(eta, "eta", (B, H))
    if y is None:
        y = torch.empty((B, H, d), dtype=torch.float32, device=S.device)
    _chk(y, "y", (B, H, d))
    code = lib().lattice_step(_ptr(S), _ptr(x), _dt(x), _ptr(c), _ptr(q), _dt(q), _ptr(mu),
                              _ptr(eta), _ptr(y), B, H, m, d, _MODE[mode], _stream(stream))
    _raise(code, "lattice_step")
    return y


def readout(S: torch.Tensor, q: torch.Tensor, y: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """y[b,h,:] = sum_i q[b,h,i] S[b,h,i,:]."""
    B, H, m, d = S.shape
    _chk(S, "S", (B, H, m, d))
    _chk(q, "q", (B, H, m), _XQ)
    if y is None:
        y = torch.empty((B, H, d), dtype=torch.float32, device=S.device)
    _chk(y, "y", (B, H, d))
    code = lib().lattice_readout(_ptr(S), _ptr(q), _dt(q), _ptr(y), B, H, m, d, _stream(stream))
    _raise(code, "lattice_readout")
    return y


def chunk_impl(B: int, H: int, m: int, d: int, chunk: int, x_dtype=torch.bfloat16,
               q_dtype=torch.bfloat16) -> str:
    """Name of the kernel the automatic choice runs for a chunked scan of B x H sequences:
    "split_reg", "tcgen05_split", "tcgen05" or "simt"."""
    dt = lambda t: _BF16 if t == torch.bfloat16 else _F32
    code = lib().lattice_chunk_impl(B, H, m, d, chunk, dt(x_dtype), dt(q_dtype))
    return {1: "simt", 2: "tcgen05", 3: "tcgen05_split", 4: "split_reg", 5: "split_reg8"}[code]


def device_status(stream=None) -> int:
    """Synchronise the stream; raise LatticeError if a kernel gave up a bounded wait."""
    code = lib().lattice_get_device_status(_stream(stream))
    _raise(code, "lattice_get_device_status")
    return code


def selftest_bounded_wait(limit_ns: int = 1_000_000, stream=None) -> None:
    """Launch the library's bounded-wait self-test: one warp waits on a barrier that
    nothing completes and gives up after limit_ns. The next device_status() on the
    same stream then raises LatticeError with code ERR_TIMEOUT."""
    _raise(lib().lattice_selftest_bounded_wait(int(limit_ns), _stream(stream)),
           "lattice_selftest_bounded_wait")
