"""Shared test helpers: device upload of generated inputs and the error metric."""
import numpy as np

try:
    import torch
except Exception:  # pragma: no cover
    torch = None


def rel_err_per_slice(gpu, ref, slice_axes):
    """Relative error of the design notes: per (b,h) slice max|gpu-ref| / max|ref|,
    then the max over slices. `slice_axes` are the axes that index a slice."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    other = tuple(a for a in range(ref.ndim) if a not in slice_axes)
    num = np.abs(gpu - ref).max(axis=other)
    den = np.abs(ref).max(axis=other)
    return float((num / np.maximum(den, 1e-30)).max())


def y_err(gpu_y, ref_y):
    """y is [B,T,H,d]: slices are (b, h)."""
    return rel_err_per_slice(gpu_y, ref_y, (0, 2))


def s_err(gpu_S, ref_S):
    """S is [B,H,m,d]: slices are (b, h)."""
    return rel_err_per_slice(gpu_S, ref_S, (0, 1))


def dev_inputs(inp, device="cuda"):
    """Upload a lattice_inputs dict: bf16 tensors from their bit patterns, fp32 otherwise."""
    def vec(name):
        bits = inp.get(name + "_bits")
        if bits is not None:
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(inp[name], dtype=np.float32)).to(device)

    out = dict(x=vec("x"), q=vec("q"),
               c=torch.from_numpy(np.ascontiguousarray(inp["c"], np.float32)).to(device),
               mu=torch.from_numpy(np.ascontiguousarray(inp["mu"], np.float32)).to(device))
    if "S0" in inp:
        out["S0"] = torch.from_numpy(np.ascontiguousarray(inp["S0"], np.float32)).to(device)
    eta = inp.get("eta")
    out["eta"] = None if eta is None else torch.from_numpy(
        np.ascontiguousarray(eta, np.float32)).to(device)
    return out
