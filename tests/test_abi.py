"""The C-ABI library loads and exports every entry point include/lattice.h
declares; host-side argument checks answer before anything reaches a GPU."""
import ctypes
import os
import re

import pytest

import orthogonal_update_recurrent_b200 as L
from orthogonal_update_recurrent_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "lattice.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lattice_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("lattice_scan_fwd", "lattice_step", "lattice_readout", "lattice_get_device_status",
              "lattice_status_string", "lattice_scan_fwd_impl", "lattice_version", "lattice_scan_bwd",
              "lattice_scan_bwd_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert lib.lattice_version() >= 100


def test_status_strings(lib):
    for code in range(5):
        assert lib.lattice_status_string(code)
    assert lib.lattice_status_string(99) == b"unknown status"


def _scan(lib, **kw):
    a = dict(x=1 << 20, xdt=0, c=2 << 20, q=3 << 20, qdt=0, mu=4 << 20, eta=None, S0=5 << 20,
             So=6 << 20, y=7 << 20, B=1, T=4, H=1, m=4, d=16, chunk=1, mode=0, impl=0)
    a.update(kw)
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return lib.lattice_scan_fwd_impl(v(a["x"]), a["xdt"], v(a["c"]), v(a["q"]), a["qdt"], v(a["mu"]),
                                     v(a["eta"]), v(a["S0"]), v(a["So"]), v(a["y"]), a["B"], a["T"],
                                     a["H"], a["m"], a["d"], a["chunk"], a["mode"], a["impl"], None)


def test_argument_checks_return_before_launch(lib):
    # Every case below fails validation, so no CUDA call is made (none could run here).
    assert _scan(lib, x=None) == L.ERR_INVALID_ARG
    assert _scan(lib, S0=None) == L.ERR_INVALID_ARG
    assert _scan(lib, B=0) == L.ERR_INVALID_ARG
    assert _scan(lib, T=-1) == L.ERR_INVALID_ARG
    assert _scan(lib, chunk=0) == L.ERR_INVALID_ARG
    assert _scan(lib, d=48) == L.ERR_UNSUPPORTED
    assert _scan(lib, m=257) == L.ERR_UNSUPPORTED
    assert _scan(lib, xdt=7) == L.ERR_INVALID_ARG
    assert _scan(lib, mode=2) == L.ERR_INVALID_ARG
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    ex = lambda form, impl: lib.lattice_scan_fwd_ex(v(1 << 20), 0, v(2 << 20), v(3 << 20), 0, v(4 << 20), None,
                                                    v(5 << 20), v(6 << 20), v(7 << 20), 1, 4, 1, 64, 64, 64,
                                                    0, form, impl, None)
    assert ex(5, 0) == L.ERR_INVALID_ARG        # unknown chunk form
    assert ex(4, 0) == L.ERR_INVALID_ARG
    assert ex(2, 3) == L.ERR_UNSUPPORTED        # normalisation at chunk boundaries: CUDA-core kernel
    assert ex(1, 2) == L.ERR_UNSUPPORTED        # linearisation 1 runs on the CUDA-core kernel
    assert _scan(lib, mode=1, impl=2) == L.ERR_UNSUPPORTED  # DEC runs on the CUDA-core kernels
    assert _scan(lib, mode=1, chunk=64, impl=3) == L.ERR_UNSUPPORTED
    assert _scan(lib, impl=9) == L.ERR_INVALID_ARG
    assert _scan(lib, impl=2) == L.ERR_UNSUPPORTED          # tensor cores need chunk > 1
    assert _scan(lib, chunk=64, impl=2) == L.ERR_UNSUPPORTED  # and bf16 x/q, m,d in {64,128}
    assert _scan(lib, y=(1 << 20) + 64) == L.ERR_INVALID_ARG  # y overlaps x
    assert _scan(lib, So=(5 << 20) + 16) == L.ERR_INVALID_ARG  # partial S0/S_out aliasing
    assert _scan(lib, x=(1 << 20) + 4) == L.ERR_INVALID_ARG   # misaligned x
    v = ctypes.c_void_p
    assert lib.lattice_step(None, v(1 << 20), 0, v(2 << 20), v(3 << 20), 0, v(4 << 20), None,
                            v(5 << 20), 1, 1, 4, 16, 0, None) == L.ERR_INVALID_ARG
    assert lib.lattice_readout(v(1 << 20), v(2 << 20), 0, v(3 << 20), 1, 1, 4, 24,
                               None) == L.ERR_UNSUPPORTED


def _bwd(lib, **kw):
    a = dict(x=1 << 20, xdt=0, c=2 << 20, q=3 << 20, qdt=0, mu=4 << 20, eta=None, S0=5 << 20,
             dy=6 << 20, dST=None, dx=7 << 20, dc=8 << 20, dq=9 << 20, dmu=10 << 20, deta=None,
             dS0=11 << 20, ws=12 << 20, wsb=1 << 20, B=1, T=4, H=1, m=4, d=16, chunk=1, seg=0)
    a.update(kw)
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return lib.lattice_scan_bwd(v(a["x"]), a["xdt"], v(a["c"]), v(a["q"]), a["qdt"], v(a["mu"]),
                                v(a["eta"]), v(a["S0"]), v(a["dy"]), v(a["dST"]), v(a["dx"]),
                                v(a["dc"]), v(a["dq"]), v(a["dmu"]), v(a["deta"]), v(a["dS0"]),
                                v(a["ws"]), a["wsb"], a["B"], a["T"], a["H"], a["m"], a["d"],
                                a["chunk"], a["seg"], None)


def test_backward_workspace_and_argument_checks(lib):
    # workspace: B*H*(n_seg - 1 + seg)*m*d*4 bytes; the default segment is the
    # smallest multiple of the chunk size that is >= 64 tokens
    ws = lib.lattice_scan_bwd_workspace_bytes
    assert ws(1, 4, 1, 4, 16, 1, 0) == 64 * 4 * 16 * 4
    assert ws(2, 200, 3, 4, 16, 1, 0) == 2 * 3 * (3 + 64) * 4 * 16 * 4
    assert ws(1, 200, 1, 4, 16, 24, 0) == (2 + 72) * 4 * 16 * 4
    assert ws(1, 200, 1, 4, 16, 128, 0) == (1 + 128) * 4 * 16 * 4
    assert ws(1, 200, 1, 4, 16, 4, 10) == 0      # segment not a multiple of the chunk
    # one sequence on a 148-SM device: a cluster of G CTAs, each with ceil(m/G) scratch rows
    assert ws(1, 200, 1, 64, 16, 1, 0) == 4 * (3 + 64) * 16 * 16 * 4     # G = 4, 16 rows each
    assert ws(1, 200, 1, 5, 16, 1, 0) == 2 * (3 + 64) * 3 * 16 * 4       # G = 2, 3 rows each (one unused)
    assert ws(100, 200, 1, 64, 16, 1, 0) == 100 * (3 + 64) * 64 * 16 * 4  # batch fills the SMs: G = 1
    assert ws(1, 200, 1, 129, 16, 1, 0) == 0     # m > 128
    # chunks of 2..64 at d >= 32 may run the chunk-parallel kernel: the workspace covers
    # both kernels, its own term being ceil(m/16) CTAs x ceil(T/C) chunk-start states
    tok = 4 * (3 + 64) * 10 * 64 * 4                        # G = 4, 10 rows each, seg 64
    assert ws(1, 200, 1, 40, 64, 16, 0) == max(tok, 3 * 13 * 16 * 64 * 4) == tok
    tok = 4 * (102 + 640) * 16 * 128 * 4                    # seg 640: 103 segments
    cb = 4 * 1024 * 16 * 128 * 4                            # 1024 chunks of 64
    assert ws(1, 65536, 1, 64, 128, 64, 640) == max(tok, cb) == cb
    # every case below fails validation before any CUDA call
    assert _bwd(lib, wsb=64 * 4 * 16 * 4 - 4) == L.ERR_INVALID_ARG   # workspace too small
    assert _bwd(lib, ws=None) == L.ERR_INVALID_ARG
    assert _bwd(lib, chunk=4, seg=10) == L.ERR_INVALID_ARG
    assert _bwd(lib, m=129) == L.ERR_UNSUPPORTED
    assert _bwd(lib, d=48) == L.ERR_UNSUPPORTED
    assert _bwd(lib, dy=None) == L.ERR_INVALID_ARG
    assert _bwd(lib, dS0=None) == L.ERR_INVALID_ARG
    assert _bwd(lib, dx=(1 << 20) + 16) == L.ERR_INVALID_ARG    # dx overlaps x
    assert _bwd(lib, dc=(7 << 20) + 4) == L.ERR_INVALID_ARG     # dc overlaps dx
    assert _bwd(lib, ws=(11 << 20) + 64) == L.ERR_INVALID_ARG   # workspace overlaps dS0
    assert _bwd(lib, ws=(12 << 20) + 8) == L.ERR_INVALID_ARG    # misaligned workspace


def test_binding_rejects_host_tensors():
    import torch
    x = torch.zeros(1, 2, 1, 16)
    with pytest.raises(TypeError):
        L.scan_fwd(x, torch.zeros(1, 2, 1, 4), torch.zeros(1, 2, 1, 4), torch.zeros(1, 2, 1),
                   torch.zeros(1, 1, 4, 16))


def test_noalloc_backward_rejects_shapes_beyond_its_scratch(lib):
    """lattice_scan_bwd_noalloc: the small training shape's backward workspace (about
    50 MB) fits the library's static 64 MiB scratch array; a shape that needs more is
    refused on the host, before any device work (no CUDA call is made here)."""
    lib.lattice_scan_bwd_noalloc.restype = ctypes.c_int
    assert 0 < lib.lattice_scan_bwd_workspace_bytes(4, 2048, 8, 64, 64, 64, 0) <= 64 << 20
    big = lib.lattice_scan_bwd_workspace_bytes(8, 4096, 16, 128, 128, 64, 0)
    assert big > 64 << 20
    v = ctypes.c_void_p
    code = lib.lattice_scan_bwd_noalloc(v(1 << 20), 0, v(2 << 20), v(3 << 20), 0, v(4 << 20), None,
                                        v(5 << 20), v(6 << 20), None, v(7 << 20), v(8 << 20),
                                        v(9 << 20), v(10 << 20), None, v(11 << 20), 8, 4096, 16, 128,
                                        128, 64, 0, None)
    assert code == L.ERR_UNSUPPORTED
    # rejected arguments are named by the same checks as lattice_scan_bwd's
    code = lib.lattice_scan_bwd_noalloc(v(1 << 20), 0, v(2 << 20), v(3 << 20), 0, v(4 << 20), None,
                                        v(5 << 20), v(6 << 20), None, v(7 << 20), v(8 << 20),
                                        v(9 << 20), v(10 << 20), None, v(11 << 20), 1, 4, 1, 4,
                                        48, 1, 0, None)
    assert code == L.ERR_UNSUPPORTED  # d = 48


def test_bounded_wait_selftest_checks_its_limit(lib):
    # out-of-range limits are refused before any launch (no CUDA call is made here)
    assert lib.lattice_selftest_bounded_wait(0, None) == L.ERR_INVALID_ARG
    assert lib.lattice_selftest_bounded_wait(2_000_000_000, None) == L.ERR_INVALID_ARG
