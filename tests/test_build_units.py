"""The library's build: one translation unit per kernel family (csrc/tu_*.cu) plus the
C ABI, compiled whole and linked into one shared library. Each unit is a module of its
own on the device, with its own copy of the device status word, so the ABI must read
every unit's copy. These checks need no GPU."""
import glob
import os
import re

from orthogonal_update_recurrent_b200 import build

CSRC = build.CSRC


def test_every_unit_is_built():
    units = {os.path.basename(p) for p in glob.glob(os.path.join(CSRC, "*.cu"))}
    assert units == set(build.UNITS)
    assert "lattice_abi.cu" in units


def test_no_split_compilation():
    # split compilation gave different register allocations (and spills) from build to build
    flags = " ".join(build.COMPILE_FLAGS + build.LINK_FLAGS)
    assert "split-compile" not in flags
    assert "arch=compute_100a,code=sm_100a" in flags


def test_device_status_is_read_from_every_unit():
    with open(os.path.join(CSRC, "launch.h")) as f:
        declared = set(re.findall(r"cudaError_t (status_\w+)\(unsigned int\* v\);", f.read()))
    defined = set()
    for p in glob.glob(os.path.join(CSRC, "tu_*.cu")):
        with open(p) as f:
            found = re.findall(r"cudaError_t (status_\w+)\(unsigned int\* v\) \{ return read_clear_module_status\(v\); \}",
                               f.read())
        assert len(found) == 1, p  # each unit reads its own copy
        defined |= set(found)
    assert declared == defined
    with open(os.path.join(CSRC, "lattice_abi.cu")) as f:
        abi = f.read()
    body = abi[abi.index("lattice_status lattice_get_device_status("):]
    body = body[:body.index("\n}\n")]
    assert "read_clear_module_status" in body  # the ABI unit's own copy (the self-test kernel)
    for name in declared:
        assert name in body, name
