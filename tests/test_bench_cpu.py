"""The benchmark's arithmetic and its reference arm, on CPU.

The roofline figures bench.py prints divide algorithmic bytes (or flops) by a
measured time, so the byte and flop models are pinned here to values worked out
by hand from the workloads' shapes: per token and head, x and q at their storage
width, c and mu in fp32, y written in fp32; the state read and written once.
"""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import lattice_inputs as LI  # noqa: E402


def test_scan_bytes_per_token_and_head():
    # small training shape: 64*2 (x) + 64*2 (q) + 64*4 (c) + 4 (mu) + 64*4 (y) = 772 B
    w = LI.WORKLOADS["small_train"]
    assert bench.scan_alg_bytes(w) == 4 * 2048 * 8 * 772 + 2 * 4 * 4 * 8 * 64 * 64
    # mid-size layer: 256 + 256 + 512 + 4 + 512 = 1540 B; long context: 256 + 128 + 256 + 4 + 512 = 1156 B
    assert bench.scan_alg_bytes(LI.WORKLOADS["mid_layer"]) == 8 * 4096 * 16 * 1540 + 8 * 8 * 16 * 128 * 128
    assert bench.scan_alg_bytes(LI.WORKLOADS["long_ctx"]) == 65536 * 16 * 1156 + 8 * 16 * 64 * 128


def test_decode_step_bytes():
    # per head: 2 * 4 * m * d state bytes + 128*2 + 128*2 + 128*4 + 4 + 128*4 = 132,612 B
    w = LI.WORKLOADS["decode"]
    assert bench.step_alg_bytes(w) == 256 * 32 * 132612
    assert bench.step_alg_bytes(w) == 1086357504


def test_chunk_mma_flops():
    # 6md + C(m+d) per token and head: 6*64*64 + 64*128 = 32,768 on the small training shape
    w = LI.WORKLOADS["small_train"]
    assert bench.chunk_mma_flops(w, 64) == 4 * 2048 * 8 * 32768
    assert bench.chunk_mma_flops(LI.WORKLOADS["mid_layer"], 64) == 8 * 4096 * 16 * 114688


def test_backward_bytes():
    # reads: x, q (128 + 128 B), c (256 B), mu (4 B), dy (256 B); writes: dx (256 B),
    # dc and dq (2 * 256 B), dmu (4 B): 1544 B per token and head; S0, dS_T, dS0 once
    w = LI.WORKLOADS["small_train"]
    assert bench.bwd_alg_bytes(w) == 4 * 2048 * 8 * 1544 + 3 * 4 * 4 * 8 * 64 * 64


def test_reference_arm_prints_one_contract_line(monkeypatch):
    """Rank 0 of the reference arm times the fp64 oracle on the host cores and prints
    one JSON line with the contract's keys."""
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.main() == 0
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "long_ctx"


def test_bench_rejects_too_few_warmup_steps(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--warmup", "2"])
    with pytest.raises(AssertionError):
        bench.main()


def test_captured_traffic_is_dropped_once_the_kernel_changes(monkeypatch):
    """A DRAM-traffic figure is reported only while the kernel's source file still has
    the hash recorded with its capture; each entry names its profile summary."""
    for (kern, wl), e in bench.CAPTURED_TRAFFIC.items():
        assert os.path.exists(os.path.join(ROOT, e["profile"])), e["profile"]
        expect = e["bytes"] if e["sha"] is not None and bench.source_sha(e["source"]) == e["sha"] else None
        assert bench.traffic_for(kern, wl) == expect
    key = next(iter(bench.CAPTURED_TRAFFIC))
    monkeypatch.setitem(bench.CAPTURED_TRAFFIC, key, dict(bench.CAPTURED_TRAFFIC[key], sha="000000000000"))
    assert bench.traffic_for(*key) is None
    assert bench.traffic_for("no_such_kernel", "small_train") is None


def test_backward_kernel_label_follows_the_dispatch_rule():
    # the library runs the chunk-parallel backward for chunks of 2..64 at d in {32, 64, 128}
    # (16-byte-aligned buffers), and the token-by-token kernel otherwise
    assert bench.bwd_kernel_name(64, 64) == "chunk_bwd_kernel"
    assert bench.bwd_kernel_name(2, 128) == "chunk_bwd_kernel"
    assert bench.bwd_kernel_name(16, 32) == "chunk_bwd_kernel"
    assert bench.bwd_kernel_name(1, 64) == "scan_bwd_kernel<exact>"
    assert bench.bwd_kernel_name(128, 64) == "scan_bwd_kernel<chunked>"
    assert bench.bwd_kernel_name(16, 16) == "scan_bwd_kernel<chunked>"
    # and every workload's backward names a kernel with a captured-traffic entry or none
    for w in ("small_train", "mid_layer"):
        name = bench.bwd_kernel_name(LI.WORKLOADS[w].chunk, LI.WORKLOADS[w].d)
        assert (name, w) in bench.CAPTURED_TRAFFIC
