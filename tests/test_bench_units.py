"""The algorithmic work and bytes behind bench.py's rates and roofline fractions, pinned to
hand counts (CPU only).

Prefill: per chunk of l tokens the causal triangle has l (l + 1) / 2 entries; C B^T is
formed once per group (N terms each), its masked product with X once per head (P terms),
the chunk state and the state-to-output term are P N per token and head, and the chunk
recurrence P N per chunk and head; every multiply-add is 2 FLOPs.  Bytes: x and y (io
dtype), B and C (io dtype), dt (fp32), h0 and h_final (fp32), A and D (fp32).
Decode: every layer's fp32 state is read and written, the conv window (fp32, k - 1 taps)
read and written, the step's inputs and y (io dtype) and dt moved once, the weights read.
"""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_units", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_prefill_flops_by_hand(bench):
    # one chunk of 4 tokens, one head and group, P = N = 1: triangle 10 entries
    assert bench.prefill_flops(1, 4, 1, 1, 1, 1, 4) == 2 * 10 + 2 * 10 + 2 * 4 + 2 * 4 + 2 * 1
    # ragged: T = 6 at L = 4 -> chunks of 4 and 2 -> triangle 10 + 3
    assert bench.prefill_flops(1, 6, 1, 1, 1, 1, 4) == 2 * 13 + 2 * 13 + 2 * 6 + 2 * 6 + 2 * 2


def test_prefill_work_at_the_configurations(bench):
    # the 2.7B-layer shape: 130.3 GFLOP at L = 256, 108.4 GFLOP for the 128-token chunks
    # the tensor-core kernel evaluates; 740.3 MB of algorithmic bytes with h0 and h_final
    f256 = bench.prefill_flops(8, 4096, 80, 64, 128, 1, 256)
    f128 = bench.prefill_flops(8, 4096, 80, 64, 128, 1, 128)
    assert abs(f256 / 1e9 - 130.3) < 0.05 and abs(f128 / 1e9 - 108.4) < 0.05
    assert bench.prefill_bytes(8, 4096, 80, 64, 128, 1) == 740295296.0
    tok = 8 * 4096
    assert bench.prefill_bytes(8, 4096, 80, 64, 128, 1) == (
        tok * 80 * 64 * 2 * 2 + tok * 128 * 2 * 2 + tok * 80 * 4 + 8 * 80 * 64 * 128 * 4 * 2 + 2 * 80 * 4)
    # the long-context shape (no h0): 1634.2 MB
    assert abs(bench.prefill_bytes(1, 65536, 80, 64, 128, 8, with_h0=False) / 1e6 - 1634.2) < 0.05


def test_decode_bytes_at_the_cache_shape(bench):
    # 64 layers, 80 x 64 x 128 state, width-4 conv over 5376 channels: 352.1 MB per step at
    # batch 1, 11.05 GB at batch 32 (the state alone is 335.5 MB per sequence)
    b1 = bench.decode_bytes_per_step(64, 1, 80, 64, 128, 1)
    b32 = bench.decode_bytes_per_step(64, 32, 80, 64, 128, 1)
    assert abs(b1 / 1e6 - 352.1) < 0.05
    assert abs(b32 / 1e9 - 11.05) < 0.005
    state = 2 * 64 * 80 * 64 * 128 * 4
    assert abs(state / 1e6 - 335.5) < 0.05 and b1 > state
