"""The benchmark's work counts, against figures worked out independently of bench.py.

The forward counts every causal (i, j) pair once: 4d FLOP per query head (QK^T and PV) plus
2d per KV head (the key-key similarity behind the decay); the backward 10d per query head and
6d per KV head.  The totals below for the standard workloads were computed by hand from those
definitions (T(T+1)/2 causal pairs per sequence), as were the transcendental-op counts of the
tensor-core forward (two exp2 and one log2 per decay element, one exp2 per probability)."""
import pytest

import bench
from kv_cache_compression_ua_b200 import inputs as I


@pytest.mark.parametrize("name,gflop", [("prefill_1b", 618.6), ("prefill_1b_16k", 1237.0),
                                        ("fwdbwd_3b", 1924.4)])
def test_forward_flops(name, gflop):
    assert bench.fwd_flops(I.WORKLOADS[name]) / 1e9 == pytest.approx(gflop, abs=0.05)


def test_backward_flops():
    assert bench.bwd_flops(I.WORKLOADS["fwdbwd_3b"]) / 1e9 == pytest.approx(4948.4, abs=0.05)


def test_transcendental_ops_of_the_1b_prefill():
    # 8 sequences x 4096*4097/2 pairs x (3 per KV head x 8 + 1 per query head x 32) = 56 per pair
    w = I.WORKLOADS["prefill_1b"]
    assert bench.mufu_ops(w) == 8 * 4096 * 4097 // 2 * 56


def test_tiny_case_counts_by_enumeration():
    w = I.Workload("t", 2, 5, 4, 2, 8, "f32", 1)
    pairs = sum(1 for i in range(w.T) for j in range(w.T) if j <= i) * w.B
    assert bench.fwd_flops(w) == pairs * (w.H * 4 * w.d + w.Hkv * 2 * w.d)
    assert bench.bwd_flops(w) == pairs * (w.H * 10 * w.d + w.Hkv * 6 * w.d)
    assert bench.mufu_ops(w) == pairs * (3 * w.Hkv + w.H)
