"""The algorithmic counts bench.py divides by, checked against figures worked
out independently: the per-token-head FLOP count of the chunk form at
Dk = Dv = 128, C = 64 (98,304 + 40,960 + 1,365 = 140,629), the bytes of the
headline forward (1,026 B per token-head plus the final state once per chain)
and of one decode step (the 512 MiB state read and written, plus the per-token
q, k, v, z, o and beta vectors)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def test_chunk_flops_per_token_head():
    assert bench.chunk_flops_per_token_head(128, 128, 64) == pytest.approx(140629.33, abs=0.01)
    # the three D^2 products alone at C -> 0
    assert bench.chunk_flops_per_token_head(128, 128, 0) == 6 * 128 * 128


def test_headline_forward_bytes():
    w = workloads.workload("gva_bf16")
    per = 256 + 256 + 2 + 256 + 512 / 2        # v, z, beta, o, (q + k) shared by 2 value heads
    expect = w.B * w.T * w.HV * per + w.B * w.HV * 128 * 128 * 4   # + S_T (no S0 in this workload)
    assert bench.chunk_bytes(w) == expect == 1084227584


def test_decode_step_bytes():
    w = workloads.workload("decode_bf16")
    state = 2 * 256 * 32 * 128 * 128 * 4
    assert state == 1073741824
    vec = bench.decode_bytes(w) - state
    # q, k [256, 32, 128]; v, o, z [256, 32, 128]; beta [256, 32]; all bf16
    assert vec == 2 * (2 * 256 * 32 * 128) + 2 * (3 * 256 * 32 * 128) + 2 * 256 * 32 == 10502144
