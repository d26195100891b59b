"""Pins of the layer prologue / epilogue oracle (oracle/layer.py) against what
the pages and the mathematics fix, each independent of the oracle's own code."""
import numpy as np
from scipy.special import expit

from oracle import layer

RNG = np.random.default_rng(11)


def test_identity_initialisation_is_a_no_op():
    """Page "KDA 模块交互式演示" 1.1: weight[:, -1] = 1, others 0, is a no-op."""
    x = RNG.standard_normal((2, 9, 8))
    w = np.zeros((8, 4)); w[:, -1] = 1.0
    u, _ = layer.short_conv(x, w)
    assert np.array_equal(u, x)


def test_hand_worked_taps_and_zero_padding():
    """One channel, K = 4, x = 1..5: u[t] = sum_j w[j] x[t-3+j], zeros before t = 0."""
    x = np.arange(1.0, 6.0).reshape(1, 5, 1)
    w = np.array([[10.0, 100.0, 1000.0, 1.0]])
    u, st = layer.short_conv(x, w, bias=np.array([0.5]))
    expect = [1 + 0.5, 2 + 1000 * 1 + 0.5, 3 + 1000 * 2 + 100 * 1 + 0.5,
              4 + 1000 * 3 + 100 * 2 + 10 * 1 + 0.5, 5 + 1000 * 4 + 100 * 3 + 10 * 2 + 0.5]
    assert np.allclose(u[0, :, 0], expect, rtol=0, atol=1e-12)
    assert np.array_equal(st[0, :, 0], [3.0, 4.0, 5.0])


def test_causal():
    x = RNG.standard_normal((1, 12, 4)); w = RNG.standard_normal((4, 4))
    x2 = x.copy(); x2[:, 7:] += 3.0
    u1, _ = layer.short_conv(x, w); u2, _ = layer.short_conv(x2, w)
    assert np.array_equal(u1[:, :7], u2[:, :7]) and not np.allclose(u1[:, 7:], u2[:, 7:])


def test_pieces_with_carried_window_equal_one_run():
    """Page 1.1, decode: a K-1 sliding window makes piecewise runs exact."""
    x = RNG.standard_normal((2, 11, 6)); w = RNG.standard_normal((6, 4)); b = RNG.standard_normal(6)
    u, st = layer.short_conv(x, w, b)
    parts, state = [], None
    for lo, hi in [(0, 1), (1, 2), (2, 7), (7, 11)]:
        up, state = layer.short_conv(x[:, lo:hi], w, b, state)
        parts.append(up)
    assert np.allclose(np.concatenate(parts, axis=1), u, atol=1e-13) and np.allclose(state, st)


def test_silu_and_head_norm():
    u = RNG.standard_normal(1000) * 4
    assert np.allclose(layer.silu(u), u * expit(u), rtol=1e-13)
    y = layer.l2norm_heads(RNG.standard_normal((3, 256)), 128, eps=0.0)
    assert np.allclose(np.linalg.norm(y.reshape(3, 2, 128), axis=-1), 1.0)


def test_output_gate_rms_and_gate():
    o = RNG.standard_normal((5, 3, 128)) * 7
    big = np.full_like(o, 60.0)          # sigmoid -> 1
    y = layer.output_gate(o, big, eps=0.0)
    assert np.allclose(np.sqrt((y * y).mean(axis=-1)), 1.0)
    assert np.allclose(layer.output_gate(3.0 * o, big, eps=0.0), y)          # scale invariant
    half = layer.output_gate(o, np.zeros_like(o), eps=0.0)
    assert np.allclose(half, 0.5 * y)
    w = RNG.standard_normal(128)
    assert np.allclose(layer.output_gate(o, big, w, eps=0.0), y * w)
