"""Pins of the gate variants (oracle/gates.py) against what the pages print
and the mathematics fixes, independent of the oracle's own code."""
import json
import os

import numpy as np
from scipy.special import expit

import oracle
from oracle import brute, gates

Z = np.linspace(-6.0, 6.0, 24001)
with open(os.path.join(os.path.dirname(__file__), "golden", "gate_curves_tab3.json")) as f:
    TAB3 = json.load(f)["printed"]


def _alpha_and_slope(gfun):
    a = np.exp(gfun(Z))
    h = 1e-5
    d = (np.exp(gfun(Z + h)) - np.exp(gfun(Z - h))) / (2 * h)
    return a, d


def _v1(z):
    z = np.asarray(z)[..., None, None]
    return gates.softplus_gate(z)[..., 0, 0]


def _v2_floor_001(z):
    z = np.asarray(z)[..., None, None]
    return gates.bounded_gate(z, g_min=np.log(0.01))[..., 0, 0]


def test_tab3_v1_curve():
    """Page "线性注意力交互式演示", Tab 3: v1 alpha falls from ~1.0 at z = -6 to
    ~0 at z = 6; its slope is most negative, ~-0.25, at z ~ 0."""
    a, d = _alpha_and_slope(_v1)
    assert abs(a[0] - TAB3["v1_alpha_at_z_minus6"]) < 0.005
    assert abs(a[-1] - TAB3["v1_alpha_at_z_plus6"]) < 0.005
    assert np.all(np.diff(a) < 0)
    i = d.argmin()
    assert abs(d[i] - TAB3["v1_slope_min"]) < 0.005 and abs(Z[i] - TAB3["v1_slope_min_at_z"]) < 0.05


def test_tab3_v2_curve_with_floor_001():
    """Tab 3 with the floor alpha = 0.01: v2 flattens onto the floor at z = 6,
    never crosses it, and its slope is most negative, ~-0.29, near z ~ -1.5."""
    a, d = _alpha_and_slope(_v2_floor_001)
    floor = TAB3["v2_floor_alpha"]
    assert np.all(a > floor) and abs(a[-1] - floor) < 5e-4
    i = d.argmin()
    assert abs(d[i] - TAB3["v2_slope_min"]) < 0.01 and abs(Z[i] - TAB3["v2_slope_min_at_z"]) < 0.5
    # v1 goes below the floor, v2 does not (the two separate for z > 0)
    a1, _ = _alpha_and_slope(_v1)
    assert a1[-1] < 0.01 < a[-1]


def test_k3_bounded_range_and_midpoint():
    """Page "Implémenter KDA", "La décroissance bornée": g in (g_min, 0), alpha
    in (e^-5, 1); at exp(A_log)(z + dt_bias) = 0 the gate is g_min / 2."""
    r = np.random.default_rng(0)
    z = 20 * r.standard_normal((7, 3, 5))
    A = r.standard_normal(3); dt = r.standard_normal((3, 5))
    g = gates.bounded_gate(z, A, dt)
    assert np.all(g >= -5.0) and np.all(g <= 0.0)          # saturates to the ends in fp64
    g = gates.bounded_gate(z / 10, A, dt)
    assert np.all(g > -5.0) and np.all(g < 0.0)
    assert np.allclose(gates.bounded_gate(-dt[None], A, dt), -2.5, rtol=0, atol=1e-15)


def test_softplus_gate_closed_forms():
    """-exp(A) softplus(z + b): -ln 2 exp(A) at z = -b, -> -exp(A) z for large z,
    -> 0 for very negative z, and scales linearly in exp(A_log)."""
    A = np.array([0.0, np.log(3.0)])
    dt = np.array([[0.5], [-1.0]])
    g0 = gates.softplus_gate(-dt[None], A, dt)
    assert np.allclose(g0[0, :, 0], -np.log(2.0) * np.exp(A), rtol=1e-15)
    big = gates.softplus_gate(np.full((1, 2, 1), 800.0), A, dt)
    assert np.allclose(big[0, :, 0], -np.exp(A) * (800.0 + dt[:, 0]), rtol=1e-15)
    assert np.all(np.isfinite(big))
    small = gates.softplus_gate(np.full((1, 2, 1), -800.0), A, dt)
    assert np.all(small <= 0.0) and np.all(small > -1e-300)


def test_gdn_gate_is_log_sigmoid():
    """Gated DeltaNet (Eq. 6): alpha = sigmoid(z), checked against SciPy's expit."""
    z = np.linspace(-30, 30, 601)
    assert np.allclose(np.exp(gates.gdn_gate(z)), expit(z), rtol=1e-14, atol=0)
    assert np.all(np.isfinite(gates.gdn_gate(np.array([-1e4, 1e4]))))


def test_unbounded_gate_overflows_a_float32_chunk_factor():
    """Page "KDA 模块交互式演示", the chunk-overflow tab: within a 16-token chunk
    the retention factor 1/gamma = exp(-sum g) stays finite in float32 for the
    bounded gate (|sum g| <= 80 < ln(FLT_MAX) ~ 88.7) but overflows, for all
    but a tail of draws, for the softplus gate driven at z + 6."""
    r = np.random.default_rng(1)
    z = r.standard_normal((1000, 16, 1, 1))
    gb = gates.bounded_gate(z + 6.0)
    gs = gates.softplus_gate(z + 6.0)
    with np.errstate(over="ignore"):
        fb = np.exp(-gb.sum(1)).astype(np.float32)
        fs = np.exp(-gs.sum(1)).astype(np.float32)
    assert np.all(np.isfinite(fb))
    assert np.mean(np.isinf(fs)) > 0.9      # sum of 16 softplus(z + 6) ~ 96 +- 4 > 88.7


def test_scalar_gate_keeps_the_delta_overwrite():
    """Page "线性注意力交互式演示", Delta Rule: with beta = 1 and a unit key the
    state read back along that key equals the latest write, whatever the
    (scalar) decay of Gated DeltaNet."""
    r = np.random.default_rng(2)
    T, Dk, Dv = 9, 6, 4
    k = r.standard_normal(Dk); k /= np.linalg.norm(k)
    K = np.tile(k, (T, 1))
    V = r.standard_normal((T, Dv))
    g = gates.broadcast_channels(gates.gdn_gate(r.standard_normal(T)), Dk)
    _, S, _ = brute.affine_run(K, K, V, g, np.ones(T), S0=r.standard_normal((Dk, Dv)))
    assert np.allclose(S.T @ k, V[-1], rtol=1e-12, atol=1e-12)


def test_broadcast_scalar_gate_matches_the_c_oracle_per_channel_run():
    """A per-head decay broadcast over Dk through the C oracle equals the dense
    affine product with the scalar decay matrix alpha I."""
    r = np.random.default_rng(3)
    T, Dk, Dv = 11, 5, 3
    q = r.standard_normal((1, T, 1, Dk)); k = r.standard_normal((1, T, 1, Dk))
    v = r.standard_normal((1, T, 1, Dv)); beta = r.uniform(0, 1, (1, T, 1))
    gh = gates.gdn_gate(r.standard_normal((1, T, 1)))
    f = oracle.kda_fwd(q, k, v, gates.broadcast_channels(gh, Dk), beta,
                       qk_l2norm=False, beta_sigmoid=False, gate_in=False)
    S = np.zeros((Dk, Dv))
    for t in range(T):
        a = np.exp(gh[0, t, 0])
        kt = k[0, t, 0]
        S = (np.eye(Dk) - beta[0, t, 0] * np.outer(kt, kt)) @ (a * S) + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
    assert np.allclose(f["S_T"][0, 0], S, rtol=1e-12, atol=1e-12)
