"""Pins of the FP64 oracle to facts the pages and the mathematics fix.

Each test cites the passage it checks.  None of them re-types the oracle's own
formula: they use special cases with closed forms, an independent dense
restatement (oracle.brute), the chunk-parallel form (oracle.chunkwise), library
routines (scipy.special.expit, numpy.linalg.norm) and identities.
"""
import json
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle
from oracle import brute, chunkwise

RNG = np.random.default_rng(12345)
with open(os.path.join(os.path.dirname(__file__), "golden", "composition_tests.json")) as _f:
    COMPOSITION = json.load(_f)


def _chain(T, Dk, Dv, rng, g_lo=-5.0, g_hi=0.0, unit_keys=True):
    q = rng.standard_normal((T, Dk))
    k = rng.standard_normal((T, Dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, Dv))
    g = rng.uniform(g_lo, g_hi, (T, Dk))
    beta = rng.uniform(0.0, 1.0, T)
    return q, k, v, g, beta


def _run(q, k, v, g, beta, S0=None, want_M=False, scale=1.0):
    """C oracle on one chain with all switches off (inputs used as given)."""
    out = oracle.kda_fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                         g[None, :, None], beta[None, :, None],
                         S0=None if S0 is None else S0[None, None], scale=scale,
                         qk_l2norm=False, beta_sigmoid=False, gate_in=False,
                         want_M=want_M)
    o = out["o"][0, :, 0]
    S = out["S_T"][0, 0]
    M = out["M_T"][0, 0] if want_M else None
    return o, S, M


# ---------------------------------------------------------------------------
# Page "Implémenter KDA", "Test 1 - comportements limites".
# ---------------------------------------------------------------------------
def test_beta_zero_is_pure_decay():
    Dk, Dv = 7, 5
    S = RNG.standard_normal((Dk, Dv))
    q, k, v, g, _ = _chain(1, Dk, Dv, RNG)
    beta = np.zeros(1)
    o, S1, _ = _run(q, k, v, g, beta, S0=S)
    alpha = np.exp(g[0])
    np.testing.assert_array_equal(S1, alpha[:, None] * S)
    np.testing.assert_allclose(o[0], (alpha[:, None] * S).T @ q[0], rtol=0, atol=1e-14)


def test_alpha_one_beta_one_recalls_value_exactly():
    Dk, Dv = 8, 6
    q, k, v, _, _ = _chain(1, Dk, Dv, RNG)
    g = np.zeros((1, Dk))
    beta = np.ones(1)
    # From zero (the page's case) and from an arbitrary state (stronger form:
    # with |k| = 1 the erase removes exactly what S held along k).
    for S0 in (np.zeros((Dk, Dv)), RNG.standard_normal((Dk, Dv))):
        _, S1, _ = _run(q, k, v, g, beta, S0=S0)
        np.testing.assert_allclose(S1.T @ k[0], v[0], rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Page "Implémenter KDA", "Trois pièges": the output reads the state AFTER the
# update.  With S0 = 0 and one token, o = S_1^T q = beta (k.q) v.
# ---------------------------------------------------------------------------
def test_output_reads_updated_state():
    Dk, Dv = 6, 4
    q, k, v, g, beta = _chain(1, Dk, Dv, RNG)
    o, _, _ = _run(q, k, v, g, beta)
    np.testing.assert_allclose(o[0], beta[0] * (k[0] @ q[0]) * v[0], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Worked cases with orthogonal keys, solvable by hand (page "KDA 模块交互式演示"
# section 1.3: the delta rule writes only the error between the value and what
# the key currently retrieves).
# ---------------------------------------------------------------------------
def test_hand_worked_orthogonal_keys_and_channel_decay():
    Dk, Dv = 2, 2
    e1, e2 = np.eye(2)
    v1, v2 = np.array([2.0, 3.0]), np.array([-1.0, 4.0])
    q = np.stack([e1, e1 + e2])
    k = np.stack([e1, e2])
    v = np.stack([v1, v2])
    a = np.array([0.25, 0.5])                 # channel decays of token 2
    g = np.stack([np.zeros(2), np.log(a)])
    beta = np.array([0.5, 0.75])
    o, S, _ = _run(q, k, v, g, beta)
    # token 1: S1 = 0.5 e1 v1^T ; o1 = S1^T e1 = 0.5 v1
    np.testing.assert_allclose(o[0], 0.5 * v1, atol=1e-15)
    # token 2: decay scales row 1 by 0.25; e2 is orthogonal to the stored key,
    # so the erase along e2 removes nothing: S2 = 0.125 e1 v1^T + 0.75 e2 v2^T
    S2 = 0.125 * np.outer(e1, v1) + 0.75 * np.outer(e2, v2)
    np.testing.assert_allclose(S, S2, atol=1e-15)
    np.testing.assert_allclose(o[1], 0.125 * v1 + 0.75 * v2, atol=1e-15)


def test_hand_worked_same_key_overwrites():
    e1 = np.array([1.0, 0.0, 0.0])
    v1, v2 = np.array([1.0, -2.0]), np.array([3.0, 5.0])
    q = np.stack([e1, e1])
    k = np.stack([e1, e1])
    v = np.stack([v1, v2])
    g = np.zeros((2, 3))
    # beta = 1: the second write replaces the first (page "线性注意力交互式演示",
    # Delta Rule key property with alpha=1, beta=1 and the same key).
    o, S, _ = _run(q, k, v, g, np.ones(2))
    np.testing.assert_allclose(o[1], v2, atol=1e-15)
    np.testing.assert_allclose(S, np.outer(e1, v2), atol=1e-15)
    # beta = 1/2: S1 = e1 (v1/2)^T, S2 = S1 + (1/2) e1 (v2 - v1/2)^T = e1 (v1/4 + v2/2)^T
    o, S, _ = _run(q, k, v, g, np.full(2, 0.5))
    np.testing.assert_allclose(S, np.outer(e1, 0.25 * v1 + 0.5 * v2), atol=1e-15)
    np.testing.assert_allclose(o[1], 0.25 * v1 + 0.5 * v2, atol=1e-15)


# ---------------------------------------------------------------------------
# Brute force on tiny shapes: the explicit dense affine product (independent
# restatement with P5's transition matrix M_t = (I - beta k k^T) Diag(alpha)).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,Dk,Dv", [(1, 1, 1), (3, 2, 3), (6, 4, 2), (8, 3, 4)])
def test_brute_force_affine_product(T, Dk, Dv):
    rng = np.random.default_rng(100 + T * 10 + Dk)
    q, k, v, g, beta = _chain(T, Dk, Dv, rng)
    S0 = rng.standard_normal((Dk, Dv))
    o, S, M = _run(q, k, v, g, beta, S0=S0, want_M=True, scale=0.7)
    ob, Sb, Mb = brute.affine_run(q, k, v, g, beta, S0=S0, scale=0.7)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(S, Sb, rtol=0, atol=1e-13)
    np.testing.assert_allclose(M, Mb, rtol=0, atol=1e-13)


def test_brute_force_rejects_erase_before_decay():
    """The order of operations matters (page "Implémenter KDA", "Trois pièges"):
    Diag(alpha)(I - beta k k^T) would give a different map than the oracle."""
    rng = np.random.default_rng(7)
    q, k, v, g, beta = _chain(4, 3, 2, rng)
    S0 = rng.standard_normal((3, 2))
    _, S, _ = _run(q, k, v, g, beta, S0=S0)
    Sw = S0.copy()
    for t in range(4):
        Mw = np.diag(np.exp(g[t])) @ (np.eye(3) - beta[t] * np.outer(k[t], k[t]))
        Sw = Mw @ Sw + beta[t] * np.outer(k[t], v[t])
    assert np.max(np.abs(S - Sw)) > 1e-3


# ---------------------------------------------------------------------------
# Page "Implémenter KDA", "Test 2 - l'identité de composition": run(S0) equals
# M S0 + run(0) (printed error 6.94e-18, tolerance 1e-9).
# ---------------------------------------------------------------------------
def test_kcp_composition_identity():
    rng = np.random.default_rng(2)
    T, Dk, Dv = 48, 12, 9
    q, k, v, g, beta = _chain(T, Dk, Dv, rng, g_lo=-0.1)
    beta *= 0.3
    S0 = rng.standard_normal((Dk, Dv))
    o_direct, S_direct, M = _run(q, k, v, g, beta, S0=S0, want_M=True)
    _, S_zero, _ = _run(q, k, v, g, beta)
    err = np.max(np.abs(S_direct - (S_zero + M @ S0)))
    assert err < COMPOSITION["asserted_bound"] and err < 1e-12
    # M is the product of the page's transition matrices, newest on the left.
    Md = np.eye(Dk)
    for t in range(T):
        Md = brute.transition(k[t], np.exp(g[t]), beta[t]) @ Md
    np.testing.assert_allclose(M, Md, rtol=0, atol=1e-12)
    # The decay is slow enough that M is far from zero, so the identity is not vacuous.
    assert np.abs(M).max() > 1e-3


# ---------------------------------------------------------------------------
# Page "Implémenter KDA", "Test 3 - le balayage préfixe sur plusieurs rangs":
# four segments run from zero, combined by S <- M S + S_local (printed error
# 1.39e-17 on 4 ranks, tolerance 1e-9).
# ---------------------------------------------------------------------------
def test_prefix_scan_over_segments_matches_full_run():
    rng = np.random.default_rng(3)
    T, Dk, Dv, nseg = 64, 8, 8, 4
    q, k, v, g, beta = _chain(T, Dk, Dv, rng, g_lo=-0.1)
    beta *= 0.3
    S_init = rng.standard_normal((Dk, Dv))
    _, S_full, _ = _run(q, k, v, g, beta, S0=S_init)
    L = T // nseg
    Ms, Ss = [], []
    for s in range(nseg):
        sl = slice(s * L, (s + 1) * L)
        _, S_loc, M_loc = _run(q[sl], k[sl], v[sl], g[sl], beta[sl], want_M=True)
        Ms.append(M_loc)
        Ss.append(S_loc)
    S_in = oracle.kda_compose(np.stack(Ms)[:, None], np.stack(Ss)[:, None], S_init[None])
    err = np.max(np.abs(S_in[-1, 0] - S_full))
    assert err < COMPOSITION["asserted_bound"] and err < 1e-12
    # Every intermediate entry is the state at that segment boundary.
    for s in range(1, nseg):
        _, S_b, _ = _run(q[: s * L], k[: s * L], v[: s * L], g[: s * L], beta[: s * L], S0=S_init)
        assert np.max(np.abs(S_in[s, 0] - S_b)) < 1e-12


def test_compose_is_associative():
    """Page "Implémenter KDA", "La loi de composition associative": combining
    (M2,S2) after (M1,S1) equals combining with the pair (M2 M1, M2 S1 + S2)."""
    rng = np.random.default_rng(4)
    Dk, Dv = 5, 3
    M1, M2 = rng.standard_normal((2, Dk, Dk)) * 0.5
    S1, S2, S0 = rng.standard_normal((3, Dk, Dv))
    seq = oracle.kda_compose(np.stack([M1, M2])[:, None], np.stack([S1, S2])[:, None], S0[None])
    pair = oracle.kda_compose((M2 @ M1)[None, None], (M2 @ S1 + S2)[None, None], S0[None])
    np.testing.assert_allclose(seq[-1], pair[-1], rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Page "KDA 模块交互式演示" Tab 8 (recurrent vs chunkwise, max error ~1e-16 in
# fp64, threshold 1e-10) and section 1.5 Eqs. 3-4.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
@pytest.mark.parametrize("T", [1, 50, 128])
def test_chunkwise_form_equals_recurrence(chunk, T):
    rng = np.random.default_rng(chunk * 1000 + T)
    Dk, Dv = 16, 12
    q, k, v, g, beta = _chain(T, Dk, Dv, rng)       # fast decay: G reaches about -5*chunk
    S0 = rng.standard_normal((Dk, Dv)) * 0.1
    o, S, M = _run(q, k, v, g, beta, S0=S0, want_M=True)
    oc, Sc, Mc = chunkwise.chunk_run(q, k, v, g, beta, S0=S0, chunk=chunk)
    assert np.max(np.abs(o - oc)) < 1e-10
    assert np.max(np.abs(S - Sc)) < 1e-10
    assert np.max(np.abs(M - Mc)) < 1e-10


def test_chunkwise_literal_print_needs_decay_weighting():
    """The page prints the UT matrix as tril(Diag(beta) K K^T, -1).  Taken
    literally it matches the recurrence only without decay; with decay the
    Gamma-weighted matrix is the one that matches (the class of error the
    linear-attention page reports as a 0.812 recurrent/chunk mismatch)."""
    rng = np.random.default_rng(5)
    T, Dk, Dv = 64, 8, 8
    q, k, v, g, beta = _chain(T, Dk, Dv, rng, g_lo=-1.0)
    o, _, _ = _run(q, k, v, g, beta)
    o_lit, _, _ = chunkwise.chunk_run(q, k, v, g, beta, chunk=16, ut_with_decay=False)
    assert np.max(np.abs(o - o_lit)) > 1e-3
    g0 = np.zeros_like(g)
    o0, _, _ = _run(q, k, v, g0, beta)
    o0_lit, _, _ = chunkwise.chunk_run(q, k, v, g0, beta, chunk=16, ut_with_decay=False)
    assert np.max(np.abs(o0 - o0_lit)) < 1e-10


# ---------------------------------------------------------------------------
# The three in-kernel switches (page "KDAAttention 层", "chunk_kda 内部做了什么")
# against library routines, and the bounded gate (page "KDA 模块交互式演示"
# section 1.4 Eq. 5; page "Implémenter KDA", "La décroissance bornée").
# ---------------------------------------------------------------------------
def test_switches_match_library_preprocessing():
    rng = np.random.default_rng(6)
    B, T, H, HV, Dk, Dv = 2, 9, 2, 4, 8, 5
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, HV, Dv))
    z = rng.standard_normal((B, T, HV, Dk)) * 2
    bl = rng.standard_normal((B, T, HV))
    A_log = rng.uniform(-1, 1, HV)
    dt_bias = rng.standard_normal((HV, Dk)) * 0.5
    S0 = rng.standard_normal((B, HV, Dk, Dv)) * 0.1
    eps = 1e-6
    on = oracle.kda_fwd(q, k, v, z, bl, A_log=A_log, dt_bias=dt_bias, S0=S0, l2_eps=eps)
    qn = q / np.sqrt(np.linalg.norm(q, axis=-1, keepdims=True) ** 2 + eps)
    kn = k / np.sqrt(np.linalg.norm(k, axis=-1, keepdims=True) ** 2 + eps)
    g = -5.0 * expit(np.exp(A_log)[None, None, :, None] * (z + dt_bias[None, None]))
    off = oracle.kda_fwd(qn, kn, v, g, expit(bl), S0=S0,
                         qk_l2norm=False, beta_sigmoid=False, gate_in=False)
    np.testing.assert_allclose(on["o"], off["o"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(on["S_T"], off["S_T"], rtol=0, atol=1e-13)


def _decay_product(z, A_log=0.0, g_min=-5.0):
    """prod_t alpha_t per channel, read back from the oracle: with beta = 0 and
    S0 = I the state after T tokens is Diag(prod alpha)."""
    T, Dk = z.shape
    q = np.ones((1, T, 1, Dk))
    k = np.ones((1, T, 1, Dk))
    v = np.zeros((1, T, 1, Dk))
    bl = np.full((1, T, 1), -np.inf)            # sigmoid(-inf) = 0
    out = oracle.kda_fwd(q, k, v, z[None, :, None], bl, A_log=np.array([A_log]),
                         S0=np.eye(Dk)[None, None], g_min=g_min)
    return np.diag(out["S_T"][0, 0])


def test_bounded_gate_range_and_special_values():
    # z = 0: sigmoid = 1/2, g = g_min/2 exactly.
    np.testing.assert_allclose(_decay_product(np.zeros((1, 3))), np.exp(-2.5), rtol=1e-15)
    # z -> +inf: g -> g_min; over a 16-token tile 1/gamma reaches its bound e^80
    # (page "Implémenter KDA": 16 x 5 = 80, e^80 ~ 5.5e34 < 3e38).
    gam = _decay_product(np.full((16, 4), 1e4))
    np.testing.assert_allclose(gam, np.exp(-80.0), rtol=1e-13)
    assert 1.0 / gam.min() < 3.0e38
    # z -> -inf: g -> 0, alpha -> 1 (no forgetting)
    np.testing.assert_allclose(_decay_product(np.full((5, 2), -1e4)), 1.0, rtol=0, atol=1e-300)
    # Any finite z keeps alpha inside (e^g_min, 1): 1/gamma of a random tile is
    # finite and below e^80.
    z = RNG.standard_normal((16, 64)) * 3
    gam = _decay_product(z, A_log=0.7)
    assert np.all(gam > np.exp(-80.0)) and np.all(gam < 1.0)
    # exp(A_log) scales the gate input: A_log = log 2 with z equals A_log = 0 with 2z.
    np.testing.assert_allclose(_decay_product(z[:3], A_log=np.log(2.0)),
                               _decay_product(2 * z[:3]), rtol=1e-13)


# ---------------------------------------------------------------------------
# Grouped value heads: value head hv reads q/k head hv // (HV/H); equivalently
# the q/k heads repeated per group with HV == H.
# ---------------------------------------------------------------------------
def test_grouped_value_heads_mapping():
    rng = np.random.default_rng(8)
    B, T, H, HV, Dk, Dv = 1, 12, 2, 6, 4, 3
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, HV, Dv))
    z = rng.standard_normal((B, T, HV, Dk))
    bl = rng.standard_normal((B, T, HV))
    A_log = np.zeros(HV)
    grouped = oracle.kda_fwd(q, k, v, z, bl, A_log=A_log)
    rep = HV // H
    expanded = oracle.kda_fwd(np.repeat(q, rep, axis=2), np.repeat(k, rep, axis=2), v, z, bl,
                              A_log=A_log)
    np.testing.assert_array_equal(grouped["o"], expanded["o"])
    np.testing.assert_array_equal(grouped["S_T"], expanded["S_T"])


# ---------------------------------------------------------------------------
# Decode: one kda_step per token reproduces the sequence forward (page "KDA
# 模块交互式演示", Tab 13 "单步匹配递推").
# ---------------------------------------------------------------------------
def test_step_matches_sequence():
    rng = np.random.default_rng(9)
    B, T, H, HV, Dk, Dv = 2, 7, 1, 2, 6, 5
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, HV, Dv))
    z = rng.standard_normal((B, T, HV, Dk))
    bl = rng.standard_normal((B, T, HV))
    A_log = rng.uniform(-1, 1, HV)
    S0 = rng.standard_normal((B, HV, Dk, Dv))
    full = oracle.kda_fwd(q, k, v, z, bl, A_log=A_log, S0=S0)
    S = S0
    for t in range(T):
        S, o = oracle.kda_step(S, q[:, t], k[:, t], v[:, t], z[:, t], bl[:, t], A_log=A_log)
        np.testing.assert_allclose(o, full["o"][:, t], rtol=0, atol=1e-13)
    np.testing.assert_allclose(S, full["S_T"], rtol=0, atol=1e-13)


def test_linear_in_values_and_initial_state():
    """The map (V, S0) -> (O, S_T) is linear for fixed keys and gates."""
    rng = np.random.default_rng(10)
    T, Dk, Dv = 20, 5, 4
    q, k, v, g, beta = _chain(T, Dk, Dv, rng)
    S0 = rng.standard_normal((Dk, Dv))
    v2 = rng.standard_normal((T, Dv))
    S02 = rng.standard_normal((Dk, Dv))
    o1, s1, _ = _run(q, k, v, g, beta, S0=S0)
    o2, s2, _ = _run(q, k, v2, g, beta, S0=S02)
    o3, s3, _ = _run(q, k, 2 * v - 3 * v2, g, beta, S0=2 * S0 - 3 * S02)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s3, 2 * s1 - 3 * s2, rtol=0, atol=1e-12)


def test_empty_sequence_returns_initial_state():
    Dk, Dv = 4, 3
    S0 = RNG.standard_normal((1, 1, Dk, Dv))
    e = np.zeros((1, 0, 1, Dk))
    out = oracle.kda_fwd(e, e, np.zeros((1, 0, 1, Dv)), e, np.zeros((1, 0, 1)),
                         A_log=np.zeros(1), S0=S0, want_M=True)
    np.testing.assert_array_equal(out["S_T"], S0)
    np.testing.assert_array_equal(out["M_T"][0, 0], np.eye(Dk))
