"""Pins of the backward oracle (oracle/backward.py).

The gradient is checked against central finite differences of the C forward
oracle (an independent implementation of the recurrence), and the gradient
w.r.t. the initial state against the closed form dS0 = M_T^T dS_T, M_T being
the cumulative transition the C oracle returns (the state recurrence is
affine in S0: page "Implémenter KDA", the composition test)."""
import numpy as np
import pytest

import oracle
from oracle import backward

RNG = np.random.default_rng(2024)
H_FD = 1e-6


def _inputs(B=1, T=6, H=1, HV=2, Dk=4, Dv=3, seed=0):
    r = np.random.default_rng(seed)
    return dict(
        q=r.standard_normal((B, T, H, Dk)), k=r.standard_normal((B, T, H, Dk)),
        v=r.standard_normal((B, T, HV, Dv)), g=r.standard_normal((B, T, HV, Dk)),
        beta=r.standard_normal((B, T, HV)), A_log=0.3 * r.standard_normal(HV),
        dt_bias=0.5 * r.standard_normal((HV, Dk)), S0=r.standard_normal((B, HV, Dk, Dv)),
    ), r.standard_normal((B, T, HV, Dv)), r.standard_normal((B, HV, Dk, Dv))


def _loss(x, do, dS, **sw):
    f = oracle.kda_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], A_log=x["A_log"],
                       dt_bias=x["dt_bias"], S0=x["S0"], **sw)
    return float((f["o"] * do).sum() + (f["S_T"] * dS).sum())


def _grads(x, do, dS, **sw):
    return backward.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], A_log=x["A_log"],
                                 dt_bias=x["dt_bias"], S0=x["S0"], do=do, dS_T=dS, **sw)


SWITCHES = [
    dict(),
    dict(scale=0.5, g_min=-3.0),
    dict(qk_l2norm=False, beta_sigmoid=False, gate_in=False),
]
_GRAD_NAME = {"q": "q", "k": "k", "v": "v", "g": "g", "beta": "beta", "S0": "S0",
              "A_log": "A_log", "dt_bias": "dt_bias"}


@pytest.mark.parametrize("sw", SWITCHES, ids=["default", "scaled", "switches_off"])
def test_directional_derivatives_match_finite_differences(sw):
    """<grad_X, U> equals (L(X + hU) - L(X - hU)) / 2h for a random U, per input X."""
    x, do, dS = _inputs(seed=1)
    if not sw.get("beta_sigmoid", True):
        x["beta"] = 1.0 / (1.0 + np.exp(-x["beta"]))     # activated betas in (0, 1)
    if not sw.get("gate_in", True):
        x["g"] = -np.abs(x["g"])                           # log-decays <= 0
    gr = _grads(x, do, dS, **sw)
    names = ["q", "k", "v", "g", "beta", "S0"] + (["A_log", "dt_bias"] if sw.get("gate_in", True) else [])
    for name in names:
        U = RNG.standard_normal(x[name].shape)
        xp = dict(x); xp[name] = x[name] + H_FD * U
        xm = dict(x); xm[name] = x[name] - H_FD * U
        fd = (_loss(xp, do, dS, **sw) - _loss(xm, do, dS, **sw)) / (2 * H_FD)
        an = float((gr[_GRAD_NAME[name]] * U).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


def test_elementwise_finite_differences_tiny():
    """Every entry of every gradient on a 3-token, Dk = Dv = 2 problem."""
    x, do, dS = _inputs(T=3, HV=1, Dk=2, Dv=2, seed=3)
    gr = _grads(x, do, dS)
    for name in ["q", "k", "v", "g", "beta", "S0", "A_log", "dt_bias"]:
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(*x[name].shape):
            xp = dict(x); xp[name] = x[name].copy(); xp[name][idx] += H_FD
            xm = dict(x); xm[name] = x[name].copy(); xm[name][idx] -= H_FD
            fd[idx] = (_loss(xp, do, dS) - _loss(xm, do, dS)) / (2 * H_FD)
        assert np.allclose(gr[name], fd, rtol=1e-6, atol=1e-7), name


def test_initial_state_gradient_is_the_transposed_transition():
    """With do = 0, dS0 = M_T^T dS_T exactly (S_T = M_T S0 + run from zero)."""
    x, _, dS = _inputs(B=2, T=9, H=2, HV=4, Dk=5, Dv=3, seed=5)
    do = np.zeros((2, 9, 4, 3))
    f = oracle.kda_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], A_log=x["A_log"],
                       dt_bias=x["dt_bias"], S0=x["S0"], want_M=True)
    gr = _grads(x, do, dS)
    expect = np.einsum("bhij,bhiv->bhjv", f["M_T"], dS)
    assert np.allclose(gr["S0"], expect, rtol=1e-12, atol=1e-12)


def test_chain_forward_matches_the_c_oracle():
    """The reverse pass replays its own forward; it must be the C oracle's."""
    x, _, _ = _inputs(T=7, HV=1, Dk=4, Dv=3, seed=7)
    f = oracle.kda_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], S0=x["S0"],
                       qk_l2norm=False, beta_sigmoid=False, gate_in=False)
    o, S_T, _ = backward.chain_forward(x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0],
                                       x["g"][0, :, 0], x["beta"][0, :, 0], x["S0"][0, 0])
    assert np.allclose(o, f["o"][0, :, 0], rtol=1e-12, atol=1e-12)
    assert np.allclose(S_T, f["S_T"][0, 0], rtol=1e-12, atol=1e-12)


def test_zero_beta_passes_no_gradient_to_v_and_k_through_the_write():
    """beta = 0 (activated): the state only decays, so dv = 0 and dk = 0."""
    x, do, dS = _inputs(seed=9)
    x["beta"] = np.zeros_like(x["beta"])
    gr = _grads(x, do, dS, beta_sigmoid=False)
    assert np.array_equal(gr["v"], np.zeros_like(gr["v"]))
    assert np.allclose(gr["k"], 0.0, atol=0.0)


def test_gva_heads_sum_into_the_shared_qk_gradient():
    """With HV = 2 H, dq of a q/k head is the sum over the value heads that read it."""
    x, do, dS = _inputs(HV=2, seed=11)
    both = _grads(x, do, dS)
    parts = []
    for hv in range(2):
        do1 = do.copy(); do1[:, :, 1 - hv] = 0
        dS1 = dS.copy(); dS1[:, 1 - hv] = 0
        parts.append(_grads(x, do1, dS1))
    assert np.allclose(both["q"], parts[0]["q"] + parts[1]["q"], rtol=1e-12, atol=1e-12)
    assert np.allclose(both["k"], parts[0]["k"] + parts[1]["k"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T,chunk", [(16, 16), (37, 16), (40, 8), (5, 16)])
def test_chunk_backward_equals_the_token_backward(T, chunk):
    """The chunk-parallel reverse pass (the algebra a chunk kernel follows) gives
    the token-by-token gradient, ragged last chunk included."""
    from oracle import chunkwise
    r = np.random.default_rng(T * 31 + chunk)
    Dk, Dv = 6, 5
    q = r.standard_normal((T, Dk)); k = r.standard_normal((T, Dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = r.standard_normal((T, Dv)); g = -0.3 * np.abs(r.standard_normal((T, Dk)))
    b = r.uniform(0.1, 0.9, T); S0 = r.standard_normal((Dk, Dv))
    do = r.standard_normal((T, Dv)); dS = r.standard_normal((Dk, Dv))
    ref = backward.chain_backward(q, k, v, g, b, S0, do, dS, scale=0.7)
    got = chunkwise.chunk_backward(q, k, v, g, b, S0, do, dS, chunk=chunk, scale=0.7)
    for name in ref:
        assert np.allclose(got[name], ref[name], rtol=1e-9, atol=1e-10), name


def _loss_variant(x, do, dS, gate, per_head):
    """Forward through the gate variants of oracle/gates.py, then the C oracle
    with its own gate switched off."""
    from oracle import gates
    Dk = x["q"].shape[-1]
    if per_head:
        z = x["z"][..., None]
        bias = x["dt_bias"][:, None]
    else:
        z, bias = x["z"], x["dt_bias"]
    if gate == "bounded":
        g = gates.bounded_gate(z, x["A_log"], bias)
    else:
        g = gates.softplus_gate(z, x["A_log"], bias)
    g = np.broadcast_to(g, z.shape[:-1] + (Dk,))
    f = oracle.kda_fwd(x["q"], x["k"], x["v"], np.ascontiguousarray(g), x["beta"], S0=x["S0"], gate_in=False)
    return float((f["o"] * do).sum() + (f["S_T"] * dS).sum())


@pytest.mark.parametrize("gate,per_head", [("softplus", False), ("bounded", True), ("softplus", True)])
def test_gate_variant_gradients_match_finite_differences(gate, per_head):
    """Softplus (v1) gate and the per-head (Gated DeltaNet) layout: directional
    derivatives of every input, including z, A_log and dt_bias."""
    x, do, dS = _inputs(seed=13)
    r = np.random.default_rng(14)
    x["z"] = r.standard_normal(x["g"].shape[:-1]) if per_head else x["g"]
    if per_head:
        x["dt_bias"] = 0.5 * r.standard_normal(x["dt_bias"].shape[0])
    gr = backward.kda_backward(x["q"], x["k"], x["v"], x["z"], x["beta"], A_log=x["A_log"],
                               dt_bias=x["dt_bias"], S0=x["S0"], do=do, dS_T=dS, gate=gate, per_head=per_head)
    for name, gname in [("z", "g"), ("A_log", "A_log"), ("dt_bias", "dt_bias"), ("q", "q"), ("beta", "beta")]:
        U = RNG.standard_normal(x[name].shape)
        xp = dict(x); xp[name] = x[name] + H_FD * U
        xm = dict(x); xm[name] = x[name] - H_FD * U
        fd = (_loss_variant(xp, do, dS, gate, per_head) - _loss_variant(xm, do, dS, gate, per_head)) / (2 * H_FD)
        an = float((gr[gname] * U).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


# --- the summed magnitudes A_log_l1 / dt_bias_l1 ---------------------------
# They are the denominators the parameter-gradient bars use (a float sum is
# accurate to the l1 norm of its terms), so they are pinned too: by the
# triangle inequality on random draws, by their invariance when the loss
# changes sign, by additivity over independent batch rows, and exactly on
# inputs built so that every term has one sign.

@pytest.mark.parametrize("gate,per_head", [("bounded", False), ("softplus", False),
                                           ("bounded", True), ("softplus", True)])
def test_l1_bounds_the_parameter_gradients(gate, per_head):
    """|sum of terms| <= sum of |terms|, element by element, and strictly below
    it somewhere (random draws give terms of both signs)."""
    x, do, dS = _inputs(B=2, T=7, seed=31)
    if per_head:
        r = np.random.default_rng(32)
        x["g"] = r.standard_normal(x["g"].shape[:-1])
        x["dt_bias"] = 0.5 * r.standard_normal(x["dt_bias"].shape[0])
    gr = _grads(x, do, dS, gate=gate, per_head=per_head)
    for name in ("A_log", "dt_bias"):
        l1, s = gr[name + "_l1"], gr[name]
        assert l1.shape == s.shape
        assert np.all(np.abs(s) <= l1 * (1 + 1e-12))
        assert np.any(np.abs(s) < 0.999 * l1)


@pytest.mark.parametrize("gate", ["bounded", "softplus"])
def test_l1_is_even_in_the_loss_and_additive_over_batch_rows(gate):
    """Negating do and dS_T negates every gradient but leaves the summed
    magnitudes unchanged; two independent batch rows add their magnitudes."""
    x, do, dS = _inputs(B=2, T=5, seed=33)
    gp = _grads(x, do, dS, gate=gate)
    gm = _grads(x, -do, -dS, gate=gate)
    rows = [_grads({n: (a[b:b + 1] if n in ("q", "k", "v", "g", "beta", "S0") else a) for n, a in x.items()},
                   do[b:b + 1], dS[b:b + 1], gate=gate) for b in range(2)]
    for name in ("A_log", "dt_bias"):
        np.testing.assert_allclose(gm[name], -gp[name], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gm[name + "_l1"], gp[name + "_l1"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(rows[0][name + "_l1"] + rows[1][name + "_l1"], gp[name + "_l1"],
                                   rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("gate,per_head", [("bounded", False), ("softplus", False), ("bounded", True)])
def test_l1_equals_the_sum_when_every_term_has_one_sign(gate, per_head):
    """With beta = 0 the recurrence is pure decay, S_T = prod(alpha) S0; with
    S0 >= 0, dS_T >= 0 and do = 0 every dL/dg is >= 0, so every gate term
    (dz, and for positive pre-activations the A_log terms) has one sign and
    the sum of magnitudes equals the magnitude of the sum."""
    r = np.random.default_rng(35)
    B, T, H, HV, Dk, Dv = 2, 9, 1, 2, 4, 3
    zshape = (B, T, HV) if per_head else (B, T, HV, Dk)
    x = dict(q=r.standard_normal((B, T, H, Dk)), k=r.standard_normal((B, T, H, Dk)),
             v=r.standard_normal((B, T, HV, Dv)),
             g=np.abs(r.standard_normal(zshape)) + 0.1,               # z > 0
             beta=np.zeros((B, T, HV)), A_log=0.3 * r.standard_normal(HV),
             dt_bias=np.abs(r.standard_normal((HV,) if per_head else (HV, Dk))),   # z + dt_bias > 0
             S0=np.abs(r.standard_normal((B, HV, Dk, Dv))))
    do = np.zeros((B, T, HV, Dv))
    dS = np.abs(r.standard_normal((B, HV, Dk, Dv)))
    gr = backward.kda_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], A_log=x["A_log"],
                               dt_bias=x["dt_bias"], S0=x["S0"], do=do, dS_T=dS, beta_sigmoid=False,
                               gate=gate, per_head=per_head)
    for name in ("A_log", "dt_bias"):
        assert np.all(np.abs(gr[name]) > 0)
        np.testing.assert_allclose(gr[name + "_l1"], np.abs(gr[name]), rtol=1e-12)
