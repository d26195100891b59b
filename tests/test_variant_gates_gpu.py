"""GPU parity of the gate variants (softplus gate of the first KDA version; one
decay per (token, head) as in Gated DeltaNet) on the SIMT kernels -- chunk
forward, decode step and backward -- against the FP64 oracle, which takes the
variant gates precomputed by oracle/gates.py.  The tensor-core kernel takes
the per-head decay, and the softplus gate under a guard: its exponent bound
needs g >= g_min, so it clamps there and reports the clamp.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_157_b200 as kda
import oracle
import workloads
from helpers import TOL_BF16, TOL_F32, max_rel, sum_rel, to_device, to_np
from oracle import backward, gates

pytestmark = pytest.mark.gpu


def _variant_inputs(B, T, H, HV, Dk, Dv, chunk, dtype, seed, per_head, z_mean=0.0):
    w = workloads.Workload("gate", B=B, T=T, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=chunk, dtype=dtype, seed=seed,
                           a_log="uniform", dt_bias_std=0.5, s0_std=0.1)
    inp = workloads.chunk_inputs(w, z_mean=z_mean)
    if per_head:      # the generator's draws cut to one gate value per (token, head)
        inp["g"] = inp["g"][..., 0].contiguous()
        inp["dt_bias"] = inp["dt_bias"][:, 0].contiguous()
    return w, inp


def _log_decay(inp, gate, per_head, Dk):
    z, A, b = to_np(inp["g"]), to_np(inp["A_log"]), to_np(inp["dt_bias"])
    if per_head:
        z, b = z[..., None], b[:, None]
    g = (gates.bounded_gate if gate == "bounded" else gates.softplus_gate)(z, A, b)
    return np.ascontiguousarray(np.broadcast_to(g, z.shape[:-1] + (Dk,)))


def _oracle_fwd(inp, gate, per_head, Dk):
    return oracle.kda_fwd(*(to_np(inp[n]) for n in ("q", "k", "v")), _log_decay(inp, gate, per_head, Dk),
                          to_np(inp["beta"]), S0=to_np(inp["S0"]), gate_in=False)


def _fwd(d, w, gate, per_head, algo="auto", S_chunks=None):
    return kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"], dt_bias=d["dt_bias"],
                             S0=d["S0"], chunk=w.chunk, gate_in_kernel=gate, g_per_head=per_head, algo=algo,
                             S_chunks=S_chunks)


FWD_CASES = [
    # B, T, H, HV, Dk, Dv, chunk, dtype, gate, per_head
    (1, 100, 1, 2, 32, 32, 32, "f32", "softplus", False),
    (2, 77, 1, 2, 16, 24, 16, "f32", "bounded", True),
    (1, 130, 2, 4, 128, 128, 64, "bf16", "softplus", True),
    (1, 130, 1, 2, 128, 128, 64, "bf16", "softplus", False),
]


@pytest.mark.parametrize("case", FWD_CASES, ids=lambda c: "x".join(map(str, c)))
def test_chunk_forward_gate_variants(cuda_device, case):
    B, T, H, HV, Dk, Dv, chunk, dtype, gate, per_head = case
    w, inp = _variant_inputs(B, T, H, HV, Dk, Dv, chunk, dtype, seed=60 + T, per_head=per_head)
    d = to_device(inp, cuda_device)
    o, S_T, _ = _fwd(d, w, gate, per_head)
    ref = _oracle_fwd(inp, gate, per_head, Dk)
    assert max_rel(to_np(o), ref["o"]) <= (TOL_F32 if dtype == "f32" else TOL_BF16)
    assert max_rel(to_np(S_T), ref["S_T"]) <= TOL_F32          # SIMT: fp32 state from exact inputs


def _clamped_oracle(inp, Dk, g_min=-5.0):
    g = np.maximum(_log_decay(inp, "softplus", False, Dk), g_min)
    return oracle.kda_fwd(*(to_np(inp[n]) for n in ("q", "k", "v")), g, to_np(inp["beta"]),
                          S0=to_np(inp["S0"]), gate_in=False)


def test_tensor_core_kernel_guards_the_softplus_gate(cuda_device):
    """The softplus gate is unbounded below and the tensor-core kernel's
    exponent bound needs g >= g_min.  Where the gate stays above g_min
    (small exp(A_log)), algo='tc' matches the oracle at the bf16 bar with no
    report; where it falls below (large exp(A_log)), the kernel clamps g to
    g_min, reports KDA_ERR_RANGE and matches the oracle on the clamped decay.
    'auto' keeps the exact SIMT kernel (bit for bit)."""
    from helpers import fro_rel
    w, inp = _variant_inputs(1, 200, 1, 2, 128, 128, 64, "bf16", seed=70, per_head=False)
    inp["A_log"] = torch.full_like(inp["A_log"], -1.5)          # exp(A_log) = 0.22: g > -2
    assert float(_log_decay(inp, "softplus", False, 128).min()) > -5.0
    d = to_device(inp, cuda_device)
    kda.kda_device_status()
    o, S_T, _ = _fwd(d, w, "softplus", False, algo="tc")
    kda.kda_device_status()                                     # nothing reported
    ref = _oracle_fwd(inp, "softplus", False, 128)
    assert max_rel(to_np(o), ref["o"]) <= TOL_BF16
    assert fro_rel(to_np(S_T), ref["S_T"]) <= TOL_BF16

    inp["A_log"] = torch.full_like(inp["A_log"], 2.0)           # exp(A_log) = 7.4: g well below -5
    assert float(_log_decay(inp, "softplus", False, 128).min()) < -8.0
    d = to_device(inp, cuda_device)
    o, S_T, _ = _fwd(d, w, "softplus", False, algo="tc")
    with pytest.raises(kda.KdaError) as e:
        kda.kda_device_status()
    assert e.value.status == 7                                  # KDA_ERR_RANGE
    kda.kda_device_status()                                     # and cleared
    ref = _clamped_oracle(inp, 128)
    assert max_rel(to_np(o), ref["o"]) <= TOL_BF16
    assert fro_rel(to_np(S_T), ref["S_T"]) <= TOL_BF16
    a, b = _fwd(d, w, "softplus", False, algo="auto"), _fwd(d, w, "softplus", False, algo="simt")
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_per_head_gate_on_the_tensor_core_kernel(cuda_device):
    """One bounded decay per (token, head) on the tensor-core kernel (AUTO takes
    it for this shape), against the oracle at the bf16 bars."""
    from helpers import fro_rel
    w, inp = _variant_inputs(1, 130, 2, 4, 128, 128, 64, "bf16", seed=72, per_head=True)
    d = to_device(inp, cuda_device)
    o, S_T, _ = _fwd(d, w, "bounded", True, algo="tc")
    a = _fwd(d, w, "bounded", True, algo="auto")
    assert torch.equal(a[0], o) and torch.equal(a[1], S_T)
    ref = _oracle_fwd(inp, "bounded", True, 128)
    assert max_rel(to_np(o), ref["o"]) <= TOL_BF16
    assert fro_rel(to_np(S_T), ref["S_T"]) <= TOL_BF16


def test_unbounded_gate_stays_finite_where_the_factorised_form_overflows(cuda_device):
    """Page "KDA 模块交互式演示", the chunk-overflow tab: the softplus gate driven at
    z + 6 makes exp(-sum g) over a 16-token chunk overflow in fp32.  The SIMT
    kernel only exponentiates differences G_r - G_i <= 0, so it stays finite
    and on the oracle."""
    w, inp = _variant_inputs(1, 96, 1, 2, 32, 32, 16, "f32", seed=71, per_head=False, z_mean=6.0)
    inp["A_log"] = torch.zeros(2)                       # g = -softplus(z), as on the tab
    inp["dt_bias"] = torch.zeros(2, 32)
    g = _log_decay(inp, "softplus", False, 32)
    with np.errstate(over="ignore"):                    # the factor the tab plots, per chunk and channel
        factor = np.exp(-g[0].reshape(6, 16, 2, 32).sum(axis=1)).astype(np.float32)
    assert np.isinf(factor).mean() > 0.5
    d = to_device(inp, cuda_device)
    o, S_T, _ = _fwd(d, w, "softplus", False)
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(S_T).all())
    ref = _oracle_fwd(inp, "softplus", False, 32)
    assert max_rel(to_np(o), ref["o"]) <= TOL_F32


STEP_CASES = [
    # B, H, HV, Dk, Dv, dtype, gate, per_head
    (4, 2, 4, 128, 128, "bf16", "softplus", False),
    (4, 2, 4, 128, 128, "bf16", "bounded", True),
    (2, 1, 2, 64, 32, "f32", "softplus", True),
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: "x".join(map(str, c)))
def test_decode_step_gate_variants(cuda_device, case):
    B, H, HV, Dk, Dv, dtype, gate, per_head = case
    w, inp = _variant_inputs(B, 1, H, HV, Dk, Dv, 1, dtype, seed=80 + Dk, per_head=per_head)
    x = {n: inp[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "beta")}
    S = inp["S0"].clone().to(cuda_device)
    o = kda.kda_step(S, *(x[n].to(cuda_device) for n in ("q", "k", "v", "g", "beta")),
                     A_log=inp["A_log"].to(cuda_device), dt_bias=inp["dt_bias"].to(cuda_device),
                     gate_in_kernel=gate, g_per_head=per_head)
    g = _log_decay({"g": inp["g"][:, 0], "A_log": inp["A_log"], "dt_bias": inp["dt_bias"]}, gate, per_head, Dk)
    S_ref, o_ref = oracle.kda_step(to_np(inp["S0"]), *(to_np(x[n]) for n in ("q", "k", "v")), g,
                                   to_np(x["beta"]), gate_in=False)
    assert max_rel(to_np(o), o_ref) <= (TOL_F32 if dtype == "f32" else TOL_BF16)
    assert max_rel(to_np(S), S_ref) <= TOL_F32


BWD_CASES = [
    # B, T, H, HV, Dk, Dv, chunk, dtype, gate, per_head
    (1, 70, 1, 2, 32, 32, 32, "f32", "softplus", False),
    (2, 50, 1, 2, 16, 40, 16, "f32", "bounded", True),
    (1, 130, 1, 2, 128, 128, 64, "bf16", "softplus", True),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "x".join(map(str, c)))
def test_backward_gate_variants(cuda_device, case):
    B, T, H, HV, Dk, Dv, chunk, dtype, gate, per_head = case
    w, inp = _variant_inputs(B, T, H, HV, Dk, Dv, chunk, dtype, seed=90 + T, per_head=per_head)
    gen = torch.Generator().manual_seed(91 + T)
    dout = torch.randn((B, T, HV, Dv), generator=gen).to(inp["q"].dtype)
    dS_T = torch.randn((B, HV, Dk, Dv), generator=gen)
    d = to_device(inp, cuda_device)
    S_ch = torch.empty((B, HV, -(-T // chunk), Dk, Dv), device=cuda_device)
    _fwd(d, w, gate, per_head, algo="simt", S_chunks=S_ch)
    gr = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S_ch, dout.to(cuda_device),
                           dS_T.to(cuda_device), A_log=d["A_log"], dt_bias=d["dt_bias"], chunk=chunk,
                           gate_in_kernel=gate, g_per_head=per_head)
    ref = backward.kda_backward(*(to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]), S0=to_np(inp["S0"]),
                                do=to_np(dout), dS_T=to_np(dS_T), gate=gate, per_head=per_head)
    for n, rn in {"dq": "q", "dk": "k", "dv": "v", "dg": "g", "dbeta": "beta", "dS0": "S0"}.items():
        assert max_rel(to_np(gr[n]), ref[rn]) <= TOL_F32, n
    for n, rn in {"dA_log": "A_log", "ddt_bias": "dt_bias"}.items():   # sums over tokens
        assert sum_rel(to_np(gr[n]), ref[rn], ref[rn + "_l1"]) <= TOL_F32, n
