"""GPU parity of the training path: the per-chunk states kda_chunk_fwd keeps,
kda_chunk_bwd, and the autograd function built on them, against the FP64
oracle (oracle/backward.py, itself pinned by finite differences).

The backward computes in FP32 from the exact (widened) inputs, so every
gradient is held to the FP32 bar, max|gpu - ref| / max|ref| <= 1e-4, for bf16
inputs too.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_157_b200 as kda
import oracle
import workloads
from helpers import TOL_F32, max_rel, sum_rel, to_device, to_np
from oracle import backward

pytestmark = pytest.mark.gpu


def _inputs(B, T, H, HV, Dk, Dv, chunk, dtype, seed, flags=True, s0=0.3, dST=True):
    """Raw draws (switches on) or activated draws (switches off), plus dout, dS_T."""
    w = workloads.Workload("bwd", B=B, T=T, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=chunk, dtype=dtype,
                           seed=seed, a_log="uniform", dt_bias_std=0.5, s0_std=s0)
    inp = workloads.chunk_inputs(w) if flags else workloads.activated_inputs(w)
    tdt = inp["q"].dtype
    gen = torch.Generator().manual_seed(seed + 1000)
    inp["dout"] = torch.randn((B, T, HV, Dv), generator=gen).to(tdt)
    inp["dS_T"] = torch.randn((B, HV, Dk, Dv), generator=gen) if dST else None
    return w, inp


def _oracle_grads(inp, flags, scale):
    return backward.kda_backward(*(to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                 A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]),
                                 S0=to_np(inp["S0"]), do=to_np(inp["dout"]), dS_T=to_np(inp["dS_T"]),
                                 scale=scale, qk_l2norm=flags, beta_sigmoid=flags, gate_in=flags)


def _forward_with_states(d, w, flags, scale, algo="simt"):
    NC = -(-w.T // w.chunk)
    S_chunks = torch.full((w.B, w.HV, NC, w.Dk, w.Dv), float("nan"), device=d["q"].device)
    o, S_T, _ = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                                  dt_bias=d["dt_bias"], S0=d["S0"], chunk=w.chunk, scale=scale,
                                  qk_l2norm_in_kernel=flags, beta_sigmoid_in_kernel=flags,
                                  gate_in_kernel=flags, S_chunks=S_chunks, algo=algo)
    return o, S_T, S_chunks


STATE_SHAPES = [
    # B, T, H, HV, Dk, Dv, chunk, dtype
    (1, 100, 1, 2, 16, 16, 16, "f32"),
    (2, 77, 2, 4, 32, 24, 32, "f32"),
    (1, 200, 1, 2, 128, 128, 64, "bf16"),
]


@pytest.mark.parametrize("shape", STATE_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_chunk_states_are_the_prefix_states(cuda_device, shape):
    """S_chunks[:, :, c] is the state after the first c * chunk tokens."""
    w, inp = _inputs(*shape, seed=21)
    d = to_device(inp, cuda_device)
    o, S_T, S_ch = _forward_with_states(d, w, True, 1.0)
    o2, S_T2, _ = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                                    dt_bias=d["dt_bias"], S0=d["S0"], chunk=w.chunk, algo="simt")
    assert torch.equal(o, o2) and torch.equal(S_T, S_T2)   # keeping the states changes nothing
    S_ch = to_np(S_ch)
    for c in range(S_ch.shape[2]):
        t = c * w.chunk
        if t == 0:
            ref = np.zeros_like(S_ch[:, :, 0]) if inp["S0"] is None else to_np(inp["S0"])
        else:
            ref = oracle.kda_fwd(*(to_np(inp[n])[:, :t] for n in ("q", "k", "v", "g", "beta")),
                                 A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]),
                                 S0=to_np(inp["S0"]))["S_T"]
        assert max_rel(S_ch[:, :, c], ref) <= TOL_F32, c


def test_tensor_core_kernel_writes_chunk_states(cuda_device):
    """The tensor-core kernel (which AUTO takes for this shape) writes the state
    entering each chunk: keeping the states changes neither o nor S_T, and the
    states are the prefix states within the bf16 bar."""
    from helpers import TOL_BF16, fro_rel
    w, inp = _inputs(1, 200, 1, 2, 128, 128, 64, "bf16", seed=22, s0=0.05)
    d = to_device(inp, cuda_device)
    a = _forward_with_states(d, w, True, 1.0, algo="auto")
    b = _forward_with_states(d, w, True, 1.0, algo="tc")
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    o, S_T, _ = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                                  dt_bias=d["dt_bias"], S0=d["S0"], chunk=64, algo="tc")
    assert torch.equal(o, b[0]) and torch.equal(S_T, b[1])
    S_ch = to_np(b[2])
    for c in range(S_ch.shape[2]):
        if c == 0:
            ref = to_np(inp["S0"])
        else:
            ref = oracle.kda_fwd(*(to_np(inp[n])[:, :c * 64] for n in ("q", "k", "v", "g", "beta")),
                                 A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]),
                                 S0=to_np(inp["S0"]))["S_T"]
        assert fro_rel(S_ch[:, :, c], ref) <= TOL_BF16, c


BWD_CASES = [
    # B, T, H, HV, Dk, Dv, chunk, dtype, flags, scale, s0, dST
    (1, 37, 1, 2, 16, 12, 16, "f32", True, 1.0, 0.3, True),
    (2, 77, 2, 4, 32, 24, 32, "f32", False, 1.0, 0.3, True),
    (1, 64, 1, 1, 128, 128, 64, "f32", True, 1.0, None, False),   # one whole chunk, zero S0, dS_T
    (2, 130, 2, 4, 64, 48, 64, "bf16", True, 1.0, 0.1, True),     # grouped heads, ragged
    (1, 200, 1, 1, 128, 128, 64, "bf16", True, 0.8, 0.02, True),  # full head size, ragged
    (1, 5, 1, 1, 1, 1, 1, "f32", False, 1.0, 0.3, True),          # Dk = Dv = chunk = 1 (see below)
    (2, 23, 1, 3, 3, 5, 7, "f32", True, 1.0, 0.3, True),          # odd sizes everywhere
    (1, 1, 1, 1, 8, 8, 16, "f32", True, 1.0, 0.3, True),          # one token
    (1, 64, 1, 1, 128, 1, 64, "f32", True, 1.0, 0.3, True),       # Dv = 1
]
# At Dk = 1 the in-kernel L2 norm is degenerate (q / |q| = +-1): its gradient,
# eps / |q|^3 times dq, is the difference of two terms of size |dq| / |q|, which
# FP32 cannot resolve to 1e-4 of the tiny exact value.  That shape runs with
# the switches off.


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "x".join(map(str, c[:8])) + ("" if c[8] else "-raw"))
def test_backward_matches_the_oracle(cuda_device, case):
    B, T, H, HV, Dk, Dv, chunk, dtype, flags, scale, s0, dST = case
    w, inp = _inputs(B, T, H, HV, Dk, Dv, chunk, dtype, seed=30 + T, flags=flags, s0=s0, dST=dST)
    d = to_device(inp, cuda_device)
    _, _, S_ch = _forward_with_states(d, w, flags, scale)
    gr = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S_ch, d["dout"], d["dS_T"],
                           A_log=d["A_log"], dt_bias=d["dt_bias"], chunk=chunk, scale=scale,
                           qk_l2norm_in_kernel=flags, beta_sigmoid_in_kernel=flags, gate_in_kernel=flags)
    torch.cuda.synchronize()
    ref = _oracle_grads(inp, flags, scale)
    names = {"dq": "q", "dk": "k", "dv": "v", "dg": "g", "dbeta": "beta", "dS0": "S0"}
    if flags:
        names.update(dA_log="A_log", ddt_bias="dt_bias")
    for n, rn in names.items():
        if rn in ("A_log", "dt_bias"):     # sums over tokens: against their summed magnitudes
            assert sum_rel(to_np(gr[n]), ref[rn], ref[rn + "_l1"]) <= TOL_F32, n
        else:
            assert max_rel(to_np(gr[n]), ref[rn]) <= TOL_F32, n


def test_backward_of_an_empty_sequence(cuda_device):
    """T = 0: the state passes through, so dS0 = dS_T; the parameter sums are 0."""
    w, inp = _inputs(2, 0, 1, 2, 16, 16, 16, "f32", seed=40)
    d = to_device(inp, cuda_device)
    S_ch = torch.empty((2, 2, 0, 16, 16), device=cuda_device)
    gr = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S_ch, d["dout"], d["dS_T"],
                           A_log=d["A_log"], dt_bias=d["dt_bias"], chunk=16)
    assert torch.equal(gr["dS0"], d["dS_T"])
    assert torch.count_nonzero(gr["dA_log"]) == 0 and torch.count_nonzero(gr["ddt_bias"]) == 0


def test_autograd_function_gradients(cuda_device):
    """torch.autograd through kda_chunk gives the oracle's gradients."""
    w, inp = _inputs(1, 90, 1, 2, 32, 32, 32, "f32", seed=50)
    d = to_device(inp, cuda_device)
    leaves = {n: d[n].clone().requires_grad_(True) for n in ("q", "k", "v", "g", "beta", "A_log",
                                                             "dt_bias", "S0")}
    o, S_T = kda.kda_chunk(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["beta"],
                           A_log=leaves["A_log"], dt_bias=leaves["dt_bias"], S0=leaves["S0"], chunk=32)
    loss = (o * d["dout"]).sum() + (S_T * d["dS_T"]).sum()
    loss.backward()
    ref = _oracle_grads(inp, True, 1.0)
    for n in leaves:
        if n in ("A_log", "dt_bias"):
            assert sum_rel(to_np(leaves[n].grad), ref[n], ref[n + "_l1"]) <= TOL_F32, n
        else:
            assert max_rel(to_np(leaves[n].grad), ref[n]) <= TOL_F32, n


def test_backward_gva_workload_sampled(cuda_device):
    """The full headline shape (B=4, H=16, HV=32, T=8192, Dk=Dv=128, bf16), run
    whole on the GPU; one q/k head and its two value heads of one batch row are
    checked against the oracle (per-token gradients and dS0 of those chains)."""
    w = workloads.workload("gva_bf16")
    inp = workloads.chunk_inputs(w)
    gen = torch.Generator().manual_seed(123)
    dout = torch.randn((w.B, w.T, w.HV, w.Dv), generator=gen).to(torch.bfloat16)
    d = to_device(inp, cuda_device)
    d_out = dout.to(cuda_device)
    S_ch = torch.empty((w.B, w.HV, w.T // w.chunk, w.Dk, w.Dv), device=cuda_device)
    kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"], dt_bias=d["dt_bias"],
                      S0=d["S0"], chunk=w.chunk, S_chunks=S_ch, output_final_state=False, algo="simt")
    gr = kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S_ch, d_out, None,
                           A_log=d["A_log"], dt_bias=d["dt_bias"], chunk=w.chunk)
    torch.cuda.synchronize()
    del S_ch
    b, h = 1, 5
    hv = slice(2 * h, 2 * h + 2)                     # the two value heads reading q/k head h
    sl = {"q": inp["q"][b:b + 1, :, h:h + 1], "k": inp["k"][b:b + 1, :, h:h + 1],
          "v": inp["v"][b:b + 1, :, hv], "g": inp["g"][b:b + 1, :, hv], "beta": inp["beta"][b:b + 1, :, hv]}
    ref = backward.kda_backward(*(to_np(sl[n]) for n in ("q", "k", "v", "g", "beta")),
                                A_log=to_np(inp["A_log"][hv]), dt_bias=to_np(inp["dt_bias"][hv]),
                                do=to_np(dout[b:b + 1, :, hv]))
    got = {"q": gr["dq"][b:b + 1, :, h:h + 1], "k": gr["dk"][b:b + 1, :, h:h + 1], "v": gr["dv"][b:b + 1, :, hv],
           "g": gr["dg"][b:b + 1, :, hv], "beta": gr["dbeta"][b:b + 1, :, hv], "S0": gr["dS0"][b:b + 1, hv]}
    for n, t in got.items():
        assert max_rel(to_np(t), ref[n]) <= TOL_F32, n
