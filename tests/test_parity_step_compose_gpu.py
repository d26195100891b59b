"""GPU parity of kda_step (decode) and kda_compose (KCP combine) against the
FP64 oracle, plus the end-to-end segmented forward."""
import pytest
import torch

import gated_delta_rule_157_b200 as kda
import oracle
import workloads
from helpers import TOL_BF16, TOL_F32, max_rel, oracle_chunk, to_device, to_np

pytestmark = pytest.mark.gpu


def _oracle_step(S, inp, flags=True):
    return oracle.kda_step(to_np(S), *(to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                           A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]),
                           qk_l2norm=flags, beta_sigmoid=flags, gate_in=flags)


def _gpu_step(S, d, flags=True):
    return kda.kda_step(S, d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                        dt_bias=d["dt_bias"], qk_l2norm_in_kernel=flags,
                        beta_sigmoid_in_kernel=flags, gate_in_kernel=flags)


@pytest.mark.parametrize("B,H,HV,Dk,Dv,dt", [
    (8, 4, 4, 128, 128, "bf16"),
    (3, 2, 4, 64, 32, "f32"),
    (2, 1, 3, 20, 12, "f32"),
    (1, 1, 1, 128, 4, "bf16"),
])
def test_step_consecutive(cuda_device, B, H, HV, Dk, Dv, dt):
    w = workloads.Workload("dec", B=B, T=1, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=1, dtype=dt, seed=9,
                           s0_std=0.05, steps=4)
    S_ref = to_np(workloads.decode_state(w))
    S = workloads.decode_state(w).to(cuda_device)
    for step in range(w.steps):
        inp = workloads.decode_step_inputs(w, step)
        S_ref, o_ref = _oracle_step(S_ref, inp)
        o = _gpu_step(S, to_device(inp, cuda_device))
        tol = TOL_F32 if dt == "f32" else TOL_BF16
        assert max_rel(to_np(o), o_ref) <= tol
        assert max_rel(to_np(S), S_ref) <= TOL_F32   # fp32 state, fp32 math


def test_decode_workload_full_batch(cuda_device):
    """B=256, H=HV=32, Dk=Dv=128, fp32 state ~ N(0, 0.05), bf16 q/k/v: two
    consecutive steps on every chain, compared with the oracle everywhere."""
    w = workloads.workload("decode_bf16")
    S = workloads.decode_state(w)
    S_ref = to_np(S)
    S = S.to(cuda_device)
    for step in range(2):
        inp = workloads.decode_step_inputs(w, step)
        S_ref, o_ref = _oracle_step(S_ref, inp)
        o = _gpu_step(S, to_device(inp, cuda_device))
        assert max_rel(to_np(o), o_ref) <= TOL_BF16
        assert max_rel(to_np(S), S_ref) <= TOL_F32


def test_decode_workload_512_steps_sampled(cuda_device):
    """The decode workload as the benchmark runs it: B=256, H=HV=32, 512
    consecutive steps against the resident fp32 state, every chain updated on
    the GPU; a sample of chains (spread over batch rows and heads) is followed
    by the oracle through all 512 steps, o checked at every step and the state
    at the end (the fp32 state must not drift from the FP64 one)."""
    import numpy as np
    w = workloads.workload("decode_bf16")
    S0 = workloads.decode_state(w)
    chains = [(0, 0), (17, 5), (128, 31), (255, 16), (63, 9), (200, 22)]
    bi = np.array([c[0] for c in chains]); hi = np.array([c[1] for c in chains])
    S_ref = to_np(S0)[bi, hi][:, None]                           # [n, 1, Dk, Dv]
    S = S0.to(cuda_device)
    bt, ht = torch.from_numpy(bi).to(cuda_device), torch.from_numpy(hi).to(cuda_device)
    worst_o = 0.0
    for step in range(w.steps):
        inp = workloads.decode_step_inputs(w, step, device=cuda_device)
        o = _gpu_step(S, inp)
        sub = {n: to_np(inp[n][bt, ht])[:, None] for n in ("q", "k", "v", "g", "beta")}
        sub["A_log"] = to_np(inp["A_log"])[:1]
        sub["dt_bias"] = None
        S_ref, o_ref = _oracle_step(S_ref, sub)
        worst_o = max(worst_o, max_rel(to_np(o[bt, ht])[:, None], o_ref))
    assert worst_o <= TOL_BF16, worst_o
    assert max_rel(to_np(S[bt, ht])[:, None], S_ref) <= TOL_F32


def test_step_matches_chunk_forward(cuda_device):
    """T consecutive decode steps equal one chunked forward over the T tokens."""
    w = workloads.Workload("sm", B=2, T=24, H=1, HV=2, Dk=32, Dv=32, chunk=16, dtype="f32",
                           seed=12, s0_std=0.1)
    d = to_device(workloads.chunk_inputs(w), cuda_device)
    o_seq, S_seq, _ = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                        A_log=d["A_log"], S0=d["S0"], chunk=16, algo="simt")
    S = d["S0"].clone()
    for t in range(w.T):
        o = kda.kda_step(S, d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                         d["v"][:, t].contiguous(), d["g"][:, t].contiguous(),
                         d["beta"][:, t].contiguous(), A_log=d["A_log"])
        assert max_rel(to_np(o), to_np(o_seq[:, t])) <= TOL_F32
    assert max_rel(to_np(S), to_np(S_seq)) <= TOL_F32


@pytest.mark.parametrize("n_seg,BH,Dk,Dv,init", [(8, 4, 128, 128, True), (3, 2, 40, 24, False),
                                                 (0, 2, 16, 16, True), (1, 1, 7, 33, True)])
def test_compose(cuda_device, n_seg, BH, Dk, Dv, init):
    g = torch.Generator().manual_seed(n_seg * 100 + Dk)
    M = torch.randn(n_seg, BH, Dk, Dk, generator=g) / Dk ** 0.5
    S_seg = torch.randn(n_seg, BH, Dk, Dv, generator=g)
    S_init = torch.randn(BH, Dk, Dv, generator=g) if init else None
    ref = oracle.kda_compose(to_np(M), to_np(S_seg), to_np(S_init))
    S_in = kda.kda_compose(M.to(cuda_device), S_seg.to(cuda_device),
                           None if S_init is None else S_init.to(cuda_device))
    assert max_rel(to_np(S_in), ref) <= TOL_F32


def test_segmented_forward_equals_full_pass(cuda_device):
    """KCP on one GPU: segments run from zero with their transitions, the combine
    gives every segment's incoming state, and a rerun from those states gives
    the outputs of the unsegmented pass (slow gates so the state carries far)."""
    n_seg, L = 4, 96
    w = workloads.Workload("kcp", B=1, T=n_seg * L, H=2, HV=2, Dk=32, Dv=32, chunk=32,
                           dtype="f32", seed=13, s0_std=0.1)
    inp = workloads.chunk_inputs(w, z_mean=-6.0)
    d = to_device(inp, cuda_device)
    kw = dict(A_log=d["A_log"], chunk=w.chunk, algo="simt")
    o_full, S_full, _ = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], **kw)
    Ms, Ss = [], []
    for s in range(n_seg):
        sl = slice(s * L, (s + 1) * L)
        seg = [d[n][:, sl].contiguous() for n in ("q", "k", "v", "g", "beta")]
        _, S_loc, M_loc = kda.kda_chunk_fwd(*seg, output_transition=True, **kw)
        Ms.append(M_loc.reshape(1, -1, 32, 32))
        Ss.append(S_loc.reshape(1, -1, 32, 32))
    M = torch.cat(Ms)
    assert M.abs().max() > 1e-2           # the transition carries information
    S_in = kda.kda_compose(M, torch.cat(Ss), d["S0"].reshape(-1, 32, 32))
    assert max_rel(to_np(S_in[-1]), to_np(S_full.reshape(-1, 32, 32))) <= TOL_F32
    ref = oracle_chunk(inp)
    assert max_rel(to_np(S_in[-1]).reshape(ref["S_T"].shape), ref["S_T"]) <= TOL_F32
    for s in range(n_seg):
        sl = slice(s * L, (s + 1) * L)
        seg = [d[n][:, sl].contiguous() for n in ("q", "k", "v", "g", "beta")]
        o_s, _, _ = kda.kda_chunk_fwd(*seg, S0=S_in[s].reshape(1, 2, 32, 32).contiguous(), **kw)
        assert max_rel(to_np(o_s), ref["o"][:, sl]) <= TOL_F32
