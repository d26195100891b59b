"""GPU parity of kda_chunk_fwd against the FP64 oracle on identical seeded inputs.

Bars: FP32 inputs <= 1e-4 max relative error (o, S_T, M_T); BF16 inputs <= 2e-2 of
max|o| and <= 2e-2 relative Frobenius error of S_T.  The SIMT kernel computes
in FP32 from the exact inputs, so its fp32 outputs (S_T, M_T) are also held to
1e-4 when the inputs are bf16.
"""
import pytest
import torch

import gated_delta_rule_157_b200 as kda
import workloads
from helpers import TOL_BF16, TOL_F32, fro_rel, max_rel, oracle_chunk, to_device, to_np

pytestmark = pytest.mark.gpu


def run_gpu(inp, w, algo, flags=True, want_M=False, out_state=True, **kw):
    return kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                             A_log=inp["A_log"], dt_bias=inp["dt_bias"], S0=inp["S0"],
                             chunk=w.chunk, qk_l2norm_in_kernel=flags,
                             beta_sigmoid_in_kernel=flags, gate_in_kernel=flags,
                             output_final_state=out_state, output_transition=want_M,
                             algo=algo, **kw)


def check(o, S_T, M_T, ref, dtype, algo):
    if dtype == "f32":
        assert max_rel(to_np(o), ref["o"]) <= TOL_F32
        if S_T is not None:
            assert max_rel(to_np(S_T), ref["S_T"]) <= TOL_F32
        if M_T is not None:
            assert max_rel(to_np(M_T), ref["M_T"]) <= TOL_F32
    else:
        assert max_rel(to_np(o), ref["o"]) <= TOL_BF16
        if S_T is not None:
            assert fro_rel(to_np(S_T), ref["S_T"]) <= TOL_BF16
            if algo == "simt":
                assert max_rel(to_np(S_T), ref["S_T"]) <= TOL_F32
        if M_T is not None:
            assert fro_rel(to_np(M_T), ref["M_T"]) <= TOL_BF16
            if algo == "simt":
                assert max_rel(to_np(M_T), ref["M_T"]) <= TOL_F32


def test_tiny_fp32_workload(cuda_device):
    """B=1, H=HV=2, T=64, Dk=Dv=16, chunk=16, fp32, seed 0, A_log=0, S0=0."""
    w = workloads.workload("tiny_fp32")
    inp = workloads.chunk_inputs(w)
    ref = oracle_chunk(inp, want_M=True)
    o, S_T, M_T = run_gpu(to_device(inp, cuda_device), w, "auto", want_M=True)
    check(o, S_T, M_T, ref, "f32", "simt")


SHAPES = [
    # B, T, H, HV, Dk, Dv, chunk, dtype, s0
    (1, 100, 1, 1, 16, 16, 16, "f32", None),     # ragged tail
    (2, 77, 2, 4, 32, 24, 32, "f32", 0.1),        # Dk != Dv, grouped heads, ragged
    (1, 130, 1, 4, 48, 40, 64, "f32", 0.05),      # HV/H = 4, ragged, C=64
    (1, 64, 2, 2, 128, 128, 64, "f32", 0.02),     # full head size, one chunk
    (2, 200, 2, 2, 64, 128, 64, "bf16", 0.02),    # bf16 activations
    (1, 33, 1, 2, 8, 12, 16, "bf16", None),       # tiny odd sizes
    (1, 5, 1, 1, 4, 4, 64, "f32", 0.3),           # T < chunk
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%d_T%d_H%d_HV%d_K%d_V%d_C%d_%s" % s[:8])
@pytest.mark.parametrize("want_M", [False, True])
def test_simt_shapes(cuda_device, shape, want_M):
    B, T, H, HV, Dk, Dv, C, dt, s0 = shape
    w = workloads.Workload("case", B=B, T=T, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=C, dtype=dt,
                           seed=T + Dk, a_log="uniform", dt_bias_std=0.5, s0_std=s0)
    inp = workloads.chunk_inputs(w)
    ref = oracle_chunk(inp, want_M=want_M)
    o, S_T, M_T = run_gpu(to_device(inp, cuda_device), w, "simt", want_M=want_M)
    check(o, S_T, M_T, ref, dt, "simt")


def test_switches_off_path(cuda_device):
    """Inputs already in activated form (log-decay g, beta in (0,1), near-unit keys)."""
    w = workloads.Workload("act", B=2, T=90, H=1, HV=2, Dk=32, Dv=32, chunk=32, dtype="f32",
                           seed=11, s0_std=0.1)
    inp = workloads.activated_inputs(w)
    ref = oracle_chunk(inp, flags=False, want_M=True)
    o, S_T, M_T = run_gpu(to_device(inp, cuda_device), w, "simt", flags=False, want_M=True)
    check(o, S_T, M_T, ref, "f32", "simt")


@pytest.mark.parametrize("z_mean", [-12.0, 12.0])
def test_extreme_gates(cuda_device, z_mean):
    """z far negative: alpha -> 1 (no forgetting, long memory); z far positive:
    g -> g_min every token, so a 64-token chunk decays by e^-320 (the case
    that overflows an unguarded K/Gamma factorisation in fp32)."""
    w = workloads.Workload("gate", B=1, T=192, H=1, HV=2, Dk=64, Dv=64, chunk=64, dtype="f32",
                           seed=21, s0_std=0.1)
    inp = workloads.chunk_inputs(w, z_mean=z_mean, z_std=0.5)
    ref = oracle_chunk(inp, want_M=True)
    o, S_T, M_T = run_gpu(to_device(inp, cuda_device), w, "simt", want_M=True)
    assert torch.isfinite(o).all() and torch.isfinite(S_T).all() and torch.isfinite(M_T).all()
    check(o, S_T, M_T, ref, "f32", "simt")


def test_scale_and_null_state_outputs(cuda_device):
    w = workloads.Workload("sc", B=1, T=40, H=1, HV=1, Dk=16, Dv=16, chunk=16, dtype="f32",
                           seed=5, s0_std=0.2)
    inp = workloads.chunk_inputs(w)
    ref = oracle_chunk(inp, scale=0.125)
    o, S_T, M_T = run_gpu(to_device(inp, cuda_device), w, "simt", out_state=False, scale=0.125)
    assert S_T is None and M_T is None
    assert max_rel(to_np(o), ref["o"]) <= TOL_F32


def test_state_in_place(cuda_device):
    """S_T may be the same buffer as S0."""
    w = workloads.Workload("ip", B=2, T=50, H=1, HV=2, Dk=16, Dv=32, chunk=16, dtype="f32",
                           seed=6, s0_std=0.3)
    inp = workloads.chunk_inputs(w)
    ref = oracle_chunk(inp)
    d = to_device(inp, cuda_device)
    S = d["S0"].clone()
    d["S0"] = S
    o, S_T, _ = run_gpu(d, w, "simt", S_T=S)
    assert S_T.data_ptr() == S.data_ptr()
    assert max_rel(to_np(S), ref["S_T"]) <= TOL_F32
    assert max_rel(to_np(o), ref["o"]) <= TOL_F32


def test_empty_sequence(cuda_device):
    w = workloads.Workload("e", B=2, T=0, H=1, HV=2, Dk=8, Dv=4, chunk=16, dtype="f32", seed=7,
                           s0_std=1.0)
    d = to_device(workloads.chunk_inputs(w), cuda_device)
    o, S_T, M_T = run_gpu(d, w, "auto", want_M=True)
    assert o.numel() == 0
    torch.testing.assert_close(S_T, d["S0"], rtol=0, atol=0)
    eye = torch.eye(8, device=cuda_device).expand(2, 2, 8, 8)
    torch.testing.assert_close(M_T, eye, rtol=0, atol=0)


def test_aliasing_rejected_with_real_buffers(cuda_device):
    w = workloads.Workload("al", B=1, T=16, H=1, HV=1, Dk=16, Dv=16, chunk=16, dtype="f32",
                           seed=8)
    d = to_device(workloads.chunk_inputs(w), cuda_device)
    with pytest.raises(kda.KdaError) as ei:
        run_gpu(d, w, "simt", o=d["v"])
    assert ei.value.status == 4


def test_prefill_bf16_workload_simt(cuda_device):
    """B=1, H=HV=16, T=4096, Dk=Dv=128, chunk=64, bf16, S0 ~ N(0, 0.02), on the SIMT kernel."""
    w = workloads.workload("prefill_bf16")
    inp = workloads.chunk_inputs(w)
    ref = oracle_chunk(inp)
    o, S_T, _ = run_gpu(to_device(inp, cuda_device), w, "simt")
    check(o, S_T, None, ref, "bf16", "simt")


# ---------------------------------------------------------------------------
# Tensor-core kernel (bf16, Dk = Dv = 128, chunk = 64)
# ---------------------------------------------------------------------------
TC_CASES = [
    # B, T, H, HV, s0_std, want_M, z_mean
    (1, 64, 1, 1, None, False, 0.0),      # one chunk, no initial state
    (1, 192, 1, 2, 0.02, False, 0.0),     # three chunks, carried state
    (2, 200, 2, 4, 0.02, True, 0.0),      # ragged tail, grouped heads, transition
    (1, 256, 1, 2, 0.05, True, -8.0),     # slow decay: long memory, M_T far from 0
    (1, 128, 1, 1, 0.05, False, 12.0),    # g = g_min every token: e^-320 per chunk
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "B%d_T%d_H%d_HV%d_M%d_z%g" % (
    c[0], c[1], c[2], c[3], c[5], c[6]))
def test_tc_small(cuda_device, case):
    B, T, H, HV, s0, want_M, z_mean = case
    w = workloads.Workload("tc", B=B, T=T, H=H, HV=HV, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=31 + T, a_log="uniform", dt_bias_std=0.5, s0_std=s0)
    inp = workloads.chunk_inputs(w, z_mean=z_mean)
    ref = oracle_chunk(inp, want_M=want_M)
    o, S_T, M_T = run_gpu(to_device(inp, cuda_device), w, "tc", want_M=want_M)
    check(o, S_T, M_T, ref, "bf16", "tc")


def test_tc_switches_off(cuda_device):
    w = workloads.Workload("tcoff", B=1, T=130, H=1, HV=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=41, s0_std=0.05)
    inp = workloads.activated_inputs(w)
    ref = oracle_chunk(inp, flags=False, want_M=True)
    o, S_T, M_T = run_gpu(to_device(inp, cuda_device), w, "tc", flags=False, want_M=True)
    check(o, S_T, M_T, ref, "bf16", "tc")


def test_log_decay_below_g_min(cuda_device):
    """A log-decay given directly below g_min: the SIMT kernel uses it as is,
    and AUTO routes a caller-given decay there; the tensor-core kernel, asked
    for explicitly, clamps it to g_min and reports KDA_ERR_RANGE (its exponent bound rests on
    g >= g_min), so it matches the oracle run on the clamped values."""
    w = workloads.Workload("tclow", B=1, T=130, H=1, HV=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=42, s0_std=0.05)
    inp = workloads.activated_inputs(w, g_min=-9.0)
    assert float(inp["g"].float().min()) < -8.0
    d = to_device(inp, cuda_device)
    o, S_T, _ = run_gpu(d, w, "simt", flags=False)
    check(o, S_T, None, oracle_chunk(inp, flags=False), "bf16", "simt")
    o2, S2, _ = run_gpu(d, w, "auto", flags=False)       # AUTO takes the exact SIMT path
    assert torch.equal(o, o2) and torch.equal(S_T, S2)
    clamped = dict(inp, g=inp["g"].float().clamp(min=-5.0).to(inp["g"].dtype))
    kda.kda_device_status()
    o, S_T, _ = run_gpu(d, w, "tc", flags=False)
    with pytest.raises(kda.KdaError) as err:          # the clamp is reported
        kda.kda_device_status()
    assert err.value.status == 7                      # KDA_ERR_RANGE
    kda.kda_device_status()                           # and cleared
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(S_T).all())
    check(o, S_T, None, oracle_chunk(clamped, flags=False), "bf16", "tc")


def test_tc_is_the_default_for_its_shape(cuda_device):
    """algo='auto' picks the tensor-core kernel for bf16 / 128 / chunk 64: its
    result equals the explicit 'tc' call bit for bit."""
    w = workloads.Workload("auto", B=1, T=128, H=1, HV=1, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=43, s0_std=0.02)
    d = to_device(workloads.chunk_inputs(w), cuda_device)
    o1, S1, _ = run_gpu(d, w, "auto")
    o2, S2, _ = run_gpu(d, w, "tc")
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_prefill_bf16_workload_tc(cuda_device):
    """B=1, H=HV=16, T=4096, Dk=Dv=128, chunk=64, bf16, S0 ~ N(0, 0.02)."""
    w = workloads.workload("prefill_bf16")
    inp = workloads.chunk_inputs(w)
    ref = oracle_chunk(inp)
    o, S_T, _ = run_gpu(to_device(inp, cuda_device), w, "tc")
    check(o, S_T, None, ref, "bf16", "tc")


def _per_chain_errors(o, S_T, ref):
    """Largest per-chain o error (max|x - ref| / max|ref| over one (b, hv)
    chain's tokens and channels) and per-chain Frobenius error of S_T."""
    import numpy as np
    o, ro = to_np(o), ref["o"]
    den = np.maximum(np.abs(ro).max(axis=(1, 3)), 1e-30)            # [B, HV]
    e_o = np.abs(o - ro).max(axis=(1, 3)) / den
    del o
    S, rs = to_np(S_T), ref["S_T"]
    e_s = np.linalg.norm((S - rs).reshape(rs.shape[0], rs.shape[1], -1), axis=2) / \
        np.maximum(np.linalg.norm(rs.reshape(rs.shape[0], rs.shape[1], -1), axis=2), 1e-30)
    return float(e_o.max()), float(e_s.max())


def test_gva_bf16_workload_full(cuda_device):
    """B=4, H=16, HV=32, T=8192, Dk=Dv=128, chunk=64, in-kernel switches, in the
    launch configuration the benchmark times; every one of the 128 chains is
    compared with the oracle (o element by element, S_T by Frobenius norm)."""
    w = workloads.workload("gva_bf16")
    inp = workloads.chunk_inputs(w)
    o, S_T, _ = run_gpu(to_device(inp, cuda_device), w, "auto")
    o, S_T = o.cpu(), S_T.cpu()
    ref = oracle_chunk(inp)
    del inp
    e_o, e_s = _per_chain_errors(o, S_T, ref)
    assert e_o <= TOL_BF16, e_o
    assert e_s <= TOL_BF16, e_s


def test_kcp_workload_segmented_tc(cuda_device):
    """B=1, H=HV=16, T=65536 as 8 segments of 8192: segments with transitions in
    one batched launch, the combine, and the rerun from the combined states give
    the unsegmented pass.  Every head's o and final state are compared with the
    oracle's single pass, and every segment's transition M_seg and local state
    with the oracle run on that segment from the zero state."""
    import numpy as np
    w = workloads.workload("kcp_bf16")
    inp = workloads.chunk_inputs(w)
    d = to_device(inp, cuda_device)
    L = w.T // w.n_seg
    seg = {n: d[n].view(w.n_seg, L, *d[n].shape[2:]) for n in ("q", "k", "v", "g", "beta")}
    kw = dict(A_log=d["A_log"], chunk=w.chunk, algo="tc")
    o_none, S_loc, M_loc = kda.kda_chunk_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"],
                                             output_transition=True, output_o=False, **kw)
    assert o_none is None
    S_in = kda.kda_compose(M_loc, S_loc, d["S0"].view(w.HV, 128, 128))
    o_seg, _, _ = kda.kda_chunk_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"],
                                    S0=S_in[:w.n_seg].contiguous(), output_final_state=False, **kw)
    o_full, S_full, _ = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S0=d["S0"], **kw)
    assert fro_rel(to_np(S_in[-1]), to_np(S_full[0])) <= TOL_BF16
    assert max_rel(to_np(o_seg.reshape(o_full.shape)), to_np(o_full)) <= TOL_BF16
    # the whole sequence against the oracle, head by head
    ref = oracle_chunk(inp)
    e_o, e_s = _per_chain_errors(o_seg.reshape(o_full.shape).cpu(), S_in[-1].view(1, w.HV, 128, 128).cpu(), ref)
    assert e_o <= TOL_BF16, e_o
    assert e_s <= TOL_BF16, e_s
    del ref
    # every segment's transition and local state against the oracle from zero
    segs = {n: inp[n].view(w.n_seg, L, *inp[n].shape[2:]) for n in ("q", "k", "v", "g", "beta")}
    rseg = oracle_chunk(dict(segs, A_log=inp["A_log"], dt_bias=None, S0=None), want_M=True)
    M_np, S_np = to_np(M_loc), to_np(S_loc)
    for s_ in range(w.n_seg):
        for hv in range(w.HV):
            assert fro_rel(M_np[s_, hv], rseg["M_T"][s_, hv]) <= TOL_BF16
            assert fro_rel(S_np[s_, hv], rseg["S_T"][s_, hv]) <= TOL_BF16


@pytest.mark.parametrize("algo", ["tc", "simt"])
def test_states_only_pass_skips_o(cuda_device, algo):
    """o = NULL: only the states are computed; S_T and M_T equal those of the
    call that also writes o, bit for bit (the state path does not read o)."""
    w = workloads.Workload("noo", B=2, T=200, H=1, HV=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=44, a_log="uniform", dt_bias_std=0.5, s0_std=0.05)
    d = to_device(workloads.chunk_inputs(w), cuda_device)
    o1, S1, M1 = run_gpu(d, w, algo, want_M=True)
    o2, S2, M2 = run_gpu(d, w, algo, want_M=True, output_o=False)
    assert o2 is None and o1 is not None
    assert torch.equal(S1, S2) and torch.equal(M1, M2)


def test_prefill_bf16_seqpar(cuda_device):
    """The prefill workload (16 chains on 148 SMs) through the sequence-parallel
    forward: the policy cuts each sequence into 8 segments of 512 tokens; every
    chain's o and S_T are compared with the oracle's single pass (o element by
    element, S_T by Frobenius norm), the initial state S0 included."""
    w = workloads.workload("prefill_bf16")
    inp = workloads.chunk_inputs(w)
    d = to_device(inp, cuda_device)
    assert kda.seq_segments(w.B, w.HV, w.T, w.chunk,
                            torch.cuda.get_device_properties(cuda_device).multi_processor_count) > 1
    o, S_T = kda.kda_chunk_fwd_seqpar(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                                      dt_bias=d["dt_bias"], S0=d["S0"], chunk=w.chunk)
    e_o, e_s = _per_chain_errors(o.cpu(), S_T.cpu(), oracle_chunk(inp))
    assert e_o <= TOL_BF16, e_o
    assert e_s <= TOL_BF16, e_s


@pytest.mark.parametrize("segments", [3, 8])
def test_seqpar_ragged_batched(cuda_device, segments):
    """Two batch rows, grouped heads, segments whose length is not a multiple
    of the chunk (ragged last chunk in every segment), against the oracle."""
    w = workloads.workload("prefill_bf16", B=2, H=2, HV=4, T=600, seed=91)
    inp = workloads.chunk_inputs(w)
    d = to_device(inp, cuda_device)
    o, S_T = kda.kda_chunk_fwd_seqpar(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                                      dt_bias=d["dt_bias"], S0=d["S0"], chunk=w.chunk, segments=segments)
    ref = oracle_chunk(inp)
    check(o, S_T, None, ref, "bf16", "tc")
