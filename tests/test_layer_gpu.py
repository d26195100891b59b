"""GPU parity of the layer prologue (kda_short_conv) and epilogue
(kda_output_gate) against the FP64 oracle (oracle/layer.py) on identical inputs.

Bar: the outputs are bf16, rounded once from fp32 arithmetic on the exact bf16
inputs, so each element is within half a bf16 ulp (2^-9 relative) plus fp32
and SFU rounding; the test allows 2^-7 of the largest |reference| (4x margin).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_157_b200 as kda
from oracle import layer

pytestmark = pytest.mark.gpu
TOL = 2.0 ** -7


def _bf16(a, dev):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(dev)


def _f32(a, dev):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(dev)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rel(a, ref):
    return np.abs(a - ref).max() / max(np.abs(ref).max(), 1e-30)


@pytest.mark.parametrize("K,head_dim,act,T,with_state", [
    (4, 128, True, 100, False),     # q/k prologue, ragged token blocks
    (4, 0, True, 64, True),         # v prologue, carried window in
    (4, 0, False, 33, True),        # plain convolution
    (2, 128, True, 5, True),        # fewer taps
    (1, 0, False, 7, False),        # pointwise
])
def test_short_conv(cuda_device, K, head_dim, act, T, with_state):
    rng = np.random.default_rng(100 + T + K)
    B, C = 2, 256
    x = _bf16(rng.standard_normal((B, T, C)), cuda_device)
    w = rng.standard_normal((C, K)).astype(np.float32)
    bias = rng.standard_normal(C).astype(np.float32) * 0.1
    st = _bf16(rng.standard_normal((B, K - 1, C)), cuda_device) if with_state else None
    y, so = kda.kda_short_conv(x, _f32(w, cuda_device), _f32(bias, cuda_device), head_dim=head_dim,
                               silu=act, state_in=st, want_state=True)
    ref, ref_st = layer.prologue(_np(x), w, bias, None if st is None else _np(st), head_dim=head_dim,
                                 act=act)
    assert _rel(_np(y), ref) <= TOL
    assert np.array_equal(_np(so), ref_st)            # carried tokens are copied exactly


def test_short_conv_tiled_groups_and_tiles(cuda_device):
    """Rows of several 256-channel groups and several 128-token tiles (the
    tiled kernel): ragged last tile, carried window in and out, three taps."""
    rng = np.random.default_rng(41)
    B, T, C, K = 3, 300, 768, 3
    x = _bf16(rng.standard_normal((B, T, C)), cuda_device)
    w = rng.standard_normal((C, K)).astype(np.float32)
    bias = rng.standard_normal(C).astype(np.float32) * 0.1
    st = _bf16(rng.standard_normal((B, K - 1, C)), cuda_device)
    y, so = kda.kda_short_conv(x, _f32(w, cuda_device), _f32(bias, cuda_device), head_dim=128, state_in=st,
                               want_state=True)
    ref, ref_st = layer.prologue(_np(x), w, bias, _np(st), head_dim=128, act=True)
    assert _rel(_np(y), ref) <= TOL
    assert np.array_equal(_np(so), ref_st)
    assert kda.kda_device_status() is None


@pytest.mark.parametrize("C", [128, 512])
def test_short_conv_decode_steps_equal_one_run(cuda_device, C):
    """One token at a time with the carried window equals the whole sequence
    (C = 128: the warp kernel; C = 512: the tiled kernel, both ways)."""
    rng = np.random.default_rng(5)
    B, T = 3, 9
    x = _bf16(rng.standard_normal((B, T, C)), cuda_device)
    w = _f32(rng.standard_normal((C, 4)), cuda_device)
    full = kda.kda_short_conv(x, w, head_dim=128)
    state = torch.zeros((B, 3, C), dtype=torch.bfloat16, device=cuda_device)
    steps = []
    for t in range(T):
        yt, state = kda.kda_short_conv(x[:, t:t + 1].contiguous(), w, head_dim=128, state_in=state,
                                       want_state=True)
        steps.append(yt)
    assert torch.equal(torch.cat(steps, dim=1), full)


def test_short_conv_identity_init_and_empty(cuda_device):
    rng = np.random.default_rng(6)
    x = _bf16(rng.standard_normal((1, 40, 128)), cuda_device)
    w = torch.zeros((128, 4), dtype=torch.float32, device=cuda_device)
    w[:, -1] = 1.0
    assert torch.equal(kda.kda_short_conv(x, w, silu=False), x)
    st = _bf16(rng.standard_normal((1, 3, 128)), cuda_device)
    _, so = kda.kda_short_conv(x[:, :0].contiguous(), w, state_in=st, want_state=True)
    assert torch.equal(so, st)


@pytest.mark.parametrize("N,HV,with_w", [(37, 4, True), (8, 1, False)])
def test_output_gate(cuda_device, N, HV, with_w):
    rng = np.random.default_rng(N)
    o = _bf16(rng.standard_normal((N, HV, 128)) * 3, cuda_device)
    g = _bf16(rng.standard_normal((N, HV, 128)) * 2, cuda_device)
    wt = rng.standard_normal(128).astype(np.float32) if with_w else None
    y = kda.kda_output_gate(o, g, None if wt is None else _f32(wt, cuda_device))
    ref = layer.output_gate(_np(o), _np(g), wt)
    assert _rel(_np(y), ref) <= TOL


def test_layer_core_composition(cuda_device):
    """Prologue -> core -> epilogue (the layer without its projections) against the
    oracle's composition: q, k, v from the short convolutions, the core with its
    in-kernel gate and beta, the output gate on o.

    Each stage is held to its own bar on the previous stage's actual output:
    the prologue to 2^-7 of max|ref| (bf16 output), the core to the bf16 core
    bar 2e-2 of max|o| on the prologue's bf16 rows, the epilogue to 2^-7 on the
    core's o.  The composed output is also compared with the oracle's whole
    composition on the rows whose RMS is at least a tenth of the largest: the
    epilogue divides every row by its own RMS, so a row far below the tensor's
    largest carries the core's absolute error (bounded relative to max|o|)
    amplified by that ratio, which no max-relative bar on the composition
    covers."""
    import workloads
    from helpers import oracle_chunk, to_device
    rng = np.random.default_rng(9)
    w = workloads.Workload("layer", B=1, T=130, H=1, HV=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=71, a_log="uniform", dt_bias_std=0.5)
    inp = to_device(workloads.chunk_inputs(w), cuda_device)
    B, T = w.B, w.T
    wq, wk, wv = (rng.standard_normal((C, 4)).astype(np.float32) * 0.5 for C in (128, 128, 256))
    q = kda.kda_short_conv(inp["q"].view(B, T, 128), _f32(wq, cuda_device), head_dim=128).view(B, T, 1, 128)
    k = kda.kda_short_conv(inp["k"].view(B, T, 128), _f32(wk, cuda_device), head_dim=128).view(B, T, 1, 128)
    v = kda.kda_short_conv(inp["v"].view(B, T, 256), _f32(wv, cuda_device)).view(B, T, 2, 128)
    o, _, _ = kda.kda_chunk_fwd(q, k, v, inp["g"], inp["beta"], A_log=inp["A_log"], dt_bias=inp["dt_bias"],
                                chunk=64, algo="tc")
    gate = _bf16(rng.standard_normal((B, T, 2, 128)), cuda_device)
    y = kda.kda_output_gate(o, gate)
    # prologue stage: FP64 on the same bf16 inputs
    qr, _ = layer.prologue(_np(inp["q"]).reshape(B, T, 128), wq, head_dim=128)
    kr, _ = layer.prologue(_np(inp["k"]).reshape(B, T, 128), wk, head_dim=128)
    vr, _ = layer.prologue(_np(inp["v"]).reshape(B, T, 256), wv)
    for got, want in ((q, qr), (k, kr), (v, vr)):
        assert _rel(_np(got).reshape(want.shape), want) <= 2.0 ** -7
    # core stage: the oracle on the prologue's own bf16 rows (its q/k norm is
    # idempotent on normalised rows)
    core_in = {"q": _np(q), "k": _np(k), "v": _np(v), "g": _np(inp["g"]), "beta": _np(inp["beta"]),
               "A_log": _np(inp["A_log"]), "dt_bias": _np(inp["dt_bias"]), "S0": None}
    o_ref = oracle_chunk(core_in)["o"]
    assert _rel(_np(o), o_ref) <= 2e-2
    # epilogue stage: the oracle gate on the core's own o
    assert _rel(_np(y), layer.output_gate(_np(o), _np(gate))) <= 2.0 ** -7
    # the whole composition on the rows the RMS division does not amplify
    ref = layer.output_gate(o_ref, _np(gate))
    rms = np.sqrt((o_ref ** 2).mean(-1))
    keep = rms >= 0.1 * rms.max()
    assert keep.sum() >= keep.size // 2
    assert _rel(_np(y)[keep], ref[keep]) <= 2e-2
