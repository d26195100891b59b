"""Sequence-parallel forward on one GPU (kda_chunk_fwd_seqpar): the host
logic on CPU, with the FP64 oracle as the compute steps.

Cutting every sequence into segments, running them from zero with their
transitions, composing the incoming states and rerunning must equal one pass
over the whole sequences to rounding (the composition identity of page
"Implémenter KDA", Tests 2 and 3), for every batch row, with and without an
initial state.  The segment policy fills the SMs only when the chains leave
them idle.
"""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from test_kcp_dist_cpu import OracleOps  # noqa: E402


class _SeqparOracleOps(OracleOps):
    @staticmethod
    def compose_into(M, S_seg, S_init, S_in):
        S_in.copy_(OracleOps.compose(M, S_seg, S_init))


def _inputs(B, T, H, HV, D, seed):
    g = torch.Generator().manual_seed(seed)
    return {"q": torch.randn(B, T, H, D, generator=g, dtype=torch.float64),
            "k": torch.randn(B, T, H, D, generator=g, dtype=torch.float64),
            "v": torch.randn(B, T, HV, D, generator=g, dtype=torch.float64),
            "g": torch.randn(B, T, HV, D, generator=g, dtype=torch.float64),
            "beta": torch.randn(B, T, HV, generator=g, dtype=torch.float64),
            "A_log": torch.rand(HV, generator=g, dtype=torch.float64) * 2 - 1,
            "dt_bias": torch.randn(HV, D, generator=g, dtype=torch.float64) * 0.5,
            "S0": torch.randn(B, HV, D, D, generator=g, dtype=torch.float64) * 0.05}


@pytest.mark.parametrize("B,T,segments,with_S0", [(2, 96, 4, True), (1, 90, 3, False), (2, 40, 1, True)])
def test_seqpar_equals_single_pass(B, T, segments, with_S0):
    from gated_delta_rule_157_b200.kcp import kda_chunk_fwd_seqpar
    import oracle
    x = _inputs(B, T, 1, 2, 8, seed=11 + T)
    S0 = x["S0"] if with_S0 else None
    kw = dict(A_log=x["A_log"], dt_bias=x["dt_bias"], chunk=16, g_min=-5.0, scale=1.0, l2_eps=1e-6,
              qk_l2norm_in_kernel=True, beta_sigmoid_in_kernel=True, gate_in_kernel=True)
    o, S_T = kda_chunk_fwd_seqpar(x["q"], x["k"], x["v"], x["g"], x["beta"], S0=S0, segments=segments,
                                  ops=_SeqparOracleOps, **kw)
    ref = oracle.kda_fwd(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), x["g"].numpy(), x["beta"].numpy(),
                         A_log=x["A_log"].numpy(), dt_bias=x["dt_bias"].numpy(),
                         S0=None if S0 is None else S0.numpy(), g_min=-5.0, scale=1.0, l2_eps=1e-6,
                         qk_l2norm=True, beta_sigmoid=True, gate_in=True, want_state=True)
    assert np.abs(o.numpy() - ref["o"]).max() <= 1e-10 * max(1.0, np.abs(ref["o"]).max())
    assert np.abs(S_T.numpy() - ref["S_T"]).max() <= 1e-10 * max(1.0, np.abs(ref["S_T"]).max())


def test_seqpar_rejects_uneven_segments():
    from gated_delta_rule_157_b200.kcp import kda_chunk_fwd_seqpar
    x = _inputs(1, 30, 1, 1, 4, seed=3)
    with pytest.raises(ValueError):
        kda_chunk_fwd_seqpar(x["q"], x["k"], x["v"], x["g"], x["beta"], segments=4, ops=_SeqparOracleOps,
                             A_log=x["A_log"], dt_bias=x["dt_bias"])


def test_segment_policy():
    from gated_delta_rule_157_b200.kcp import seq_segments
    # 16 chains on 148 SMs: eight segments of 512 tokens (two waves of the
    # states-only pass with its transition CTAs, one output wave)
    assert seq_segments(1, 16, 4096, 64, 148) == 8
    # 128 chains already fill the SMs: one pass
    assert seq_segments(4, 32, 8192, 64, 148) == 1
    # too short to cut (a segment keeps at least two chunks)
    assert seq_segments(1, 2, 64, 64, 148) == 1
    # never more segments than divide T
    n = seq_segments(1, 4, 3 * 512, 64, 148)
    assert 1536 % n == 0
