"""Context-parallel forward (kcp_chunk_fwd) across two gloo ranks on CPU.

The host logic (segment order, the all-gather of (M, S_seg), the combine and
the rerun from the incoming state) runs exactly as on GPUs; the compute steps
are the FP64 oracle, so every rank's output rows and the final state must
equal the oracle's single pass over the whole sequence to rounding.
"""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

SEGMENTS = [40, 56]          # unequal segment lengths, rank order


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = torch.Generator().manual_seed(7)
    B, H, HV, D, T = 1, 1, 2, 8, sum(SEGMENTS)
    x = {"q": torch.randn(B, T, H, D, generator=g, dtype=torch.float64),
         "k": torch.randn(B, T, H, D, generator=g, dtype=torch.float64),
         "v": torch.randn(B, T, HV, D, generator=g, dtype=torch.float64),
         "g": torch.randn(B, T, HV, D, generator=g, dtype=torch.float64),
         "beta": torch.randn(B, T, HV, generator=g, dtype=torch.float64),
         "A_log": torch.rand(HV, generator=g, dtype=torch.float64) * 2 - 1,
         "dt_bias": torch.randn(HV, D, generator=g, dtype=torch.float64) * 0.5,
         "S0": torch.randn(B, HV, D, D, generator=g, dtype=torch.float64) * 0.05}
    return x


class OracleOps:
    """The compute steps of kcp_chunk_fwd on the FP64 oracle."""

    @staticmethod
    def forward(q, k, v, g, beta, S0, want_M, **kw):
        import oracle
        r = oracle.kda_fwd(q.numpy(), k.numpy(), v.numpy(), g.numpy(), beta.numpy(),
                           A_log=kw["A_log"].numpy(), dt_bias=kw["dt_bias"].numpy(),
                           S0=None if S0 is None else S0.numpy(), g_min=kw["g_min"],
                           scale=kw["scale"], l2_eps=kw["l2_eps"],
                           qk_l2norm=kw["qk_l2norm_in_kernel"], beta_sigmoid=kw["beta_sigmoid_in_kernel"],
                           gate_in=kw["gate_in_kernel"], want_state=True, want_M=want_M)
        M = torch.from_numpy(r["M_T"]) if want_M else None
        return torch.from_numpy(r["o"]), torch.from_numpy(r["S_T"]), M

    @staticmethod
    def compose(M, S_seg, S_init):
        import oracle
        return torch.from_numpy(oracle.kda_compose(M.numpy(), S_seg.numpy(),
                                                   None if S_init is None else S_init.numpy()))

    @staticmethod
    def all_gather(t, world, group):
        from gated_delta_rule_157_b200.kcp import _KernelOps
        return _KernelOps.all_gather(t, world, group)


def _rank_main(rank, world, port, out_dir, segments=None):
    global SEGMENTS
    if segments is not None:
        SEGMENTS = segments
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from gated_delta_rule_157_b200.kcp import kcp_chunk_fwd
    x = _inputs()
    lo = sum(SEGMENTS[:rank])
    hi = lo + SEGMENTS[rank]
    seg = {n: x[n][:, lo:hi].contiguous() for n in ("q", "k", "v", "g", "beta")}
    o, S_T = kcp_chunk_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"], A_log=x["A_log"],
                           dt_bias=x["dt_bias"], S0=x["S0"], chunk=16, ops=OracleOps)
    np.save(os.path.join(out_dir, "o%d.npy" % rank), o.numpy())
    np.save(os.path.join(out_dir, "S%d.npy" % rank), S_T.numpy())
    dist.destroy_process_group()


def _check_against_single_pass(tmp_path, segments):
    import oracle
    global SEGMENTS
    SEGMENTS = segments
    x = _inputs()
    ref = oracle.kda_fwd(*(x[n].numpy() for n in ("q", "k", "v", "g", "beta")), A_log=x["A_log"].numpy(),
                         dt_bias=x["dt_bias"].numpy(), S0=x["S0"].numpy())
    lo = 0
    for r, L in enumerate(segments):
        o = np.load(tmp_path / ("o%d.npy" % r))
        S = np.load(tmp_path / ("S%d.npy" % r))
        assert o.shape[1] == L
        if L:
            assert np.abs(o - ref["o"][:, lo:lo + L]).max() <= 1e-10 * max(1.0, np.abs(ref["o"]).max())
        assert np.abs(S - ref["S_T"]).max() <= 1e-10 * max(1.0, np.abs(ref["S_T"]).max())
        lo += L


def test_two_rank_context_parallel_equals_single_pass(tmp_path):
    segments = [40, 56]
    mp.spawn(_rank_main, args=(len(segments), _free_port(), str(tmp_path), segments), nprocs=len(segments),
             join=True)
    _check_against_single_pass(tmp_path, segments)


def test_three_ranks_with_an_empty_segment(tmp_path):
    """A rank with no tokens contributes the identity transition and a zero state."""
    segments = [30, 0, 66]
    mp.spawn(_rank_main, args=(len(segments), _free_port(), str(tmp_path), segments), nprocs=len(segments),
             join=True)
    _check_against_single_pass(tmp_path, segments)
