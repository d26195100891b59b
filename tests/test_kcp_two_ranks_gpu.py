"""Context-parallel forward (kcp_chunk_fwd) with two ranks whose compute runs
in the library's CUDA kernels.

Two processes share the one GPU; each runs its segment of one sequence
(unequal, ragged lengths) with the kernels, and the ranks exchange their
(M_seg, S_seg) blocks through a gloo group (host copies of the device
blocks), combine them and rerun their segment from its incoming state
(page "Implémenter KDA", "Test 3 - le balayage préfixe sur plusieurs
rangs").  No kernel of one rank waits on the other's: the only exchange is
the host-side all-gather.  Every rank's o rows and the final state must match
the oracle's single pass over the whole sequence at the bf16 bars.
"""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

pytestmark = pytest.mark.gpu

SEGMENTS = [200, 328]        # rank order; neither is a multiple of the chunk


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    import workloads
    return workloads.Workload("kcp2", B=1, T=sum(SEGMENTS), H=1, HV=2, Dk=128, Dv=128, chunk=64,
                              dtype="bf16", seed=71, a_log="uniform", dt_bias_std=0.5, s0_std=0.05)


def _rank_main(rank, world, port, out_dir, algo):
    import torch.distributed as dist
    import workloads
    import gated_delta_rule_157_b200 as kda
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = _workload()
    x = workloads.chunk_inputs(w, z_mean=-3.0)     # slower decay: the incoming state matters
    lo = sum(SEGMENTS[:rank])
    hi = lo + SEGMENTS[rank]
    seg = {n: x[n][:, lo:hi].contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")}
    o, S_T = kda.kcp_chunk_fwd(seg["q"], seg["k"], seg["v"], seg["g"], seg["beta"], A_log=x["A_log"].to(dev),
                               dt_bias=x["dt_bias"].to(dev), S0=x["S0"].to(dev), chunk=w.chunk, algo=algo)
    kda.kda_device_status()
    np.save(os.path.join(out_dir, "o%d.npy" % rank), o.float().cpu().numpy())
    np.save(os.path.join(out_dir, "S%d.npy" % rank), S_T.cpu().numpy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("algo", ["tc", "simt"])
def test_two_ranks_on_the_kernels_equal_the_single_pass(cuda_device, tmp_path, algo):
    from helpers import TOL_BF16, fro_rel, max_rel, oracle_chunk
    import workloads
    mp.spawn(_rank_main, args=(len(SEGMENTS), _free_port(), str(tmp_path), algo), nprocs=len(SEGMENTS),
             join=True)
    ref = oracle_chunk(workloads.chunk_inputs(_workload(), z_mean=-3.0))
    lo = 0
    for r, L in enumerate(SEGMENTS):
        o = np.load(tmp_path / ("o%d.npy" % r))
        S = np.load(tmp_path / ("S%d.npy" % r))
        assert o.shape[1] == L
        assert max_rel(o, ref["o"][:, lo:lo + L]) <= TOL_BF16
        assert fro_rel(S, ref["S_T"]) <= TOL_BF16
        lo += L
