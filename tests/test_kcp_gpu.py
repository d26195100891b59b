"""kcp_chunk_fwd on one GPU (a one-rank group: segment from zero, combine with
the initial state, rerun) against the FP64 oracle's single pass."""
import pytest

import gated_delta_rule_157_b200 as kda
import workloads
from helpers import TOL_BF16, fro_rel, max_rel, oracle_chunk, to_device, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("algo", ["tc", "simt"])
def test_one_rank_context_parallel(cuda_device, algo):
    w = workloads.Workload("kcp1", B=2, T=200, H=1, HV=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=61, a_log="uniform", dt_bias_std=0.5, s0_std=0.05)
    inp = workloads.chunk_inputs(w)
    ref = oracle_chunk(inp)
    d = to_device(inp, cuda_device)
    o, S_T = kda.kcp_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                               dt_bias=d["dt_bias"], S0=d["S0"], chunk=w.chunk, algo=algo)
    kda.kda_device_status()
    assert max_rel(to_np(o), ref["o"]) <= TOL_BF16
    assert fro_rel(to_np(S_T), ref["S_T"]) <= TOL_BF16
