"""Failure path of the tensor-core chunk kernel, exercised without a GPU fault.

kda_debug_chunk_stall launches the kernel with its prep warps never handing a
chunk over, so the state warps' bounded wait gives up (about two seconds): the
kernel must record the device error word and return, kda_device_status must
report KDA_ERR_TIMEOUT, and the context must stay usable for the next call,
whose result is checked against the oracle.
"""
import time

import pytest

import gated_delta_rule_157_b200 as kda
import workloads
from helpers import TOL_BF16, fro_rel, max_rel, oracle_chunk, to_device, to_np

pytestmark = pytest.mark.gpu


def _case(T=192, want_M=True):
    w = workloads.Workload("stall", B=1, T=T, H=1, HV=2, Dk=128, Dv=128, chunk=64, dtype="bf16",
                           seed=51, s0_std=0.02)
    return w, workloads.chunk_inputs(w)


def _run(d, w, want_M, **kw):
    return kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                             dt_bias=d["dt_bias"], S0=d["S0"], chunk=w.chunk,
                             output_transition=want_M, algo="tc", **kw)


def test_withheld_handover_times_out_and_context_recovers(cuda_device):
    w, inp = _case()
    d = to_device(inp, cuda_device)
    t0 = time.perf_counter()
    _run(d, w, True, _withhold_ready=True)
    with pytest.raises(kda.KdaError) as err:
        kda.kda_device_status()
    elapsed = time.perf_counter() - t0
    assert err.value.status == 6                      # KDA_ERR_TIMEOUT
    assert elapsed < 60.0
    # The error word was cleared and the context still works.
    kda.kda_device_status()
    ref = oracle_chunk(inp, want_M=True)
    o, S_T, M_T = _run(d, w, True)
    kda.kda_device_status()
    assert max_rel(to_np(o), ref["o"]) <= TOL_BF16
    assert fro_rel(to_np(S_T), ref["S_T"]) <= TOL_BF16
    assert fro_rel(to_np(M_T), ref["M_T"]) <= TOL_BF16


def test_stall_hook_only_for_the_tensor_core_kernel(cuda_device):
    w, inp = _case(T=64, want_M=False)
    d = to_device(inp, cuda_device)
    with pytest.raises(kda.KdaError) as err:
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], A_log=d["A_log"],
                          dt_bias=d["dt_bias"], chunk=w.chunk, algo="simt", _withhold_ready=True)
    assert err.value.status == 2                      # KDA_ERR_UNSUPPORTED
