"""The autograd binding (gated_delta_rule_157_b200/autograd.py) driven through
the host-emulated kernels: the library calls it makes are replaced by ones
that run the same kernels compiled for the host on CPU tensors, so the
binding's argument routing, gradient order and dtype handling are checked
against the FP64 oracle without a GPU.

TEST INFRASTRUCTURE, started by tests/test_host_emu_cpu.py with the
AddressSanitizer runtime preloaded; exits non-zero on a mismatch."""
import ctypes
import os
import sys

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)
import run_parity as R  # noqa: E402
import workloads  # noqa: E402
from gated_delta_rule_157_b200 import _lib, autograd  # noqa: E402
from helpers import TOL_F32, max_rel, sum_rel, to_np  # noqa: E402
from oracle import backward  # noqa: E402

lib = ctypes.CDLL(os.path.join(HERE, "_build", "libkda_host_emu.so"))


def _p(t):
    return None if t is None else t.data_ptr()


def host_fwd(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, chunk=64, g_min=-5.0, scale=1.0,
             l2_eps=1e-6, qk_l2norm_in_kernel=True, beta_sigmoid_in_kernel=True, gate_in_kernel=True,
             S_chunks=None, g_per_head=False, algo="auto", **_):
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    o = torch.zeros((B, T, HV, Dv), dtype=q.dtype)
    S_T = torch.zeros((B, HV, Dk, Dv))
    fp = R.ChunkParams(B, T, H, HV, Dk, Dv, chunk, HV // H, g_min, scale, l2_eps, int(qk_l2norm_in_kernel),
                       int(beta_sigmoid_in_kernel), _lib._gate_code(gate_in_kernel), int(g_per_head),
                       *(_p(x) for x in (q, k, v, g, beta, A_log, dt_bias, S0, o, S_T)), None, _p(S_chunks), 0)
    assert lib.emu_chunk_fwd(ctypes.byref(fp), int(q.dtype == torch.bfloat16)) == 0
    return o, S_T, None


def host_bwd(q, k, v, g, beta, S_chunks, dout, dS_T=None, *, A_log=None, dt_bias=None, chunk=64, g_min=-5.0,
             scale=1.0, l2_eps=1e-6, qk_l2norm_in_kernel=True, beta_sigmoid_in_kernel=True, gate_in_kernel=True,
             want_dS0=True, g_per_head=False, **_):
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    gk = () if g_per_head else (Dk,)
    out = {"dq": torch.zeros((B, T, H, Dk)), "dk": torch.zeros((B, T, H, Dk)), "dv": torch.zeros((B, T, HV, Dv)),
           "dg": torch.zeros((B, T, HV) + gk), "dbeta": torch.zeros((B, T, HV)),
           "dS0": torch.zeros((B, HV, Dk, Dv)) if want_dS0 else None,
           "dA_log": torch.zeros(HV) if gate_in_kernel else None,
           "ddt_bias": torch.zeros((HV,) + gk) if (gate_in_kernel and dt_bias is not None) else None}
    bp = R.BwdParams(B, T, H, HV, Dk, Dv, chunk, HV // H, g_min, scale, l2_eps, int(qk_l2norm_in_kernel),
                     int(beta_sigmoid_in_kernel), _lib._gate_code(gate_in_kernel), int(g_per_head),
                     *(_p(x) for x in (q, k, v, g, beta, A_log, dt_bias, S_chunks, dout, dS_T)),
                     *(_p(out[n]) for n in R.GRADS))
    assert lib.emu_chunk_bwd(ctypes.byref(bp), int(q.dtype == torch.bfloat16)) == 0
    return out


def main():
    _lib.kda_chunk_fwd = host_fwd
    _lib.kda_chunk_bwd = host_bwd
    bad = 0
    for per_head, gate in ((False, "bounded"), (True, "softplus")):
        w = workloads.Workload("ag", B=1, T=45, H=1, HV=2, Dk=16, Dv=16, chunk=16, dtype="f32", seed=40,
                               a_log="uniform", dt_bias_std=0.5, s0_std=0.2)
        inp = workloads.chunk_inputs(w)
        if per_head:
            inp["g"] = inp["g"][..., 0].contiguous()
            inp["dt_bias"] = inp["dt_bias"][:, 0].contiguous()
        gen = torch.Generator().manual_seed(41)
        do = torch.randn((1, 45, 2, 16), generator=gen)
        dS = torch.randn((1, 2, 16, 16), generator=gen)
        leaves = {n: inp[n].clone().requires_grad_(True)
                  for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0")}
        o, S_T = autograd.kda_chunk(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["beta"],
                                    A_log=leaves["A_log"], dt_bias=leaves["dt_bias"], S0=leaves["S0"], chunk=16,
                                    gate_in_kernel=gate, g_per_head=per_head)
        ((o * do).sum() + (S_T * dS).sum()).backward()
        ref = backward.kda_backward(*(to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                    A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]),
                                    S0=to_np(inp["S0"]), do=to_np(do), dS_T=to_np(dS), gate=gate,
                                    per_head=per_head)
        errs = {n: (sum_rel(to_np(leaves[n].grad), ref[n], ref[n + "_l1"]) if n in ("A_log", "dt_bias")
                    else max_rel(to_np(leaves[n].grad), ref[n])) for n in leaves}
        worst = max(errs.values())
        bad += worst > TOL_F32
        print(gate, "per_head" if per_head else "per_channel", "ok" if worst <= TOL_F32 else "MISMATCH",
              " ".join("%s=%.1e" % kv for kv in errs.items()), flush=True)
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main())
