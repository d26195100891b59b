"""Runs the host-emulated SIMT forward (with per-chunk states) and backward
kernels on small seeded problems and compares them with the FP64 oracle.

TEST INFRASTRUCTURE, started by tests/test_host_emu_cpu.py in a process with
the AddressSanitizer runtime preloaded.  Prints one line per case and exits
non-zero on a mismatch (an out-of-bounds access aborts the process first).
"""
import ctypes
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
sys.path.insert(0, os.path.dirname(HERE))
import oracle  # noqa: E402
import workloads  # noqa: E402
from helpers import TOL_BF16, TOL_F32, max_rel, to_np  # noqa: E402
from oracle import backward  # noqa: E402

_P, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


class ChunkParams(ctypes.Structure):       # kda::ChunkParams
    _fields_ = [(n, _I) for n in ("B", "T", "H", "HV", "Dk", "Dv", "C", "group")] + \
        [(n, _F) for n in ("g_min", "scale", "l2_eps")] + \
        [(n, _I) for n in ("l2norm", "beta_sigmoid", "gate_in")] + \
        [(n, _P) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0", "o", "S_T", "M_T",
                           "S_chunks")] + [("withhold_ready", _I)]


class BwdParams(ctypes.Structure):         # kda::BwdParams
    _fields_ = [(n, _I) for n in ("B", "T", "H", "HV", "Dk", "Dv", "C", "group")] + \
        [(n, _F) for n in ("g_min", "scale", "l2_eps")] + \
        [(n, _I) for n in ("l2norm", "beta_sigmoid", "gate_in")] + \
        [(n, _P) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S_chunks", "dout", "dS_T",
                           "dq", "dk", "dv", "dg", "dbeta", "dS0", "dA_log", "ddt_bias")]


GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dS0", "dA_log", "ddt_bias")


def _ptr(t):
    return None if t is None or t.numel() == 0 else t.data_ptr()


def run_case(lib, B, T, H, HV, Dk, Dv, C, dtype, flags, scale, seed):
    w = workloads.Workload("emu", B=B, T=T, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=C, dtype=dtype, seed=seed,
                           a_log="uniform", dt_bias_std=0.5, s0_std=0.2)
    inp = workloads.chunk_inputs(w) if flags else workloads.activated_inputs(w)
    gen = torch.Generator().manual_seed(seed + 7)
    dout = torch.randn((B, T, HV, Dv), generator=gen).to(inp["q"].dtype)
    dS_T = torch.randn((B, HV, Dk, Dv), generator=gen)
    bf16 = int(dtype == "bf16")
    NC = -(-T // C)
    o = torch.zeros((B, T, HV, Dv), dtype=inp["q"].dtype)
    S_T = torch.zeros((B, HV, Dk, Dv))
    S_ch = torch.full((B, HV, NC, Dk, Dv), float("nan"))
    fl = int(flags)
    fp = ChunkParams(B, T, H, HV, Dk, Dv, C, HV // H, -5.0, scale, 1e-6, fl, fl, fl,
                     *(_ptr(inp[n]) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0")),
                     _ptr(o), _ptr(S_T), None, _ptr(S_ch), 0)
    if T > 0 and lib.emu_chunk_fwd(ctypes.byref(fp), bf16) != 0:
        raise RuntimeError("forward emulation refused the shape")
    out = {"dq": torch.zeros((B, T, H, Dk)), "dk": torch.zeros((B, T, H, Dk)),
           "dv": torch.zeros((B, T, HV, Dv)), "dg": torch.zeros((B, T, HV, Dk)), "dbeta": torch.zeros((B, T, HV)),
           "dS0": torch.zeros((B, HV, Dk, Dv)), "dA_log": torch.zeros(HV) if flags else None,
           "ddt_bias": torch.zeros((HV, Dk)) if flags else None}
    bp = BwdParams(B, T, H, HV, Dk, Dv, C, HV // H, -5.0, scale, 1e-6, fl, fl, fl,
                   *(_ptr(inp[n]) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias")),
                   _ptr(S_ch), _ptr(dout), _ptr(dS_T), *(_ptr(out[n]) for n in GRADS))
    if lib.emu_chunk_bwd(ctypes.byref(bp), bf16) != 0:
        raise RuntimeError("backward emulation refused the shape")
    sw = dict(scale=scale, qk_l2norm=flags, beta_sigmoid=flags, gate_in=flags)
    args = [to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")]
    kw = dict(A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]), S0=to_np(inp["S0"]))
    err = {}            # each entry is held to TOL (o of bf16 inputs rescaled to its own bar)
    if T > 0:
        ref = oracle.kda_fwd(*args, **kw, **sw)
        # o is stored in the input dtype: bf16 rounding puts it under the bf16 bar
        err["o"] = max_rel(to_np(o), ref["o"]) * (TOL / TOL_BF16 if dtype == "bf16" else 1.0)
        err["S_T"] = max_rel(to_np(S_T), ref["S_T"])
        for c in range(1, NC):
            pre = oracle.kda_fwd(*(a[:, : c * C] for a in args), **kw, **sw)
            err["S_chunks"] = max(err.get("S_chunks", 0.0), max_rel(to_np(S_ch[:, :, c]), pre["S_T"]))
        err["S_chunks0"] = max_rel(to_np(S_ch[:, :, 0]), to_np(inp["S0"]))
    gr = backward.kda_backward(*args, **kw, do=to_np(dout), dS_T=to_np(dS_T), **sw)
    names = {"dq": "q", "dk": "k", "dv": "v", "dg": "g", "dbeta": "beta", "dS0": "S0"}
    if flags:
        names.update(dA_log="A_log", ddt_bias="dt_bias")
    for n, rn in names.items():
        err[n] = max_rel(to_np(out[n]), gr[rn])
    return err


CASES = [
    # B, T, H, HV, Dk, Dv, C, dtype, flags, scale, seed
    (1, 37, 1, 2, 16, 12, 16, "f32", True, 1.0, 1),      # ragged last chunk, grouped heads
    (2, 50, 1, 2, 32, 40, 16, "f32", True, 0.5, 2),      # two column slices, one ragged
    (1, 70, 2, 2, 16, 16, 32, "f32", False, 1.0, 3),     # switches off
    (1, 45, 1, 1, 24, 20, 16, "bf16", True, 1.0, 4),     # bf16 inputs
    (1, 70, 1, 1, 128, 128, 64, "f32", True, 1.0, 5),    # full head size, C = 64, ragged
    (2, 0, 1, 2, 16, 16, 16, "f32", True, 1.0, 6),       # empty sequence
]
TOL = TOL_F32

if __name__ == "__main__":
    lib = ctypes.CDLL(os.path.join(HERE, "_build", "libkda_host_emu.so"))
    assert lib.emu_sizeof_chunk_params() == ctypes.sizeof(ChunkParams)
    assert lib.emu_offsetof_withhold_ready() == ChunkParams.withhold_ready.offset
    assert lib.emu_sizeof_bwd_params() == ctypes.sizeof(BwdParams)
    assert lib.emu_offsetof_ddt_bias() == BwdParams.ddt_bias.offset
    bad = 0
    for case in CASES:
        err = run_case(lib, *case)
        worst = max(err.values()) if err else 0.0
        bad += worst > TOL
        print(case, "ok" if worst <= TOL else "MISMATCH", " ".join("%s=%.1e" % kv for kv in err.items()),
              flush=True)
    sys.exit(1 if bad else 0)
