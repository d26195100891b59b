"""Runs the host-emulated SIMT forward (with per-chunk states) and backward
kernels on small seeded problems and compares them with the FP64 oracle.

TEST INFRASTRUCTURE, started by tests/test_host_emu_cpu.py in a process with
the AddressSanitizer runtime preloaded.  Prints one line per case and exits
non-zero on a mismatch (an out-of-bounds access aborts the process first).
With ``--races LIB`` it runs a few cases through the ThreadSanitizer build
LIB without the oracle (a data race makes the process exit non-zero).
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
from helpers import TOL_BF16, TOL_F32, max_rel, sum_rel, to_np  # noqa: E402
from oracle import backward  # noqa: E402

_P, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


class ChunkParams(ctypes.Structure):       # kda::ChunkParams
    _fields_ = [(n, _I) for n in ("B", "T", "H", "HV", "Dk", "Dv", "C", "group")] + \
        [(n, _F) for n in ("g_min", "scale", "l2_eps")] + \
        [(n, _I) for n in ("l2norm", "beta_sigmoid", "gate_in", "g_per_head")] + \
        [(n, _P) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0", "o", "S_T", "M_T",
                           "S_chunks")] + [("withhold_ready", _I)]


class BwdParams(ctypes.Structure):         # kda::BwdParams
    _fields_ = [(n, _I) for n in ("B", "T", "H", "HV", "Dk", "Dv", "C", "group")] + \
        [(n, _F) for n in ("g_min", "scale", "l2_eps")] + \
        [(n, _I) for n in ("l2norm", "beta_sigmoid", "gate_in", "g_per_head")] + \
        [(n, _P) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S_chunks", "dout", "dS_T",
                           "dq", "dk", "dv", "dg", "dbeta", "dS0", "dA_log", "ddt_bias")]


class StepParams(ctypes.Structure):        # kda::StepParams
    _fields_ = [(n, _I) for n in ("B", "H", "HV", "Dk", "Dv", "group")] + \
        [(n, _F) for n in ("g_min", "scale", "l2_eps")] + \
        [(n, _I) for n in ("l2norm", "beta_sigmoid", "gate_in", "g_per_head")] + \
        [(n, _P) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S", "o")]


class ConvParams(ctypes.Structure):        # kda::ConvParams
    _fields_ = [(n, _I) for n in ("B", "T", "C", "K", "head_dim", "silu")] + [("l2_eps", _F)] + \
        [(n, _P) for n in ("x", "w", "bias", "state_in", "y", "state_out")]


class GateParams(ctypes.Structure):        # kda::GateParams
    _fields_ = [(n, _I) for n in ("N", "HV", "D")] + [("eps", _F)] + \
        [(n, _P) for n in ("o", "gate", "weight", "y")]


GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dS0", "dA_log", "ddt_bias")
GATE_CODE = {None: 0, "bounded": 1, "softplus": 2}


def _gate_np(z, A_log, dt_bias, gate, per_head, Dk):
    """Log-decay [.., HV, Dk] from the raw gate input, through oracle/gates.py."""
    from oracle import gates
    zc = z[..., None] if per_head else z
    bc = None if dt_bias is None else (dt_bias[:, None] if per_head else dt_bias)
    fn = gates.bounded_gate if gate == "bounded" else gates.softplus_gate
    g = fn(zc, A_log, bc)
    return np.ascontiguousarray(np.broadcast_to(g, zc.shape[:-1] + (Dk,)))


def _per_head(inp):
    """The generator's draws cut to one gate value per (token, head)."""
    inp = dict(inp)
    inp["g"] = inp["g"][..., 0].contiguous()
    if inp["dt_bias"] is not None:
        inp["dt_bias"] = inp["dt_bias"][:, 0].contiguous()
    return inp


def _ptr(t):
    return None if t is None or t.numel() == 0 else t.data_ptr()


def run_case(lib, B, T, H, HV, Dk, Dv, C, dtype, flags, scale, seed, gate="bounded", per_head=False, check=True):
    w = workloads.Workload("emu", B=B, T=T, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=C, dtype=dtype, seed=seed,
                           a_log="uniform", dt_bias_std=0.5, s0_std=0.2)
    inp = workloads.chunk_inputs(w) if flags else workloads.activated_inputs(w)
    if per_head:
        inp = _per_head(inp)
    gcode = GATE_CODE[gate] if flags else 0
    gen = torch.Generator().manual_seed(seed + 7)
    dout = torch.randn((B, T, HV, Dv), generator=gen).to(inp["q"].dtype)
    dS_T = torch.randn((B, HV, Dk, Dv), generator=gen)
    bf16 = int(dtype == "bf16")
    NC = -(-T // C)
    o = torch.zeros((B, T, HV, Dv), dtype=inp["q"].dtype)
    S_T = torch.zeros((B, HV, Dk, Dv))
    S_ch = torch.full((B, HV, NC, Dk, Dv), float("nan"))
    fl = int(flags)
    fp = ChunkParams(B, T, H, HV, Dk, Dv, C, HV // H, -5.0, scale, 1e-6, fl, fl, gcode, int(per_head),
                     *(_ptr(inp[n]) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0")),
                     _ptr(o), _ptr(S_T), None, _ptr(S_ch), 0)
    if T > 0 and lib.emu_chunk_fwd(ctypes.byref(fp), bf16) != 0:
        raise RuntimeError("forward emulation refused the shape")
    gk = () if per_head else (Dk,)
    out = {"dq": torch.zeros((B, T, H, Dk)), "dk": torch.zeros((B, T, H, Dk)),
           "dv": torch.zeros((B, T, HV, Dv)), "dg": torch.zeros((B, T, HV) + gk), "dbeta": torch.zeros((B, T, HV)),
           "dS0": torch.zeros((B, HV, Dk, Dv)), "dA_log": torch.zeros(HV) if flags else None,
           "ddt_bias": torch.zeros((HV,) + gk) if flags else None}
    bp = BwdParams(B, T, H, HV, Dk, Dv, C, HV // H, -5.0, scale, 1e-6, fl, fl, gcode, int(per_head),
                   *(_ptr(inp[n]) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias")),
                   _ptr(S_ch), _ptr(dout), _ptr(dS_T), *(_ptr(out[n]) for n in GRADS))
    if lib.emu_chunk_bwd(ctypes.byref(bp), bf16) != 0:
        raise RuntimeError("backward emulation refused the shape")
    if not check:
        return {}
    args = [to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")]
    if flags and (gate != "bounded" or per_head):
        # the oracle's forward takes the variant gates precomputed (oracle/gates.py)
        sw = dict(scale=scale, qk_l2norm=True, beta_sigmoid=True, gate_in=False)
        fargs = args[:3] + [_gate_np(args[3], to_np(inp["A_log"]), to_np(inp["dt_bias"]), gate, per_head, Dk)] + args[4:]
        kw = dict(S0=to_np(inp["S0"]))
    else:
        sw = dict(scale=scale, qk_l2norm=flags, beta_sigmoid=flags, gate_in=flags)
        fargs = args
        kw = dict(A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]), S0=to_np(inp["S0"]))
    err = {}            # each entry is held to TOL (o of bf16 inputs rescaled to its own bar)
    if T > 0:
        ref = oracle.kda_fwd(*fargs, **kw, **sw)
        # o is stored in the input dtype: bf16 rounding puts it under the bf16 bar
        err["o"] = max_rel(to_np(o), ref["o"]) * (TOL / TOL_BF16 if dtype == "bf16" else 1.0)
        err["S_T"] = max_rel(to_np(S_T), ref["S_T"])
        for c in range(1, NC):
            pre = oracle.kda_fwd(*(a[:, : c * C] for a in fargs), **kw, **sw)
            err["S_chunks"] = max(err.get("S_chunks", 0.0), max_rel(to_np(S_ch[:, :, c]), pre["S_T"]))
        err["S_chunks0"] = max_rel(to_np(S_ch[:, :, 0]), to_np(inp["S0"]))
    gr = backward.kda_backward(*args, A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]),
                               S0=to_np(inp["S0"]), do=to_np(dout), dS_T=to_np(dS_T), scale=scale,
                               qk_l2norm=flags, beta_sigmoid=flags, gate_in=flags, gate=gate or "bounded",
                               per_head=per_head)
    names = {"dq": "q", "dk": "k", "dv": "v", "dg": "g", "dbeta": "beta", "dS0": "S0"}
    if flags:
        names.update(dA_log="A_log", ddt_bias="dt_bias")
    for n, rn in names.items():
        if rn in ("A_log", "dt_bias"):     # sums over tokens: against their summed magnitudes
            err[n] = sum_rel(to_np(out[n]), gr[rn], gr[rn + "_l1"])
        else:
            err[n] = max_rel(to_np(out[n]), gr[rn])
    return err


def run_step_case(lib, B, H, HV, Dk, Dv, dtype, gate, per_head, seed, check=True):
    """One decode step against the oracle's step."""
    w = workloads.Workload("emustep", B=B, T=1, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=1, dtype=dtype, seed=seed,
                           a_log="uniform", dt_bias_std=0.5, s0_std=0.3)
    inp = workloads.chunk_inputs(w)
    if per_head:
        inp = _per_head(inp)
    S = inp["S0"].clone()
    x = {n: inp[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "beta")}
    o = torch.zeros((B, HV, Dv), dtype=x["q"].dtype)
    sp = StepParams(B, H, HV, Dk, Dv, HV // H, -5.0, 1.0, 1e-6, 1, 1, GATE_CODE[gate], int(per_head),
                    *(_ptr(x[n]) for n in ("q", "k", "v", "g", "beta")), _ptr(inp["A_log"]),
                    _ptr(inp["dt_bias"]), _ptr(S), _ptr(o))
    lib.emu_step(ctypes.byref(sp), int(dtype == "bf16"))
    if not check:
        return {}
    g = _gate_np(to_np(x["g"])[:, None], to_np(inp["A_log"]), to_np(inp["dt_bias"]), gate, per_head, Dk)[:, 0]
    S_ref, o_ref = oracle.kda_step(to_np(inp["S0"]), *(to_np(x[n]) for n in ("q", "k", "v")), g,
                                   to_np(x["beta"]), gate_in=False)
    scale_o = TOL / TOL_BF16 if dtype == "bf16" else 1.0
    return {"o": max_rel(to_np(o), o_ref) * scale_o, "S": max_rel(to_np(S), S_ref)}


def run_compose_case(lib, n_seg, BH, Dk, Dv, with_init, seed):
    gen = torch.Generator().manual_seed(seed)
    M = 0.3 * torch.randn((n_seg, BH, Dk, Dk), generator=gen)
    S_seg = torch.randn((n_seg, BH, Dk, Dv), generator=gen)
    S_init = torch.randn((BH, Dk, Dv), generator=gen) if with_init else None
    S_in = torch.full((n_seg + 1, BH, Dk, Dv), float("nan"))
    lib.emu_compose(n_seg, BH, Dk, Dv, _ptr(M), _ptr(S_seg), _ptr(S_init), _ptr(S_in))
    ref = oracle.kda_compose(to_np(M), to_np(S_seg), to_np(S_init))
    return {"S_in": max_rel(to_np(S_in), ref)}


def run_layer_case(lib, B, T, C, K, head_dim, silu, with_state, seed):
    from oracle import layer
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn((B, T, C), generator=gen).to(torch.bfloat16)
    w = 0.5 * torch.randn((C, K), generator=gen)
    bias = 0.1 * torch.randn(C, generator=gen)
    st_in = torch.randn((B, K - 1, C), generator=gen).to(torch.bfloat16) if with_state else None
    y = torch.zeros((B, T, C), dtype=torch.bfloat16)
    st_out = torch.zeros((B, K - 1, C), dtype=torch.bfloat16)
    cp = ConvParams(B, T, C, K, head_dim, int(silu), 1e-6, _ptr(x), _ptr(w), _ptr(bias), _ptr(st_in), _ptr(y),
                    _ptr(st_out) if K > 1 else None)
    lib.emu_short_conv(ctypes.byref(cp))
    y_ref, st_ref = layer.prologue(to_np(x), to_np(w), to_np(bias), to_np(st_in), head_dim=head_dim, act=silu)
    # bf16 outputs: one rounding, 2^-8 relative, held to 2^-7 of the largest value
    err = {"y": max_rel(to_np(y), y_ref) * TOL / 2 ** -7}
    if K > 1:
        err["state_out"] = max_rel(to_np(st_out), st_ref)   # copied bf16 inputs: exact
    HV, D = 4, 128
    o = torch.randn((B * T, HV, D), generator=gen).to(torch.bfloat16)
    gate = torch.randn((B * T, HV, D), generator=gen).to(torch.bfloat16)
    wt = 1.0 + 0.1 * torch.randn(D, generator=gen)
    yo = torch.zeros_like(o)
    gp = GateParams(B * T, HV, D, 1e-6, _ptr(o), _ptr(gate), _ptr(wt), _ptr(yo))
    lib.emu_output_gate(ctypes.byref(gp))
    err["gate"] = max_rel(to_np(yo), layer.output_gate(to_np(o), to_np(gate), to_np(wt))) * TOL / 2 ** -7
    return err


def run_transition_case(lib, B, T, H, HV, Dk, Dv, C, seed):
    """Forward with the cumulative transition M_T and the chunk states at once
    (the transition columns ride in extra column slices)."""
    w = workloads.Workload("emu_m", B=B, T=T, H=H, HV=HV, Dk=Dk, Dv=Dv, chunk=C, dtype="f32", seed=seed,
                           a_log="uniform", s0_std=0.1)
    inp = workloads.chunk_inputs(w, z_mean=-3.0)          # slow decay: M_T far from 0
    o = torch.zeros((B, T, HV, Dv)); S_T = torch.zeros((B, HV, Dk, Dv)); M_T = torch.zeros((B, HV, Dk, Dk))
    S_ch = torch.zeros((B, HV, -(-T // C), Dk, Dv))
    fp = ChunkParams(B, T, H, HV, Dk, Dv, C, HV // H, -5.0, 1.0, 1e-6, 1, 1, 1, 0,
                     *(_ptr(inp[n]) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0")),
                     _ptr(o), _ptr(S_T), _ptr(M_T), _ptr(S_ch), 0)
    lib.emu_chunk_fwd(ctypes.byref(fp), 0)
    ref = oracle.kda_fwd(*(to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")), A_log=to_np(inp["A_log"]),
                         S0=to_np(inp["S0"]), want_M=True)
    return {"o": max_rel(to_np(o), ref["o"]), "S_T": max_rel(to_np(S_T), ref["S_T"]),
            "M_T": max_rel(to_np(M_T), ref["M_T"]), "S_chunks0": max_rel(to_np(S_ch[:, :, 0]), to_np(inp["S0"]))}


TRANSITION_CASES = [
    # B, T, H, HV, Dk, Dv, C, seed
    (1, 50, 1, 2, 16, 24, 16, 51),
    (2, 70, 1, 1, 40, 8, 32, 52),
]

def run_tc_case(lib, B, T, H, HV, want_M, s0, z_mean, seed, per_head=False, states=False, gate=1):
    """The tensor-core chunk kernel (bf16, Dk = Dv = 128, C = 64) over the host
    model of its instructions, against the oracle at the bf16 bars (o: 2e-2 of
    max|o|; S_T, M_T, chunk states: 2e-2 Frobenius), each rescaled to TOL."""
    from helpers import fro_rel
    w = workloads.Workload("emu_tc", B=B, T=T, H=H, HV=HV, Dk=128, Dv=128, chunk=64, dtype="bf16", seed=seed,
                           a_log="uniform", dt_bias_std=0.5, s0_std=s0)
    inp = workloads.chunk_inputs(w, z_mean=z_mean)
    if per_head:
        inp = _per_head(inp)
    if gate == 2:      # the softplus gate, kept above g_min (exp(A_log) = 0.22)
        inp["A_log"] = torch.full_like(inp["A_log"], -1.5)
    o = torch.zeros((B, T, HV, 128), dtype=torch.bfloat16)
    S_T = torch.zeros((B, HV, 128, 128))
    M_T = torch.zeros((B, HV, 128, 128)) if want_M else None
    NC = -(-T // 64)
    S_ch = torch.full((B, HV, NC, 128, 128), float("nan")) if states else None
    fp = ChunkParams(B, T, H, HV, 128, 128, 64, HV // H, -5.0, 1.0, 1e-6, 1, 1, gate, int(per_head),
                     *(_ptr(inp[n]) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0")),
                     _ptr(o), _ptr(S_T), _ptr(M_T), _ptr(S_ch), 0)
    if lib.emu_chunk_tc(ctypes.byref(fp)) != 0:
        return {"device_error": 1.0}
    args = [to_np(inp[n]) for n in ("q", "k", "v", "g", "beta")]
    if per_head or gate == 2:
        args[3] = _gate_np(args[3], to_np(inp["A_log"]), to_np(inp["dt_bias"]),
                           "bounded" if gate == 1 else "softplus", per_head, 128)
        kw = dict(S0=to_np(inp["S0"]), gate_in=False)
    else:
        kw = dict(A_log=to_np(inp["A_log"]), dt_bias=to_np(inp["dt_bias"]), S0=to_np(inp["S0"]))
    ref = oracle.kda_fwd(*args, want_M=want_M, **kw)
    k = TOL / TOL_BF16
    err = {"o": max_rel(to_np(o), ref["o"]) * k, "S_T": fro_rel(to_np(S_T), ref["S_T"]) * k}
    if want_M:
        err["M_T"] = fro_rel(to_np(M_T), ref["M_T"]) * k
    if states:
        worst = fro_rel(to_np(S_ch[:, :, 0]), to_np(inp["S0"]) if inp["S0"] is not None else np.zeros((B, HV, 128, 128)))
        for c in range(1, NC):
            pre = oracle.kda_fwd(*(a[:, : c * 64] for a in args), **kw)["S_T"]
            worst = max(worst, fro_rel(to_np(S_ch[:, :, c]), pre))
        err["S_chunks"] = worst * k
    return err


TC_CASES = [
    # B, T, H, HV, want_M, s0, z_mean, seed
    (1, 64, 1, 1, False, None, 0.0, 95),       # one chunk
    (1, 192, 1, 2, False, 0.02, 0.0, 223),     # three chunks, carried state
    (1, 256, 1, 2, True, 0.05, -8.0, 287),     # slow decay, with the transition CTAs
    (1, 200, 1, 2, False, 0.05, 0.0, 5, False, True),   # chunk states written
    (1, 130, 2, 4, False, 0.05, 0.0, 6, True, False),   # one decay per (token, head)
    (2, 200, 2, 4, True, 0.02, 0.0, 231),      # two batch rows, grouped heads, ragged, transition
    (1, 1, 1, 1, False, 0.05, 0.0, 32),        # a single token
    (1, 150, 1, 2, False, 0.05, 0.0, 33, False, False, 2),   # the softplus gate above g_min
]

COMPOSE_CASES = [
    # n_seg, BH, Dk, Dv, with_init, seed
    (4, 3, 16, 40, True, 21),
    (3, 2, 128, 128, False, 22),
    (0, 2, 8, 8, True, 23),
]
LAYER_CASES = [
    # B, T, C, K, head_dim, silu, with_state, seed
    (2, 100, 256, 4, 128, True, False, 31),
    (1, 7, 128, 3, 0, False, True, 32),
    (1, 0, 128, 4, 0, True, True, 33),
    (2, 150, 512, 3, 128, True, True, 34),
    (3, 1, 256, 4, 0, True, True, 35),
]

STEP_CASES = [
    # B, H, HV, Dk, Dv, dtype, gate, per_head, seed
    (2, 1, 2, 128, 128, "f32", "bounded", False, 11),
    (2, 1, 2, 64, 32, "f32", "softplus", False, 12),
    (3, 2, 4, 128, 64, "bf16", "softplus", True, 13),
    (1, 1, 1, 32, 16, "f32", "bounded", True, 14),
    (3, 1, 3, 128, 128, "bf16", "bounded", False, 15),   # 9 chains: stage reuse in the bulk-copy kernel
]

CASES = [
    # B, T, H, HV, Dk, Dv, C, dtype, flags, scale, seed
    (1, 37, 1, 2, 16, 12, 16, "f32", True, 1.0, 1),      # ragged last chunk, grouped heads
    (2, 50, 1, 2, 32, 40, 16, "f32", True, 0.5, 2),      # two column slices, one ragged
    (1, 70, 2, 2, 16, 16, 32, "f32", False, 1.0, 3),     # switches off
    (1, 45, 1, 1, 24, 20, 16, "bf16", True, 1.0, 4),     # bf16 inputs
    (1, 70, 1, 1, 128, 128, 64, "f32", True, 1.0, 5),    # full head size, C = 64, ragged
    (2, 0, 1, 2, 16, 16, 16, "f32", True, 1.0, 6),       # empty sequence
    (1, 40, 1, 2, 16, 16, 16, "f32", True, 1.0, 7, "softplus", False),   # unbounded gate
    (1, 40, 1, 2, 16, 16, 16, "f32", True, 1.0, 8, "bounded", True),     # one decay per head
    (2, 50, 1, 2, 32, 40, 16, "bf16", True, 1.0, 9, "softplus", True),   # both, bf16
    (1, 5, 1, 1, 1, 1, 1, "f32", False, 1.0, 10),      # Dk = Dv = chunk = 1
    (2, 23, 1, 3, 3, 5, 7, "f32", True, 1.0, 11),      # odd sizes everywhere
    (1, 1, 1, 1, 8, 8, 16, "f32", True, 1.0, 12),      # one token, shorter than a chunk
    (1, 150, 1, 2, 128, 128, 64, "bf16", True, 1.0, 13),  # anchored backward: three chunks, grouped heads
]
TOL = TOL_F32

def race_run(lib_path):
    """ThreadSanitizer build: run the kernels (no oracle, one torch thread) so
    that any report comes from the kernels' own synchronisation."""
    torch.set_num_threads(1)
    lib = ctypes.CDLL(lib_path)
    for case in (CASES[1], CASES[4], CASES[8], CASES[9]):
        run_case(lib, *case, check=False)
    for case in STEP_CASES[:2]:
        run_step_case(lib, *case, check=False)
    for case in TC_CASES[:2]:
        B, T, H, HV, want_M, s0, z_mean, seed = case
        w = workloads.Workload("race_tc", B=B, T=T, H=H, HV=HV, Dk=128, Dv=128, chunk=64, dtype="bf16", seed=seed,
                               a_log="uniform", dt_bias_std=0.5, s0_std=s0)
        inp = workloads.chunk_inputs(w, z_mean=z_mean)
        o = torch.zeros((B, T, HV, 128), dtype=torch.bfloat16)
        S_T = torch.zeros((B, HV, 128, 128))
        fp = ChunkParams(B, T, H, HV, 128, 128, 64, HV // H, -5.0, 1.0, 1e-6, 1, 1, 1, 0,
                         *(_ptr(inp[n]) for n in ("q", "k", "v", "g", "beta", "A_log", "dt_bias", "S0")),
                         _ptr(o), _ptr(S_T), None, None, 0)
        lib.emu_chunk_tc(ctypes.byref(fp))
    lib.emu_compose.argtypes = [_I] * 4 + [_P] * 4
    gen = torch.Generator().manual_seed(5)
    M, S_seg = torch.randn((3, 2, 16, 16), generator=gen), torch.randn((3, 2, 16, 40), generator=gen)
    S_in = torch.empty((4, 2, 16, 40))
    lib.emu_compose(3, 2, 16, 40, _ptr(M), _ptr(S_seg), None, _ptr(S_in))
    x = torch.randn((1, 70, 256), generator=gen).to(torch.bfloat16)
    w = torch.randn((256, 4), generator=gen)
    y, st = torch.empty_like(x), torch.empty((1, 3, 256), dtype=torch.bfloat16)
    lib.emu_short_conv(ctypes.byref(ConvParams(1, 70, 256, 4, 128, 1, 1e-6, _ptr(x), _ptr(w), None, None,
                                               _ptr(y), _ptr(st))))
    o = torch.randn((70, 4, 128), generator=gen).to(torch.bfloat16)
    yo = torch.empty_like(o)
    lib.emu_output_gate(ctypes.byref(GateParams(70, 4, 128, 1e-6, _ptr(o), _ptr(o), None, _ptr(yo))))
    print("race run done", flush=True)
    return 0


if __name__ == "__main__":
    if len(sys.argv) > 2 and sys.argv[1] == "--races":
        sys.exit(race_run(sys.argv[2]))
    lib = ctypes.CDLL(os.path.join(HERE, "_build", "libkda_host_emu.so"))
    assert lib.emu_sizeof_chunk_params() == ctypes.sizeof(ChunkParams)
    assert lib.emu_offsetof_withhold_ready() == ChunkParams.withhold_ready.offset
    assert lib.emu_sizeof_bwd_params() == ctypes.sizeof(BwdParams)
    assert lib.emu_offsetof_ddt_bias() == BwdParams.ddt_bias.offset
    assert lib.emu_sizeof_step_params() == ctypes.sizeof(StepParams)
    lib.emu_compose.argtypes = [_I] * 4 + [_P] * 4
    assert lib.emu_sizeof_conv_params() == ctypes.sizeof(ConvParams)
    assert lib.emu_sizeof_gate_params() == ctypes.sizeof(GateParams)
    bad = 0
    for name, fn, cases in (("tc", run_tc_case, TC_CASES), ("transition", run_transition_case, TRANSITION_CASES),
                            ("compose", run_compose_case, COMPOSE_CASES), ("layer", run_layer_case, LAYER_CASES)):
        for case in cases:
            err = fn(lib, *case)
            worst = max(err.values())
            bad += worst > TOL
            print(name, case, "ok" if worst <= TOL else "MISMATCH",
                  " ".join("%s=%.1e" % kv for kv in err.items()), flush=True)
    for case in STEP_CASES:
        err = run_step_case(lib, *case)
        worst = max(err.values())
        bad += worst > TOL
        print("step", case, "ok" if worst <= TOL else "MISMATCH", " ".join("%s=%.1e" % kv for kv in err.items()),
              flush=True)
    for case in CASES:
        err = run_case(lib, *case)
        worst = max(err.values()) if err else 0.0
        bad += worst > TOL
        print(case, "ok" if worst <= TOL else "MISMATCH", " ".join("%s=%.1e" % kv for kv in err.items()),
              flush=True)
    sys.exit(1 if bad else 0)
