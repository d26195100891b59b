"""FP64 CPU oracle for the KDA core -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The product path (gated_delta_rule_157_b200) never imports it and
shares no code with it.

Contents:
  * ``kda_fwd`` / ``kda_step`` / ``kda_compose`` -- ctypes front end of the C
    oracle in ``kda_oracle.c``: the plain token-by-token recurrence in double
    precision (page "Implémenter KDA", "La forme récurrente de référence").
  * ``brute`` -- dense affine-product form for tiny shapes (independent NumPy
    restatement used to pin the C oracle).
  * ``chunkwise`` -- FP64 NumPy restatement of the chunk-parallel form (page
    "KDA 模块交互式演示" section 1.5, Eqs. 3-4) used only to pin the reading of
    the chunk algebra against the recurrence.
  * ``layer`` -- FP64 NumPy restatements of the layer prologue (short
    convolution, SiLU, per-head L2 norm) and epilogue (per-head RMSNorm and the
    sigmoid output gate).
  * ``backward`` -- FP64 NumPy reverse-mode gradient of the forward (token by
    token, in reverse), pinned by finite differences of the C oracle.
  * ``gates`` -- the decay gates of the family (bounded KDA v2 gate, unbounded
    softplus v1 gate, per-head Gated DeltaNet gate) as maps z -> log-decay.

Inputs are NumPy arrays (any float dtype; they are widened to float64 exactly).
"""
import ctypes

import numpy as np

from .build import build_oracle

_lib = None


class _Args(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
        ("HV", ctypes.c_int), ("Dk", ctypes.c_int), ("Dv", ctypes.c_int),
        ("g_min", ctypes.c_double), ("scale", ctypes.c_double), ("l2_eps", ctypes.c_double),
        ("qk_l2norm_in_kernel", ctypes.c_int), ("beta_sigmoid_in_kernel", ctypes.c_int),
        ("gate_in_kernel", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("A_log", ctypes.c_void_p),
        ("dt_bias", ctypes.c_void_p), ("S0", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("S_T", ctypes.c_void_p), ("M_T", ctypes.c_void_p),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        lib.oracle_kda_fwd.argtypes = [ctypes.POINTER(_Args)]
        lib.oracle_kda_fwd.restype = ctypes.c_int
        lib.oracle_kda_step.argtypes = [ctypes.POINTER(_Args), ctypes.c_void_p]
        lib.oracle_kda_step.restype = ctypes.c_int
        lib.oracle_kda_compose.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 4
        lib.oracle_kda_compose.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p).value


def _fill_args(q, k, v, g, beta, A_log, dt_bias, g_min, scale, l2_eps,
               qk_l2norm, beta_sigmoid, gate_in, T):
    B, H, Dk = q.shape[0], q.shape[-2], q.shape[-1]
    HV, Dv = v.shape[-2], v.shape[-1]
    if gate_in and A_log is None:
        raise ValueError("gate_in requires A_log")
    a = _Args()
    a.B, a.T, a.H, a.HV, a.Dk, a.Dv = B, T, H, HV, Dk, Dv
    a.g_min, a.scale, a.l2_eps = float(g_min), float(scale), float(l2_eps)
    a.qk_l2norm_in_kernel = int(bool(qk_l2norm))
    a.beta_sigmoid_in_kernel = int(bool(beta_sigmoid))
    a.gate_in_kernel = int(bool(gate_in))
    a.q, a.k, a.v, a.g, a.beta = map(_ptr, (q, k, v, g, beta))
    a.A_log, a.dt_bias = _ptr(A_log), _ptr(dt_bias)
    return a


def kda_fwd(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, g_min=-5.0,
            scale=1.0, l2_eps=1e-6, qk_l2norm=True, beta_sigmoid=True, gate_in=True,
            want_state=True, want_M=False):
    """Full-sequence forward.

    Shapes: q,k [B,T,H,Dk]; v [B,T,HV,Dv]; g (or raw z) [B,T,HV,Dk]; beta (or
    logits) [B,T,HV]; A_log [HV]; dt_bias [HV,Dk]; S0 [B,HV,Dk,Dv].
    Returns dict with o [B,T,HV,Dv], S_T [B,HV,Dk,Dv], M_T [B,HV,Dk,Dk] (float64).
    """
    q, k, v, g, beta, A_log, dt_bias, S0 = map(_f64, (q, k, v, g, beta, A_log, dt_bias, S0))
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    o = np.zeros((B, T, HV, Dv))
    S_T = np.zeros((B, HV, Dk, Dv)) if want_state else None
    M_T = np.zeros((B, HV, Dk, Dk)) if want_M else None
    a = _fill_args(q, k, v, g, beta, A_log, dt_bias, g_min, scale, l2_eps,
                   qk_l2norm, beta_sigmoid, gate_in, T)
    a.S0, a.o, a.S_T, a.M_T = _ptr(S0), _ptr(o), _ptr(S_T), _ptr(M_T)
    rc = _load().oracle_kda_fwd(ctypes.byref(a))
    if rc != 0:
        raise RuntimeError("oracle_kda_fwd failed with code %d" % rc)
    return {"o": o, "S_T": S_T, "M_T": M_T}


def kda_step(S, q, k, v, g, beta, *, A_log=None, dt_bias=None, g_min=-5.0, scale=1.0,
             l2_eps=1e-6, qk_l2norm=True, beta_sigmoid=True, gate_in=True):
    """One decode step for B*HV chains.

    Shapes: S [B,HV,Dk,Dv]; q,k [B,H,Dk]; v [B,HV,Dv]; g [B,HV,Dk]; beta [B,HV].
    Returns (S_next, o [B,HV,Dv]); the input S is not modified.
    """
    S = np.array(S, dtype=np.float64, order="C", copy=True)
    q, k, v, g, beta, A_log, dt_bias = map(_f64, (q, k, v, g, beta, A_log, dt_bias))
    # Insert the T=1 axis so the [B,T,...] layouts apply.
    q, k, v, g = (x[:, None] for x in (q, k, v, g))
    beta = beta[:, None]
    q, k, v, g, beta = map(np.ascontiguousarray, (q, k, v, g, beta))
    B, HV, Dv = v.shape[0], v.shape[2], v.shape[3]
    o = np.zeros((B, 1, HV, Dv))
    a = _fill_args(q, k, v, g, beta, A_log, dt_bias, g_min, scale, l2_eps,
                   qk_l2norm, beta_sigmoid, gate_in, 1)
    a.o = _ptr(o)
    rc = _load().oracle_kda_step(ctypes.byref(a), _ptr(S))
    if rc != 0:
        raise RuntimeError("oracle_kda_step failed with code %d" % rc)
    return S, o[:, 0]


def kda_compose(M, S_seg, S_init=None):
    """Sequential segment combine.  M [n,BH,Dk,Dk], S_seg [n,BH,Dk,Dv],
    S_init [BH,Dk,Dv] or None.  Returns S_in [n+1,BH,Dk,Dv]."""
    M, S_seg, S_init = map(_f64, (M, S_seg, S_init))
    n, BH, Dk, Dv = S_seg.shape
    S_in = np.zeros((n + 1, BH, Dk, Dv))
    rc = _load().oracle_kda_compose(n, BH, Dk, Dv, _ptr(M), _ptr(S_seg), _ptr(S_init), _ptr(S_in))
    if rc != 0:
        raise RuntimeError("oracle_kda_compose failed with code %d" % rc)
    return S_in
