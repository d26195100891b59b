"""Shared test helpers: run the oracle on the exact inputs the GPU received and
measure the discrepancy the way the tolerances are stated.

Tolerances (stated for the KDA core): the FP32 path must match the FP64 oracle
to a max relative error <= 1e-4, read as max|gpu - ref| / max|ref| per output
tensor; the BF16-input / FP32-accumulate path to <= 2e-2 of max|o| for o and
<= 2e-2 of ||S_T||_F for the Frobenius error of S_T.
"""
import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
TOL_BF16 = 2e-2
# fp32 outputs carry no relative accuracy for magnitudes far below FLT_MIN
# (1.2e-38): a reference whose largest entry is below this floor (e.g. a
# cumulative transition decayed to 1e-60) is compared in absolute terms.
REL_FLOOR = 1e-30


def to_np(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.astype(np.float64, copy=False)
    return t.detach().to("cpu", torch.float64).numpy()


def max_rel(x, ref):
    """max|x - ref| / max(max|ref|, REL_FLOOR)."""
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    den = max(float(np.max(np.abs(ref))), REL_FLOOR)
    return float(np.max(np.abs(x - ref)) / den)


def sum_rel(x, ref, l1):
    """Error of a gradient that is a sum over tokens (dA_log, ddt_bias): the
    largest |x - ref| over the largest of max|ref| and the summed magnitudes
    l1 of the terms -- a sum of terms that cancel is accurate to its l1, not
    to its own value."""
    x, ref, l1 = (np.asarray(a, np.float64) for a in (x, ref, l1))
    if ref.size == 0:
        return 0.0
    den = max(float(np.max(np.abs(ref))), float(np.max(l1)), REL_FLOOR)
    return float(np.max(np.abs(x - ref)) / den)


def fro_rel(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = max(float(np.linalg.norm(ref)), REL_FLOOR)
    return float(np.linalg.norm(x - ref) / den)


def oracle_chunk(inp, *, flags=True, g_min=-5.0, scale=1.0, want_M=False, chains=None):
    """Oracle forward on the inputs dict (CPU or CUDA tensors).  ``chains`` is an
    optional list of (b, hv) pairs: the oracle then runs only those chains (one
    batch row and one value head at a time) and returns {(b, hv): result}."""
    q, k, v, g, beta = (to_np(inp[n]) for n in ("q", "k", "v", "g", "beta"))
    A_log, dt_bias, S0 = to_np(inp["A_log"]), to_np(inp["dt_bias"]), to_np(inp["S0"])
    kw = dict(g_min=g_min, scale=scale, qk_l2norm=flags, beta_sigmoid=flags, gate_in=flags,
              want_M=want_M)
    if chains is None:
        return oracle.kda_fwd(q, k, v, g, beta, A_log=A_log, dt_bias=dt_bias, S0=S0, **kw)
    H, HV = q.shape[2], v.shape[2]
    out = {}
    for b, hv in chains:
        h = hv // (HV // H)
        r = oracle.kda_fwd(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1],
                           v[b:b + 1, :, hv:hv + 1], g[b:b + 1, :, hv:hv + 1],
                           beta[b:b + 1, :, hv:hv + 1],
                           A_log=None if A_log is None else A_log[hv:hv + 1],
                           dt_bias=None if dt_bias is None else dt_bias[hv:hv + 1],
                           S0=None if S0 is None else S0[b:b + 1, hv:hv + 1], **kw)
        out[(b, hv)] = r
    return out


def to_device(inp, device):
    return {k: (None if v is None else v.to(device)) for k, v in inp.items()}
