"""FP64 oracle of the layer prologue and epilogue -- TEST INFRASTRUCTURE.

Plain NumPy restatements of the definitions on the pages, no blocking or
fusion:

  * ``short_conv`` -- page "KDA 模块交互式演示" section 1.1: causal depthwise
    convolution over K taps, left zero padding (or the K-1 carried tokens),
    identity at initialisation; page "Implémenter KDA", "La paramétrisation":
    q = l2norm(swish(short_conv(.))), v = swish(short_conv(.)).
  * ``output_gate`` -- page "Implémenter KDA", "La porte de sortie de rang
    plein" (Eq. 5): per-head RMSNorm, then the sigmoid gate (the output
    projection needs trained weights and is left out).

Readings (the pages leave them open): tap K-1 multiplies the current token
(the only indexing under which the stated identity initialisation is a no-op);
swish is SiLU, u * sigmoid(u); the L2 norm is x / sqrt(sum x^2 + eps) over one
head's channels; the RMSNorm scale is one weight per channel shared by the
heads, with eps inside the square root.
"""
import numpy as np


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def short_conv(x, w, bias=None, state_in=None):
    """x [B,T,C]; w [C,K] (tap K-1 on the current token); bias [C];
    state_in [B,K-1,C] (the K-1 tokens before x, oldest first) or None.
    Returns (u [B,T,C], state_out [B,K-1,C])."""
    x, w, bias, state_in = map(_f64, (x, w, bias, state_in))
    B, T, C = x.shape
    K = w.shape[1]
    prev = np.zeros((B, K - 1, C)) if state_in is None else state_in
    full = np.concatenate([prev, x], axis=1)           # token t of x is row t + K - 1
    u = np.zeros((B, T, C))
    for t in range(T):
        for j in range(K):
            u[:, t, :] += w[:, j] * full[:, t + j, :]  # row t + j = token t - (K-1) + j
    if bias is not None:
        u += bias
    return u, full[:, full.shape[1] - (K - 1):, :].copy()


def silu(u):
    u = _f64(u)
    return u / (1.0 + np.exp(-u))


def l2norm_heads(y, head_dim, eps=1e-6):
    """Normalise every group of head_dim channels of the last axis."""
    y = _f64(y)
    shp = y.shape
    g = y.reshape(shp[:-1] + (shp[-1] // head_dim, head_dim))
    g = g / np.sqrt((g * g).sum(axis=-1, keepdims=True) + eps)
    return g.reshape(shp)


def prologue(x, w, bias=None, state_in=None, head_dim=0, act=True, eps=1e-6):
    """The whole prologue: (y, state_out)."""
    u, st = short_conv(x, w, bias, state_in)
    y = silu(u) if act else u
    if head_dim:
        y = l2norm_heads(y, head_dim, eps)
    return y, st


def output_gate(o, gate, weight=None, eps=1e-6):
    """o, gate [..., HV, D]; weight [D].  sigmoid(gate) * weight * o / rms(o)."""
    o, gate, weight = map(_f64, (o, gate, weight))
    rms = np.sqrt((o * o).mean(axis=-1, keepdims=True) + eps)
    y = o / rms
    if weight is not None:
        y = y * weight
    return y / (1.0 + np.exp(-gate))
