"""FP64 restatements of the decay gates of the KDA family -- TEST INFRASTRUCTURE.

Each maps a raw gate input z to the log-decay g (alpha = exp(g)) that the
recurrence of the C oracle consumes with its in-kernel gate switched off.

  bounded_gate   KDA v2 / Kimi K3: g = g_min sigmoid(exp(A_log) (z + dt_bias)),
                 g in (g_min, 0) (page "Implémenter KDA", "La décroissance
                 bornée"; page "KDA 模块交互式演示" section 1.4 Eq. 5).
  softplus_gate  KDA v1 / Kimi Linear: g = -exp(A_log) softplus(z + dt_bias),
                 g in (-inf, 0), unbounded below.
  gdn_gate       Gated DeltaNet: one decay per (token, head), alpha = sigmoid(z),
                 i.e. g = log sigmoid(z) = -softplus(-z), shared by every key
                 channel (page "线性注意力交互式演示", section 1.2, Eq. 6).

The pages write the v1 gate three ways: -softplus(z) (page
"线性注意力交互式演示", "门控衰减" and Tab 3), -softplus(g_logit + exp(A_log))
(the same page, Eq. 7) and -exp(A) softplus(z) (page "Implémenter KDA", "La
décroissance bornée").  The reading taken is the last, with dt_bias added inside as
for the bounded gate; at A_log = 0, dt_bias = 0 it is -softplus(z), the curve
that Tab 3 plots (its printed extremes are the pins).  Eq. 7's placement of
exp(A_log) inside the softplus is not followed.
"""
import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def softplus(x):
    """log(1 + e^x), evaluated without overflow for large |x|."""
    x = _f64(x)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def _head_params(z, A_log, dt_bias):
    """Broadcast A_log [HV] and dt_bias [HV, Dk] against z [..., HV, Dk]."""
    z = _f64(z)
    HV, Dk = z.shape[-2], z.shape[-1]
    a = np.exp(_f64(np.zeros(HV) if A_log is None else A_log))[:, None]
    b = _f64(np.zeros((HV, Dk)) if dt_bias is None else dt_bias)
    return z, a, b


def bounded_gate(z, A_log=None, dt_bias=None, g_min=-5.0):
    """KDA v2: z [..., HV, Dk] -> g = g_min * sigmoid(exp(A_log) * (z + dt_bias))."""
    z, a, b = _head_params(z, A_log, dt_bias)
    return g_min * sigmoid(a * (z + b))


def softplus_gate(z, A_log=None, dt_bias=None):
    """KDA v1: z [..., HV, Dk] -> g = -exp(A_log) * softplus(z + dt_bias)."""
    z, a, b = _head_params(z, A_log, dt_bias)
    return -a * softplus(z + b)


def gdn_gate(z):
    """Gated DeltaNet: z [..., HV] -> per-head log-decay log sigmoid(z)."""
    return -softplus(-_f64(z))


def broadcast_channels(g_head, Dk):
    """Per-head log-decay [..., HV] -> the per-channel layout [..., HV, Dk]."""
    g_head = _f64(g_head)
    return np.repeat(g_head[..., None], Dk, axis=-1)
