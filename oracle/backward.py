"""FP64 oracle of the gradient of the KDA forward -- TEST INFRASTRUCTURE.

The pages do not describe a backward pass (one names a "dt_bias backward" fix
only); this is the plain reverse-mode derivative of the forward the library
computes (page "Implémenter KDA", "La forme récurrente de référence", with the
three in-kernel switches of page "KDAAttention 层"), written token by token in
reverse order, for one chain at a time:

  forward, per token t (S = state before the token, alpha = exp(g)):
      P = Diag(alpha) S;  e = v - P^T k;  S' = P + beta k e^T;  o = scale S'^T q
  reverse, given dS' (gradient of the loss w.r.t. S') and do:
      dS'  += scale q do^T                         (o reads the updated state)
      dq    = scale S' do
      dv    = beta dS'^T k
      dbeta = k^T dS' e
      dk    = beta dS' e - beta P (dS'^T k)
      dP    = dS' - beta k (k^T dS')               ((I - beta k k^T) dS')
      dg    = alpha * rowsum(dP * S)               (P = Diag(alpha) S)
      dS    = Diag(alpha) dP

and through the switches: q^ = q / sqrt(|q|^2 + eps) (same for k), beta =
sigmoid(logit), and the gate, g = g_min sigmoid(a (z + dt_bias)) (bounded) or
g = -a softplus(z + dt_bias) (softplus) with a = exp(A_log), per key channel or
one per (token, head).  It is pinned by central finite differences of the
forward (tests), not by itself.
"""
import numpy as np


def _l2(x, eps):
    n = np.sqrt((x * x).sum(-1, keepdims=True) + eps)
    return x / n, n


def _l2_back(x, n, dy):
    # y = x / n, n = sqrt(|x|^2 + eps):  dx = dy / n - x (x . dy) / n^3
    return dy / n - x * (x * dy).sum(-1, keepdims=True) / n ** 3


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def chain_forward(q, k, v, g, beta, S0, scale=1.0):
    """One chain, activated inputs: q, k [T,Dk]; v [T,Dv]; g [T,Dk] (log-decay);
    beta [T]; S0 [Dk,Dv].  Returns (o [T,Dv], S_T, states [T+1,Dk,Dv])."""
    T, Dk = q.shape
    S = np.array(S0, dtype=np.float64)
    states = [S.copy()]
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        P = np.exp(g[t])[:, None] * S
        e = v[t] - P.T @ k[t]
        S = P + beta[t] * np.outer(k[t], e)
        o[t] = scale * (S.T @ q[t])
        states.append(S.copy())
    return o, S, np.stack(states)


def chain_backward(q, k, v, g, beta, S0, do, dS_T, scale=1.0):
    """Gradients of <do, o> + <dS_T, S_T> w.r.t. (q, k, v, g, beta, S0) for one
    chain with activated inputs (shapes as chain_forward)."""
    T = q.shape[0]
    _, _, states = chain_forward(q, k, v, g, beta, S0, scale)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, dbeta = np.zeros_like(g), np.zeros_like(beta)
    dS = np.array(dS_T, dtype=np.float64)
    for t in range(T - 1, -1, -1):
        S_prev, S_new = states[t], states[t + 1]
        a = np.exp(g[t])
        P = a[:, None] * S_prev
        e = v[t] - P.T @ k[t]
        dS = dS + scale * np.outer(q[t], do[t])
        dq[t] = scale * (S_new @ do[t])
        dv[t] = beta[t] * (dS.T @ k[t])
        dbeta[t] = k[t] @ dS @ e
        dk[t] = beta[t] * (dS @ e) - beta[t] * (P @ (dS.T @ k[t]))
        dP = dS - beta[t] * np.outer(k[t], k[t] @ dS)
        dg[t] = a * (dP * S_prev).sum(1)
        dS = a[:, None] * dP
    return {"q": dq, "k": dk, "v": dv, "g": dg, "beta": dbeta, "S0": dS}


def _softplus(x):
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def kda_backward(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, do=None, dS_T=None,
                 g_min=-5.0, scale=1.0, l2_eps=1e-6, qk_l2norm=True, beta_sigmoid=True, gate_in=True,
                 gate="bounded", per_head=False):
    """Gradients of <do, o> + <dS_T, S_T> for the layouts of the forward
    (q, k [B,T,H,Dk]; v [B,T,HV,Dv]; g or raw z [B,T,HV,Dk]; beta or logits
    [B,T,HV]; A_log [HV]; dt_bias [HV,Dk]; S0 [B,HV,Dk,Dv]).  Returns a dict
    with dq, dk, dv, dg (w.r.t. the g / z input), dbeta (w.r.t. the beta /
    logit input), dS0, and dA_log, ddt_bias when the gate runs in-kernel (with
    A_log_l1, dt_bias_l1: the sums of the absolute values of the terms they
    add up, the scale a floating-point sum is accurate to).

    gate: the in-kernel gate, "bounded" (g = g_min sigmoid(exp(A_log)(z + dt_bias)))
    or "softplus" (g = -exp(A_log) softplus(z + dt_bias)).  per_head: g / z is
    [B,T,HV] and dt_bias [HV], one decay per (token, value head) shared by the
    key channels (the gradient w.r.t. it sums over the channels)."""
    q, k, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta))
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    grp = HV // H
    do = np.zeros((B, T, HV, Dv)) if do is None else np.asarray(do, dtype=np.float64)
    dS_T = np.zeros((B, HV, Dk, Dv)) if dS_T is None else np.asarray(dS_T, dtype=np.float64)
    S0 = np.zeros((B, HV, Dk, Dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    A_log = np.zeros(HV) if A_log is None else np.asarray(A_log, dtype=np.float64)
    bshape = (HV,) if per_head else (HV, Dk)
    dt_bias = np.zeros(bshape) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    zc = g[..., None] if per_head else g                     # [B,T,HV,1 or Dk]
    bc = dt_bias[:, None] if per_head else dt_bias           # [HV,1 or Dk]

    qh, nq = _l2(q, l2_eps) if qk_l2norm else (q, None)
    kh, nk = _l2(k, l2_eps) if qk_l2norm else (k, None)
    bt = _sig(beta) if beta_sigmoid else beta
    a = np.exp(A_log)[None, None, :, None]
    if gate_in and gate == "bounded":
        pre = a * (zc + bc[None, None])
        sg = _sig(pre)
        gg = g_min * sg
    elif gate_in and gate == "softplus":
        pre = zc + bc[None, None]
        gg = -a * _softplus(pre)
    elif gate_in:
        raise ValueError("gate must be 'bounded' or 'softplus'")
    else:
        gg = zc
    gg = np.broadcast_to(gg, (B, T, HV, Dk))
    out = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta))}
    out["S0"] = np.zeros_like(S0)
    dqh, dkh = np.zeros_like(qh), np.zeros_like(kh)
    dgg = np.zeros((B, T, HV, Dk))
    dbt = np.zeros_like(bt)
    for b in range(B):
        for hv in range(HV):
            h = hv // grp
            r = chain_backward(qh[b, :, h], kh[b, :, h], v[b, :, hv], gg[b, :, hv], bt[b, :, hv],
                               S0[b, hv], do[b, :, hv], dS_T[b, hv], scale)
            dqh[b, :, h] += r["q"]
            dkh[b, :, h] += r["k"]
            out["v"][b, :, hv] = r["v"]
            dgg[b, :, hv] = r["g"]
            dbt[b, :, hv] = r["beta"]
            out["S0"][b, hv] = r["S0"]
    out["q"] = _l2_back(q, nq, dqh) if qk_l2norm else dqh
    out["k"] = _l2_back(k, nk, dkh) if qk_l2norm else dkh
    out["beta"] = dbt * bt * (1 - bt) if beta_sigmoid else dbt
    if per_head:
        dgg = dgg.sum(axis=3, keepdims=True)                 # the decay is shared by the channels
    if gate_in and gate == "bounded":
        dpre = dgg * g_min * sg * (1 - sg)
        dz = dpre * a
        a_terms = dpre * pre                                # d pre / d A_log = pre (a = exp(A_log))
    elif gate_in:
        dz = -dgg * a * _sig(pre)                           # d softplus = sigmoid
        a_terms = dgg * gg[..., :dgg.shape[3]]              # g is linear in exp(A_log)
    else:
        dz = dgg
    if gate_in:
        out["A_log"] = a_terms.sum(axis=(0, 1, 3))
        out["dt_bias"] = dz.sum(axis=(0, 1))[:, 0] if per_head else dz.sum(axis=(0, 1))
        # the sums' conditioning: the summed magnitudes (what a float sum is accurate to)
        out["A_log_l1"] = np.abs(a_terms).sum(axis=(0, 1, 3))
        out["dt_bias_l1"] = np.abs(dz).sum(axis=(0, 1))[:, 0] if per_head else np.abs(dz).sum(axis=(0, 1))
    out["g"] = dz[..., 0] if per_head else dz
    return out
