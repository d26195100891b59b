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
sigmoid(logit), g = g_min sigmoid(a (z + dt_bias)) with a = exp(A_log).  It is
pinned by central finite differences of the forward (tests), not by itself.
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


def kda_backward(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, do=None, dS_T=None,
                 g_min=-5.0, scale=1.0, l2_eps=1e-6, qk_l2norm=True, beta_sigmoid=True, gate_in=True):
    """Gradients of <do, o> + <dS_T, S_T> for the layouts of the forward
    (q, k [B,T,H,Dk]; v [B,T,HV,Dv]; g or raw z [B,T,HV,Dk]; beta or logits
    [B,T,HV]; A_log [HV]; dt_bias [HV,Dk]; S0 [B,HV,Dk,Dv]).  Returns a dict
    with dq, dk, dv, dg (w.r.t. the g / z input), dbeta (w.r.t. the beta /
    logit input), dS0, and dA_log, ddt_bias when the gate runs in-kernel."""
    q, k, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta))
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    grp = HV // H
    do = np.zeros((B, T, HV, Dv)) if do is None else np.asarray(do, dtype=np.float64)
    dS_T = np.zeros((B, HV, Dk, Dv)) if dS_T is None else np.asarray(dS_T, dtype=np.float64)
    S0 = np.zeros((B, HV, Dk, Dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    A_log = np.zeros(HV) if A_log is None else np.asarray(A_log, dtype=np.float64)
    dt_bias = np.zeros((HV, Dk)) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)

    qh, nq = _l2(q, l2_eps) if qk_l2norm else (q, None)
    kh, nk = _l2(k, l2_eps) if qk_l2norm else (k, None)
    bt = _sig(beta) if beta_sigmoid else beta
    if gate_in:
        a = np.exp(A_log)[None, None, :, None]
        pre = a * (g + dt_bias[None, None])
        sg = _sig(pre)
        gg = g_min * sg
    else:
        gg = g
    out = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta))}
    out["S0"] = np.zeros_like(S0)
    dqh, dkh = np.zeros_like(qh), np.zeros_like(kh)
    dgg = np.zeros_like(gg)
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
    if gate_in:
        dpre = dgg * g_min * sg * (1 - sg)
        out["g"] = dpre * a
        out["dt_bias"] = (dpre * a).sum(axis=(0, 1))
        out["A_log"] = (dpre * pre).sum(axis=(0, 1, 3))   # d pre / d A_log = pre (a = exp(A_log))
    else:
        out["g"] = dgg
    return out
