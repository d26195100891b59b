"""FP64 NumPy restatement of the chunk-parallel KDA form.

TEST INFRASTRUCTURE (see oracle/__init__.py).  It exists only to pin the
reading of the chunk algebra against the recurrence; the GPU path never uses it.

Page "KDA 模块交互式演示", section 1.5 (Eqs. 3-4), per chunk of C tokens with
Gamma_r = exp(sum_{i<=r} g_i) (per key channel, relative to the chunk start):

    O    = (Q*Gamma) S + A Vt,          A = Tril[(Q*Gamma)(K/Gamma)^T]  (diagonal kept)
    Vt   = (I + M)^-1 Diag(beta) V - W S     (UT transform; page "Implémenter KDA",
                                              "La forme par blocs": Vt = U - W S)
    S_C  = Diag(Gamma_C) S + sum_r (Gamma_C/Gamma_r) k_r Vt_r^T

The page prints M = tril(Diag(beta) K K^T, -1).  Deriving the chunk form from
the recurrence gives the decay-weighted M = tril(Diag(beta)(K*Gamma)(K/Gamma)^T, -1)
and W = (I+M)^-1 Diag(beta)(K*Gamma); the two agree only when alpha == 1.
``ut_with_decay`` selects the derived reading (True, default) or the literal
print (False); the tests show the literal print disagrees with the recurrence.

In float64, K/Gamma stays finite for chunks up to ~140 tokens (exp(5*140) <
1.8e308), so the factorisation is used literally, with no sub-tiling.
"""
import numpy as np


def chunk_run(q, k, v, g, beta, S0=None, chunk=16, scale=1.0, ut_with_decay=True):
    """One chain.  q,k [T,Dk]; v [T,Dv]; g [T,Dk]; beta [T]; S0 [Dk,Dv] or None.
    Returns (o [T,Dv], S_T [Dk,Dv], M_T [Dk,Dk])."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, Dk = k.shape
    Dv = v.shape[1]
    S = np.zeros((Dk, Dv)) if S0 is None else np.array(S0, dtype=np.float64)
    M = np.eye(Dk)
    o = np.zeros((T, Dv))
    for s in range(0, T, chunk):
        e = min(s + chunk, T)
        Qc, Kc, Vc, bc = q[s:e], k[s:e], v[s:e], beta[s:e]
        G = np.cumsum(g[s:e], axis=0)
        if G.size and G.min() < -700.0:
            raise ValueError("chunk too long for an unguarded fp64 factorisation")
        Gam = np.exp(G)
        A = np.tril((Qc * Gam) @ (Kc / Gam).T)
        if ut_with_decay:
            Mk = np.tril(bc[:, None] * ((Kc * Gam) @ (Kc / Gam).T), -1)
            Kw = Kc * Gam
        else:
            Mk = np.tril(bc[:, None] * (Kc @ Kc.T), -1)
            Kw = Kc
        Tinv = np.linalg.inv(np.eye(e - s) + Mk)
        U = Tinv @ (bc[:, None] * Vc)
        W = Tinv @ (bc[:, None] * Kw)
        Vt = U - W @ S
        o[s:e] = scale * ((Qc * Gam) @ S + A @ Vt)
        Kd = Kc * np.exp(G[-1][None, :] - G)
        S = np.exp(G[-1])[:, None] * S + Kd.T @ Vt
        M = (np.diag(np.exp(G[-1])) - Kd.T @ W) @ M
    return o, S, M


def chunk_backward(q, k, v, g, beta, S0, do, dS_T, chunk=16, scale=1.0):
    """Reverse pass of ``chunk_run`` (ut_with_decay=True), chunk by chunk in
    reverse order, for one chain with activated inputs.  Returns the gradients
    of <do, o> + <dS_T, S_T> w.r.t. (q, k, v, g, beta, S0) as a dict.

    It differentiates the chunk equations above term by term (the pages print
    no backward): with S the state entering a chunk and dS' the gradient of the
    state leaving it,

        dVt = scale A^T dO + Kd dS'          dS = scale Qg^T dO + Diag(gamma_C) dS' - W^T dVt
        dQg = scale (dO S^T + tril(dO Vt^T) Kn)
        dKn = scale tril(dO Vt^T)^T Qg + dMk^T Diag(beta) Kw
        dKd = Vt dS'^T,  dgamma_C = rowsum(S * dS')
        [dU | dW] = [dVt | -dVt S^T];  dX = (I + Mk)^-T [dU | dW];
        dMk = tril(-dX [U | W]^T, -1)  (X = Diag(beta) [V | Kw])
        dV = Diag(beta) dX_v;  dKw = Diag(beta) (dX_w + dMk Kn)
        dbeta = rowsum(dX_v * V) + rowsum(dX_w * Kw) + rowsum(dMk * (Kw Kn^T))

    and then through Qg = Q Gamma, Kn = K / Gamma, Kw = K Gamma,
    Kd = K gamma_C / Gamma, gamma_C = Gamma_C, Gamma = exp(cumsum g): the
    per-token dG collects +dQg*Qg - dKn*Kn + dKw*Kw - dKd*Kd, the last row adds
    sum_r dKd_r*Kd_r + dgamma_C*gamma_C, and dg is the reverse cumulative sum of
    dG within the chunk.  The entering states are recomputed by a forward
    sweep, as a kernel would store them at chunk boundaries.
    """
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, Dk = k.shape
    Dv = v.shape[1]
    S = np.zeros((Dk, Dv)) if S0 is None else np.array(S0, dtype=np.float64)
    starts = list(range(0, T, chunk))
    states = []
    for s in starts:                                 # forward sweep: entering states
        states.append(S.copy())
        e = min(s + chunk, T)
        _, S, _ = chunk_run(q[s:e], k[s:e], v[s:e], g[s:e], beta[s:e], S, chunk=chunk, scale=scale)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, db = np.zeros_like(g), np.zeros_like(beta)
    dS = np.array(dS_T, dtype=np.float64)
    for s, S in zip(reversed(starts), reversed(states)):
        e = min(s + chunk, T)
        Q, K, V, b, dO = q[s:e], k[s:e], v[s:e], beta[s:e], do[s:e]
        G = np.cumsum(g[s:e], axis=0)
        Gam = np.exp(G)
        gC = Gam[-1]
        Qg, Kn, Kw, Kd = Q * Gam, K / Gam, K * Gam, K * (gC[None, :] / Gam)
        A = np.tril(Qg @ Kn.T)
        Mk = np.tril(b[:, None] * (Kw @ Kn.T), -1)
        L = np.eye(e - s) + Mk
        U = np.linalg.solve(L, b[:, None] * V)
        W = np.linalg.solve(L, b[:, None] * Kw)
        Vt = U - W @ S
        dVt = scale * A.T @ dO + Kd @ dS
        dS_in = scale * Qg.T @ dO + gC[:, None] * dS - W.T @ dVt
        dA = scale * np.tril(dO @ Vt.T)
        dQg = scale * dO @ S.T + dA @ Kn
        dKn = dA.T @ Qg
        dKd = Vt @ dS.T
        dgC = (S * dS).sum(1)
        dXv = np.linalg.solve(L.T, dVt)
        dXw = np.linalg.solve(L.T, -dVt @ S.T)
        dMk = np.tril(-(dXv @ U.T + dXw @ W.T), -1)
        dv[s:e] = b[:, None] * dXv
        db[s:e] = (dXv * V).sum(1) + (dXw * Kw).sum(1) + (dMk * (Kw @ Kn.T)).sum(1)
        dKw = b[:, None] * (dXw + dMk @ Kn)
        dKn = dKn + dMk.T @ (b[:, None] * Kw)
        dq[s:e] = dQg * Gam
        dk[s:e] = dKn / Gam + dKw * Gam + dKd * (gC[None, :] / Gam)
        dG = dQg * Qg - dKn * Kn + dKw * Kw - dKd * Kd
        dG[-1] += (dKd * Kd).sum(0) + dgC * gC
        dg[s:e] = np.cumsum(dG[::-1], axis=0)[::-1]
        dS = dS_in
    return {"q": dq, "k": dk, "v": dv, "g": dg, "beta": db, "S0": dS}
