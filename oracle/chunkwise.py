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
