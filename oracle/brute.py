"""Dense affine-product form of the KDA recurrence, for tiny shapes only.

TEST INFRASTRUCTURE (see oracle/__init__.py).  An independent NumPy restatement
used to pin the C oracle: every token is written as the affine map

    S_t = M_t S_{t-1} + B_t,   M_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
                               B_t = beta_t k_t v_t^T

(page "Implémenter KDA", "Test 2 - l'identité de composition" gives M_t; the
affine structure S_t = M_t S_{t-1} + B_t is stated in "Que teste réellement le
test 2 ?").  The state after token t is then the explicit sum

    S_t = (M_t ... M_1) S_0 + sum_{i<=t} (M_t ... M_{i+1}) B_i

built from dense matrices, and o_t = S_t^T q_t.  No switches: the inputs are the
already-preprocessed q, k (used as given), alpha = exp(g) and beta.
"""
import numpy as np


def transition(k, alpha, beta):
    """Dense M_t = (I - beta k k^T) Diag(alpha)."""
    Dk = k.shape[0]
    return (np.eye(Dk) - beta * np.outer(k, k)) @ np.diag(alpha)


def affine_run(q, k, v, g, beta, S0=None, scale=1.0):
    """One chain.  q,k [T,Dk]; v [T,Dv]; g [T,Dk] (log-decay); beta [T];
    S0 [Dk,Dv] or None.  Returns (o [T,Dv], S_T [Dk,Dv], M_T [Dk,Dk])."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, Dk = k.shape
    Dv = v.shape[1]
    S0 = np.zeros((Dk, Dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    alpha = np.exp(g)
    Ms = [transition(k[t], alpha[t], beta[t]) for t in range(T)]
    Bs = [beta[t] * np.outer(k[t], v[t]) for t in range(T)]
    o = np.zeros((T, Dv))
    S_t = S0
    for t in range(T):
        # (M_t ... M_1) S0
        P = np.eye(Dk)
        for s in range(t + 1):
            P = Ms[s] @ P
        S_t = P @ S0
        # + sum_i (M_t ... M_{i+1}) B_i
        for i in range(t + 1):
            Pi = np.eye(Dk)
            for s in range(i + 1, t + 1):
                Pi = Ms[s] @ Pi
            S_t = S_t + Pi @ Bs[i]
        o[t] = scale * (S_t.T @ q[t])
    M_T = np.eye(Dk)
    for t in range(T):
        M_T = Ms[t] @ M_T
    return o, (S_t if T > 0 else S0.copy()), M_T
