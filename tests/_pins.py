"""Independent fp64 reference forms used to pin the oracle (tests only).

Each is written from the equations, not from the oracle's code, and takes a
different computational route, so that a dropped term, a sign, an index or a
transposed operand in the oracle shows up as a mismatch.
"""
from __future__ import annotations

import numpy as np


def widen(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def brute_force_head(q, k, v, g, beta, S0=None, order="decay_first"):
    """Explicit product form of the recurrence for one (b, h).

    With M_r = Diag(alpha_r)(I - beta_r k_r k_r^T) (decay first) the state is
        S_t = S0 M_1 ... M_t + sum_{s<=t} beta_s v_s k_s^T M_{s+1} ... M_t,
    and o_t = S_t q_t.  Every M_r is built as a dense d_k x d_k matrix and the
    products are formed from scratch for every t (cost O(T^2 d^3): tiny inputs
    only).  order="erase_first" builds M_r = (I - beta k k^T) Diag(alpha)
    instead (used to show that the per-channel order matters).
    """
    q, k, v = widen(q), widen(k), widen(v)
    g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    S0 = np.zeros((dv, dk)) if S0 is None else np.asarray(S0, np.float64)
    I = np.eye(dk)
    Ms = []
    for r in range(T):
        alpha = np.exp(g[r]) * np.ones(dk) if np.ndim(g[r]) == 0 else np.exp(g[r])
        P = I - beta[r] * np.outer(k[r], k[r])
        Ms.append(np.diag(alpha) @ P if order == "decay_first" else P @ np.diag(alpha))
    o = np.zeros((T, dv))
    S_t = S0
    for t in range(T):
        prod = I.copy()
        for r in range(t + 1):
            prod = prod @ Ms[r]
        S_t = S0 @ prod
        for s in range(t + 1):
            tail = I.copy()
            for r in range(s + 1, t + 1):
                tail = tail @ Ms[r]
            S_t = S_t + beta[s] * np.outer(v[s], k[s]) @ tail
        o[t] = S_t @ q[t]
    return o, S_t


def deltanet_projector_head(q, k, v, beta, S0=None):
    """Ungated DeltaNet in its projector form S <- S (I - beta k k^T) + beta v k^T
    ("Linear Attention Variants (RetNet, GLA, DeltaNet, Based)", variant table,
    DeltaNet row written cleanly), with o_t = S_t q_t."""
    q, k, v = widen(q), widen(k), widen(v)
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, np.float64)
    o = np.zeros((T, dv))
    for t in range(T):
        S = S @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        o[t] = S @ q[t]
    return o, S


def rel_err(a, b):
    """max|a-b| / max|b| (the acceptance metric), with 0/0 read as 0."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.max(np.abs(b)) if b.size else 0.0
    num = np.max(np.abs(a - b)) if a.size else 0.0
    if den == 0.0:
        return num
    return num / den
