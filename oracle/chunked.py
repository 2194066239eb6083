"""Staged fp64 restatement of the chunkwise gated delta-rule forward.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  It is a debugging aid
that exposes the per-chunk intermediate matrices, so that a kernel stage can
be checked on its own.  Its end results are pinned to the token recurrence in
``gdr_fwd`` (tests/test_oracle_pins.py).

Source: "Decoding Hybrid Linear Attention Architectures", section 5
(inter-chunk state recursion and intra-chunk output computation), with the
WY/UT representation of the product of (I - beta k k^T) factors named in
"Linear Attention Variants (RetNet, GLA, DeltaNet, Based)", section "DeltaNet:
Error-Correcting Writes" and interview question 2.

Notation (one chunk of L <= C rows, X = S^T of shape d_k x d_v):
    g_r   = sum_{s<=r} log alpha_s      (log-space accumulation, section 5)
    b_r   = exp(g_r)                    (decay from chunk start to row r)
    K~ = K * b,  K^ = K / b,  Q~ = Q * b,  K- = K * (b_L / b)
    A  = strict_tril(Diag(beta) K~ K^^T)
    T  = (I + A)^{-1} Diag(beta)
    W  = T K~,  U = T V
    V' = U - W X                        ("net correction", section 5)
    O  = Q~ X + tril_incl(Q~ K^^T) V'   (intra-chunk output)
    X <- Diag(b_L) X + K-^T V'          (inter-chunk recursion)

Reading: the page labels the decay on Q with the chunk-end symbol, but the
derivation needs the decay from the chunk start to row r (b_r) on Q and the
division by that same decay on K; only the state update uses the decay to
the chunk end.  The output mask includes the diagonal (o_t reads S_t after
the write); the A mask excludes it.
"""
from __future__ import annotations

import numpy as np


def _widen(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:  # bf16 bit patterns
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def chunk_fwd_head(q, k, v, g, beta, S0=None, C=64, keep_stages=False):
    """One (batch, head).  q,k [T,dk]; v [T,dv]; g [T] or [T,dk]; beta [T].

    Returns (o [T,dv], S_T [dv,dk], stages) where stages is a list of dicts
    (one per chunk) when keep_stages is true, else None.
    """
    q, k, v = _widen(q), _widen(k), _widen(v)
    g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    X = np.zeros((dk, dv)) if S0 is None else np.array(S0, np.float64).T.copy()
    o = np.zeros((T, dv))
    stages = [] if keep_stages else None
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        L = c1 - c0
        Q, K, V, bt = q[c0:c1], k[c0:c1], v[c0:c1], beta[c0:c1]
        gc = np.cumsum(g[c0:c1], axis=0)
        b = np.exp(gc)
        if b.ndim == 1:
            b = np.repeat(b[:, None], dk, axis=1)
        Kt, Kh, Qt = K * b, K / b, Q * b
        Kb = K * (b[L - 1][None, :] / b)
        A = np.tril(bt[:, None] * (Kt @ Kh.T), -1)
        Tm = np.linalg.solve(np.eye(L) + A, np.diag(bt))
        W, U = Tm @ Kt, Tm @ V
        X0 = X
        Vp = U - W @ X0
        P = np.tril(Qt @ Kh.T, 0)
        O = Qt @ X0 + P @ Vp
        X = b[L - 1][:, None] * X0 + Kb.T @ Vp
        o[c0:c1] = O
        if keep_stages:
            stages.append(dict(g=gc, A=A, T=Tm, W=W, U=U, X0=X0, Vp=Vp, P=P, O=O, X1=X.copy()))
    return o, X.T.copy(), stages


def chunk_fwd(q, k, v, g, beta, S0=None, C=64):
    """All (batch, head) pairs; layouts as ``oracle.gdr_fwd``.  Returns (o, S_T)."""
    q = np.asarray(q)
    B, T, H, dk = q.shape
    dv = np.asarray(v).shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            s0 = None if S0 is None else np.asarray(S0)[b, h]
            gg = np.asarray(g)[b, :, h]
            ob, sb, _ = chunk_fwd_head(q[b, :, h], np.asarray(k)[b, :, h], np.asarray(v)[b, :, h],
                                       gg, np.asarray(beta)[b, :, h], s0, C)
            o[b, :, h] = ob
            S_T[b, h] = sb
    return o, S_T
