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


def chunk_bwd_head(q, k, v, g, beta, dO, S0=None, dS_T=None, C=64):
    """Gradients of ``chunk_fwd_head`` by reverse mode through the chunk
    equations ("Decoding Hybrid Linear Attention Architectures", section 5:
    backpropagation through the chunked recurrence, with the chunk's
    quantities recomputed), written as matrix products per chunk: the form a
    chunked backward kernel computes.  Pinned to the token-level backward
    ``oracle.gdr_bwd``.

    One (batch, head): q, k [T,dk]; v, dO [T,dv]; g [T] or [T,dk]; beta [T];
    S0, dS_T [dv,dk] or None.  Returns dict dq, dk, dv, dg (shape of g),
    dbeta, dS0.

    Per chunk (forward notation above; Y = (I + A)^{-1}, T = Y Diag(beta)),
    from dO and dX1 = dL/dX after the chunk:
        dV'  = P^T dO + K- dX1
        dX0  = Q~^T dO + Diag(b_L) dX1 - W^T dV'
        dP   = tril_incl(dO V'^T):  dQ~ = dO X0^T + dP K^,  dK^ = dP^T Q~
        dK-  = V' dX1^T
        dT   = dV' V^T - dV' X0^T K~^T;  dV = T^T dV';  dK~ = -T^T dV' X0^T
        dY   = dT Diag(beta);  dbeta += diag(Y^T dT) (column sums of Y . dT)
        dA   = strict_tril(-Y^T dY Y^T):  dbeta_r += sum_s dA M,
               dK~ += Diag(beta) dA K^,  dK^ += (Diag(beta) dA)^T K~   (M = K~ K^^T)
    then through K~ = K b, K^ = K / b, Q~ = Q b, K- = K b_L / b, b = e^{gc},
    gc = cumsum(g) (and b_L = b of the last row, which also scales X0).
    """
    q, k, v = _widen(q), _widen(k), _widen(v)
    g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    dO = np.asarray(dO, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    scalar = g.ndim == 1
    _, _, st = chunk_fwd_head(q, k, v, g, beta, S0, C, keep_stages=True)
    out = dict(dq=np.zeros((T, dk)), dk=np.zeros((T, dk)), dv=np.zeros((T, dv)),
               dg=np.zeros(g.shape), dbeta=np.zeros(T))
    dX = np.zeros((dk, dv)) if dS_T is None else np.array(dS_T, np.float64).T.copy()
    for ci in range(len(st) - 1, -1, -1):
        c0 = ci * C
        s = st[ci]
        L = s["O"].shape[0]
        Q, K, V, bt = q[c0:c0 + L], k[c0:c0 + L], v[c0:c0 + L], beta[c0:c0 + L]
        b = np.exp(s["g"])
        if b.ndim == 1:
            b = np.repeat(b[:, None], dk, axis=1)
        bL = b[L - 1]
        Kt, Kh, Qt, Kb = K * b, K / b, Q * b, K * (bL[None, :] / b)
        X0, Vp, P, W, Tm = s["X0"], s["Vp"], s["P"], s["W"], s["T"]
        Y = np.linalg.inv(np.eye(L) + s["A"])
        dOc = dO[c0:c0 + L]
        dX1 = dX
        dVp = P.T @ dOc + Kb @ dX1
        dX0 = Qt.T @ dOc + bL[:, None] * dX1 - W.T @ dVp
        dP = np.tril(dOc @ Vp.T, 0)
        dQt = dOc @ X0.T + dP @ Kh
        dKh = dP.T @ Qt
        dKb = Vp @ dX1.T
        dbL = np.sum(dX1 * X0, axis=1)
        dW = -dVp @ X0.T
        dTm = dVp @ V.T + dW @ Kt.T
        dV = Tm.T @ dVp
        dKt = Tm.T @ dW
        dY = dTm * bt[None, :]
        dbeta = np.sum(Y * dTm, axis=0)
        dA = np.tril(-(Y.T @ dY @ Y.T), -1)
        M = Kt @ Kh.T
        dbeta += np.sum(dA * M, axis=1)
        dM = bt[:, None] * dA
        dKt += dM @ Kh
        dKh += dM.T @ Kt
        dK = dKt * b + dKh / b + dKb * (bL[None, :] / b)
        dQ = dQt * b
        db = dKt * K - dKh * K / b ** 2 + dQt * Q - dKb * K * bL[None, :] / b ** 2
        dbL = dbL + np.sum(dKb * K / b, axis=0)
        dgc = db * b
        dgc[L - 1] += dbL * bL
        if scalar:
            dgc = dgc.sum(axis=1)
        dgs = np.cumsum(dgc[::-1], axis=0)[::-1]  # gc = cumsum(g)
        out["dq"][c0:c0 + L] = dQ
        out["dk"][c0:c0 + L] = dK
        out["dv"][c0:c0 + L] = dV
        out["dg"][c0:c0 + L] = dgs
        out["dbeta"][c0:c0 + L] = dbeta
        dX = dX0
    out["dS0"] = dX.T.copy()
    return out


def dplr_chunk_fwd_head(q, k, v, a, b, g, S0=None, C=64):
    """Chunk form of the diagonal-plus-low-rank recurrence ("Decoding Hybrid
    Linear Attention Architectures", section 3 item 5, chunked as section 5
    chunks the delta rule), one (batch, head), state S [dv, dk]:

        S_r = S_{r-1} (Diag(alpha_r) + a_r b_r^T) + v_r k_r^T,   o_r = S_r q_r.

    Within a chunk, with e_r = prod_{u<=r} alpha_u (from the chunk start,
    e_{-1} = 1), the low-rank reads x_r = S_{r-1} a_r satisfy
        x_r = S_0 a^_r + sum_{s<r} x_s (b^_s . a^_r) + sum_{s<r} v_s (k^_s . a^_r),
        a^_r = a_r e_{r-1},  b^_s = b_s / e_s,  k^_s = k_s / e_s,
    a unit lower-triangular system (the delta rule's WY structure with the
    erase direction b and the write key k kept apart):
        X = (I - strict_tril(A^ B^^T))^{-1} (A^ S_0^T + strict_tril(A^ K^^T) V)
    and then, with q~_r = q_r e_r,
        O   = Q~ S_0^T + tril_incl(Q~ B^^T) X + tril_incl(Q~ K^^T) V
        S_L^T = Diag(e_L) S_0^T + (B e_L / e)^T X + (K e_L / e)^T V.
    q, k, a, b [T,dk]; v [T,dv]; g [T] or [T,dk]; S0 [dv,dk] or None.
    Returns (o [T,dv], S_T [dv,dk]).  Pinned to ``oracle.dplr_fwd``."""
    q, k, v, a, b = (_widen(x) for x in (q, k, v, a, b))
    g = np.asarray(g, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    St = np.zeros((dk, dv)) if S0 is None else np.array(S0, np.float64).T.copy()  # S^T
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        L = c1 - c0
        Q, K, V, Aa, Bb = q[c0:c1], k[c0:c1], v[c0:c1], a[c0:c1], b[c0:c1]
        e = np.exp(np.cumsum(g[c0:c1], axis=0))
        if e.ndim == 1:
            e = np.repeat(e[:, None], dk, axis=1)
        eprev = np.vstack([np.ones((1, dk)), e[:-1]])
        Ah, Bh, Kh, Qt = Aa * eprev, Bb / e, K / e, Q * e
        Lb = np.tril(Ah @ Bh.T, -1)
        Lk = np.tril(Ah @ Kh.T, -1)
        X = np.linalg.solve(np.eye(L) - Lb, Ah @ St + Lk @ V)
        O = Qt @ St + np.tril(Qt @ Bh.T, 0) @ X + np.tril(Qt @ Kh.T, 0) @ V
        eL = e[L - 1]
        St = eL[:, None] * St + (Bb * (eL[None, :] / e)).T @ X + (K * (eL[None, :] / e)).T @ V
        o[c0:c1] = O
    return o, St.T.copy()
