"""Pins for the oracle's backward (reverse mode over the token recurrence).

CPU only.  The gradients are checked against central finite differences of
the fp64 forward (``gdr_fwd_f64``), which shares no code with the backward.
  [HLA] "Decoding Hybrid Linear Attention Architectures", section 5
  (backpropagation through the recurrence, with recomputation).
"""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(777)


def _inputs(B, T, H, dk, dv, gate):
    q = RNG.standard_normal((B, T, H, dk)).astype(np.float32)
    k = RNG.standard_normal((B, T, H, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = RNG.standard_normal((B, T, H, dv)).astype(np.float32)
    gs = (B, T, H, dk) if gate == "channel" else (B, T, H)
    g = (-0.3 * np.log1p(np.exp(RNG.standard_normal(gs)))).astype(np.float32)
    beta = (1 / (1 + np.exp(-RNG.standard_normal((B, T, H))))).astype(np.float32)
    s0 = 0.5 * RNG.standard_normal((B, H, dv, dk))
    return q, k, v, g, beta, s0


def _loss(x, Wo, WS, gate):
    o, S = oracle.gdr_fwd_f64(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gate=gate,
                              nthreads=1)
    return float(np.sum(o * Wo) + np.sum(S * WS))


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("with_dST", [True, False])
def test_backward_matches_finite_differences(gate, with_dST):
    B, T, H, dk, dv = 1, 6, 2, 3, 4
    q, k, v, g, beta, s0 = _inputs(B, T, H, dk, dv, gate)
    Wo = RNG.standard_normal((B, T, H, dv))
    WS = RNG.standard_normal((B, H, dv, dk)) if with_dST else np.zeros((B, H, dv, dk))
    grads = oracle.gdr_bwd(q, k, v, g, beta, Wo, s0, WS if with_dST else None, gate=gate,
                           nthreads=1)
    x = {n: a.astype(np.float64) for n, a in
         dict(q=q, k=k, v=v, g=g, beta=beta, S0=s0).items()}
    h = 1e-6
    for name, gname in [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"),
                        ("beta", "dbeta"), ("S0", "dS0")]:
        fd = np.zeros_like(x[name])
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[name][idx]
            x[name][idx] = old + h
            lp = _loss(x, Wo, WS, gate)
            x[name][idx] = old - h
            lm = _loss(x, Wo, WS, gate)
            x[name][idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(grads[gname] - fd)) / max(1e-12, np.max(np.abs(fd)))
        assert err < 1e-6, f"{gname}: relative error {err:.2e}"


def test_backward_of_empty_sequence_passes_dST_through():
    q, k, v, g, beta, s0 = _inputs(1, 0, 1, 4, 3, "scalar")
    WS = RNG.standard_normal((1, 1, 3, 4))
    grads = oracle.gdr_bwd(q, k, v, g, beta, np.zeros((1, 0, 1, 3)), s0, WS)
    assert np.array_equal(grads["dS0"], WS)


def test_backward_beta_zero_is_pure_decay():
    """beta = 0: S_T = S0 Diag(prod alpha), o_t = S_t q_t, so dv = 0 and
    dS0 = dS_T Diag(prod alpha) + sum_t do_t q_t^T Diag(prod_{s<=t} alpha_s)
    (closed form)."""
    B, T, H, dk, dv = 1, 5, 1, 3, 2
    q, k, v, g, beta, s0 = _inputs(B, T, H, dk, dv, "channel")
    beta[:] = 0.0
    Wo = RNG.standard_normal((B, T, H, dv))
    WS = RNG.standard_normal((B, H, dv, dk))
    grads = oracle.gdr_bwd(q, k, v, g, beta, Wo, s0, WS, gate="channel")
    assert np.max(np.abs(grads["dv"])) == 0.0
    cum = np.cumsum(g[0, :, 0].astype(np.float64), axis=0)  # [T, dk]
    want = WS[0, 0] * np.exp(cum[-1])[None, :]
    for t in range(T):
        want = want + np.outer(Wo[0, t, 0], q[0, t, 0].astype(np.float64) * np.exp(cum[t]))
    assert np.max(np.abs(grads["dS0"][0, 0] - want)) < 1e-12 * np.max(np.abs(want))


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_chunked_backward_matches_token_backward(gate):
    """The chunk-level reverse mode (matrix products per chunk, the form of a
    chunked backward kernel) equals the token-level backward: C = 16 over 40
    tokens (two full chunks and a ragged tail)."""
    from oracle import chunked

    B, T, H, dk, dv = 1, 40, 1, 6, 5
    q, k, v, g, beta, s0 = _inputs(B, T, H, dk, dv, gate)
    Wo = RNG.standard_normal((B, T, H, dv))
    WS = RNG.standard_normal((B, H, dv, dk))
    ref = oracle.gdr_bwd(q, k, v, g, beta, Wo, s0, WS, gate=gate, nthreads=1)
    got = chunked.chunk_bwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0],
                                 Wo[0, :, 0], s0[0, 0], WS[0, 0], C=16)
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        r = ref[name][0, :, 0]
        assert np.max(np.abs(got[name] - r)) <= 1e-9 * max(1.0, np.max(np.abs(r))), name
    assert np.max(np.abs(got["dS0"] - ref["dS0"][0, 0])) <= 1e-9 * np.max(np.abs(ref["dS0"]))


def test_scalar_gate_gradient_is_the_channel_sum():
    """A per-channel gate equal in every channel is the scalar gate: the same
    dq, dk, dv, dbeta, dS0, and the scalar dg is the sum of the per-channel
    dg over channels (the decay multiplies every channel)."""
    B, T, H, dk, dv = 1, 9, 2, 4, 3
    q, k, v, g, beta, s0 = _inputs(B, T, H, dk, dv, "scalar")
    gc = np.repeat(g[..., None], dk, axis=-1)
    Wo = RNG.standard_normal((B, T, H, dv))
    WS = RNG.standard_normal((B, H, dv, dk))
    a = oracle.gdr_bwd(q, k, v, g, beta, Wo, s0, WS, gate="scalar")
    c = oracle.gdr_bwd(q, k, v, gc, beta, Wo, s0, WS, gate="channel")
    for name in ("dq", "dk", "dv", "dbeta", "dS0"):
        assert np.max(np.abs(a[name] - c[name])) <= 1e-12 * np.max(np.abs(c[name])), name
    assert np.max(np.abs(a["dg"] - c["dg"].sum(axis=-1))) <= 1e-12 * np.max(np.abs(a["dg"]))
