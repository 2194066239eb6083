"""Pins for the oracle's DPLR recurrence ("Decoding Hybrid Linear Attention
Architectures", section 3 item 5): S_t = S_{t-1}(Diag(alpha_t) + a_t b_t^T)
+ v_t k_t^T, o_t = S_t q_t.  CPU only."""
import numpy as np
import pytest

import oracle
from tests._pins import rel_err

RNG = np.random.default_rng(2024)


def _inputs(B, T, H, dk, dv, gate):
    f = lambda *s: RNG.standard_normal(s).astype(np.float32)
    q, k, a, b = f(B, T, H, dk), f(B, T, H, dk), f(B, T, H, dk), f(B, T, H, dk)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a *= 0.1
    b *= 0.1
    v = f(B, T, H, dv)
    gs = (B, T, H, dk) if gate == "channel" else (B, T, H)
    g = (-0.3 * np.log1p(np.exp(RNG.standard_normal(gs)))).astype(np.float32)
    s0 = 0.5 * RNG.standard_normal((B, H, dv, dk))
    return q, k, v, a, b, g, s0


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_dplr_matches_explicit_product(gate):
    """S_T = S0 M_1 ... M_T + sum_s v_s k_s^T M_{s+1} ... M_T with dense
    M_t = Diag(alpha_t) + a_t b_t^T, formed from scratch for every t."""
    B, T, H, dk, dv = 1, 7, 2, 4, 3
    q, k, v, a, b, g, s0 = _inputs(B, T, H, dk, dv, gate)
    o, S_T = oracle.dplr_fwd(q, k, v, a, b, g, s0, gate=gate)
    for h in range(H):
        M = []
        for t in range(T):
            al = np.exp(g[0, t, h].astype(np.float64)) * np.ones(dk)
            M.append(np.diag(al) + np.outer(a[0, t, h].astype(np.float64), b[0, t, h].astype(np.float64)))
        for t in range(T):
            P = np.eye(dk)
            for r in range(t + 1):
                P = P @ M[r]
            S = s0[0, h] @ P
            for s_ in range(t + 1):
                Q = np.eye(dk)
                for r in range(s_ + 1, t + 1):
                    Q = Q @ M[r]
                S = S + np.outer(v[0, s_, h].astype(np.float64), k[0, s_, h].astype(np.float64)) @ Q
            assert rel_err(o[0, t, h], S @ q[0, t, h].astype(np.float64)) < 1e-12
        assert rel_err(S_T[0, h], S) < 1e-12


def test_dplr_reduces_to_gated_delta_rule():
    """a = -beta (alpha . k), b = k, v -> beta v is the gated delta rule with a
    per-channel gate (decay, erase along k, write; [HLA] section 3 item 6).
    a and beta v are formed in fp32, so the two agree to fp32 rounding."""
    B, T, H, dk, dv = 2, 9, 2, 5, 4
    q, k, v, _, _, g, s0 = _inputs(B, T, H, dk, dv, "channel")
    beta = (1 / (1 + np.exp(-RNG.standard_normal((B, T, H))))).astype(np.float32)
    a = (-beta[..., None] * np.exp(g.astype(np.float64)) * k).astype(np.float32)
    vb = (beta[..., None] * v).astype(np.float32)
    o, S_T = oracle.dplr_fwd(q, k, vb, a, k, g, s0, gate="channel")
    og, Sg = oracle.gdr_fwd(q, k, v, g, beta, s0, gate="channel")
    assert rel_err(o, og) < 1e-6 and rel_err(S_T, Sg) < 1e-6


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_dplr_without_low_rank_is_gla(gate):
    q, k, v, a, b, g, s0 = _inputs(2, 8, 2, 4, 3, gate)
    a[:] = 0.0
    o, S_T = oracle.dplr_fwd(q, k, v, a, b, g, s0, gate=gate)
    ol, Sl = oracle.gla_fwd(q, k, v, g, s0, gate=gate)
    assert rel_err(o, ol) < 1e-13 and rel_err(S_T, Sl) < 1e-13


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_dplr_chunk_form_matches_recurrence(gate):
    """The chunk form (a unit lower-triangular solve for the low-rank reads,
    then the chunk's output and end state as matrix products) equals the
    recurrence: C = 16 over 40 tokens (two chunks and a ragged tail)."""
    from oracle import chunked

    q, k, v, a, b, g, s0 = _inputs(1, 40, 1, 6, 5, gate)
    o, S_T = oracle.dplr_fwd(q, k, v, a, b, g, s0, gate=gate)
    oc, Sc = chunked.dplr_chunk_fwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], a[0, :, 0],
                                         b[0, :, 0], g[0, :, 0], s0[0, 0], C=16)
    assert rel_err(oc, o[0, :, 0]) < 1e-10 and rel_err(Sc, S_T[0, 0]) < 1e-10


def test_constant_channel_gate_is_the_scalar_gate():
    """DPLR and GLA with a per-channel gate equal in every channel match their
    scalar-gate runs (the gate reaches every key channel alike)."""
    q, k, v, a, b, g, s0 = _inputs(2, 8, 2, 4, 3, "scalar")
    gc = np.repeat(g[..., None], 4, axis=-1)
    o1, S1 = oracle.dplr_fwd(q, k, v, a, b, g, s0, gate="scalar")
    o2, S2 = oracle.dplr_fwd(q, k, v, a, b, gc, s0, gate="channel")
    assert rel_err(o1, o2) < 1e-14 and rel_err(S1, S2) < 1e-14
    o1, S1 = oracle.gla_fwd(q, k, v, g, s0, gate="scalar")
    o2, S2 = oracle.gla_fwd(q, k, v, gc, s0, gate="channel")
    assert rel_err(o1, o2) < 1e-14 and rel_err(S1, S2) < 1e-14
