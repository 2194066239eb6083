"""Pins for the oracle's prologue (raw projections -> q, k, g, beta) and its
fp64-input forward.  CPU only.
  [HLA] "Decoding Hybrid Linear Attention Architectures"
  [LAV] "Linear Attention Variants (RetNet, GLA, DeltaNet, Based)"
"""
import math

import numpy as np
import pytest

import oracle
from oracle import prologue as pro
from tests._pins import brute_force_head, rel_err

RNG = np.random.default_rng(4321)


def test_sigmoid_closed_forms():
    assert pro.sigmoid(0.0) == 0.5
    assert abs(pro.sigmoid(math.log(3.0)) - 0.75) < 1e-15
    x = RNG.standard_normal(100) * 5
    assert np.max(np.abs(pro.sigmoid(-x) - (1.0 - pro.sigmoid(x)))) < 1e-15
    s = pro.sigmoid(np.array([-700.0, 700.0]))
    assert s[0] > 0.0 and s[0] < 1e-300 and s[1] == 1.0


def test_softplus_closed_forms():
    assert abs(pro.softplus(0.0) - math.log(2.0)) < 1e-15
    assert abs(pro.softplus(math.log(math.e - 1.0)) - 1.0) < 1e-15
    x = RNG.standard_normal(100) * 10
    assert np.max(np.abs(pro.softplus(x) - pro.softplus(-x) - x)) < 1e-12
    assert pro.softplus(800.0) == 800.0 and 0.0 < pro.softplus(-700.0) < 1e-300


def test_log_decay_is_per_head_and_nonpositive():
    """g = -s_h softplus(a): alpha = e^g in (0, 1]; the scale follows the head
    axis ([HLA] section 4, forgetting rate per head or per channel)."""
    a = np.broadcast_to(RNG.standard_normal((1, 5, 1)), (2, 5, 3)).copy()
    s = np.array([0.1, 0.5, 2.0])
    g = pro.log_decay(a, s)
    assert np.all(g <= 0)
    for h in range(3):
        assert np.allclose(g[:, :, h] / s[h], -pro.softplus(a[:, :, 0]), rtol=1e-14, atol=0)
    a4 = RNG.standard_normal((2, 5, 3, 4))
    g4 = pro.log_decay(a4, s)
    assert g4.shape == a4.shape
    assert np.allclose(g4[:, :, 2] / 2.0, -pro.softplus(a4[:, :, 2]), rtol=1e-14, atol=0)


def test_l2_normalise():
    x = RNG.standard_normal((3, 7, 2, 16)) * 4
    y = pro.l2_normalise(x)
    n = np.linalg.norm(y, axis=-1)
    assert np.max(np.abs(n - 1.0)) < 1e-6  # eps = 1e-6 against |x|^2 ~ 256
    assert np.max(np.abs(pro.l2_normalise(3.5 * x) - y)) < 1e-8
    assert np.all(pro.l2_normalise(np.zeros((2, 4))) == 0.0)


def _raw(B, T, H, dk, dv, gate="scalar"):
    q = (RNG.standard_normal((B, T, H, dk)) * 3).astype(np.float32)
    k = (RNG.standard_normal((B, T, H, dk)) * 3).astype(np.float32)
    v = RNG.standard_normal((B, T, H, dv)).astype(np.float32)
    a = RNG.standard_normal((B, T, H, dk) if gate == "channel" else (B, T, H)).astype(np.float32)
    b = RNG.standard_normal((B, T, H)).astype(np.float32)
    s = (0.05 + 0.3 * RNG.random(H)).astype(np.float32)
    return q, k, v, a, b, s


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_f64_forward_matches_explicit_product(gate):
    """The fp64-input forward equals the explicit product of
    Diag(alpha)(I - beta k k^T) factors ([HLA] section 3 items 3 and 6) on
    inputs that only fp64 holds exactly (1/3-scaled values)."""
    B, T, H, dk, dv = 1, 8, 2, 4, 3
    q, k, v, a, b, s = _raw(B, T, H, dk, dv, gate)
    q, k, g, beta = pro.prologue(q / 3.0, k / 3.0, a, b, s)
    v = v.astype(np.float64) / 3.0
    s0 = RNG.standard_normal((B, H, dv, dk)) / 3.0
    o, S_T = oracle.gdr_fwd_f64(q, k, v, g, beta, s0, gate=gate)
    for h in range(H):
        ob, sb = brute_force_head(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], beta[0, :, h],
                                  s0[0, h])
        assert rel_err(o[0, :, h], ob) < 1e-12 and rel_err(S_T[0, h], sb) < 1e-12


def test_prologue_forward_is_scale_invariant_in_q_and_k():
    """Rescaling the raw q or k rows leaves the output unchanged when both are
    normalised; without q's normalisation the output is linear in q."""
    q, k, v, a, b, s = _raw(2, 10, 2, 8, 5)
    o, S_T = oracle.gdr_fwd_prologue(q, k, v, a, b, s)
    o2, S2 = oracle.gdr_fwd_prologue(2.5 * q, 0.25 * k, v, a, b, s)
    # exact up to eps / |x|^2 (eps = 1e-6, |0.25 k|^2 ~ 4.5)
    assert rel_err(o2, o) < 1e-5 and rel_err(S2, S_T) < 1e-5
    on, _ = oracle.gdr_fwd_prologue(q, k, v, a, b, s, norm_q=False)
    on3, _ = oracle.gdr_fwd_prologue(3.0 * q.astype(np.float64), k, v, a, b, s, norm_q=False)
    assert rel_err(on3, 3.0 * on) < 1e-12
    assert rel_err(on, o) > 1e-2


def test_prologue_saturated_write_retrieves_value():
    """b -> +inf gives beta -> 1; with a normalised key and q = k the output is
    the value just written, whatever the state and the gate ([HLA] section 3
    item 2: the write replaces what k_t mapped to)."""
    q, k, v, a, b, s = _raw(1, 6, 1, 8, 4)
    b[:] = 60.0  # sigmoid(60) = 1 - 9e-27
    s0 = RNG.standard_normal((1, 1, 4, 8))
    o, _ = oracle.gdr_fwd_prologue(5.0 * k, k, v, a, b, s, S0=s0)
    # |k^|^2 = 1 - eps / |k|^2 (eps = 1e-6, |k|^2 ~ 72): exact to ~1e-7
    assert np.max(np.abs(o - v.astype(np.float64))) < 1e-6


def test_prologue_gate_logits_to_minus_inf_remove_forgetting():
    """a -> -inf gives alpha -> 1 (no forgetting): the forward equals the
    recurrence with g = 0 on the same normalised keys."""
    q, k, v, a, b, s = _raw(1, 9, 2, 6, 3)
    a[:] = -200.0  # softplus(-200) = e^-200
    o, S_T = oracle.gdr_fwd_prologue(q, k, v, a, b, s)
    qn, kn, _, beta = pro.prologue(q, k, a, b, s)
    o0, S0_ = oracle.gdr_fwd_f64(qn, kn, v, np.zeros_like(beta), beta)
    assert rel_err(o, o0) < 1e-14 and rel_err(S_T, S0_) < 1e-14
