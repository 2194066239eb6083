"""Pins for the fp64 oracle, against what the pages and the mathematics fix.

CPU only.  Citations name the page and its section.
  [HLA] "Decoding Hybrid Linear Attention Architectures"
  [LAV] "Linear Attention Variants (RetNet, GLA, DeltaNet, Based)"
"""
import math

import numpy as np
import pytest

import oracle
from oracle import chunked
from tests._pins import brute_force_head, deltanet_projector_head, rel_err, widen

RNG = np.random.default_rng(1234)


def _rand_inputs(B, T, H, dk, dv, gate, dtype="f32", S0=True, rng=RNG, gscale=0.3):
    q = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    if dtype == "bf16":  # round to bf16 and keep the bit patterns
        def tobf(x):
            u = x.astype(np.float32).view(np.uint32)
            u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
            return u
        q, k, v = tobf(q), tobf(k), tobf(v)
    gshape = (B, T, H, dk) if gate == "channel" else (B, T, H)
    g = (-gscale * np.log1p(np.exp(rng.standard_normal(gshape)))).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))).astype(np.float32)
    s0 = (0.5 * rng.standard_normal((B, H, dv, dk))) if S0 else None
    return q, k, v, g, beta, s0


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_oracle_matches_explicit_product(gate, dtype):
    """Oracle == explicit product of Diag(alpha)(I - beta k k^T) factors
    ([HLA] section 3 items 3 and 6; [LAV] DeltaNet section), d_k != d_v."""
    B, T, H, dk, dv = 2, 11, 2, 4, 6
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, gate, dtype)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate=gate, nthreads=2)
    for b in range(B):
        for h in range(H):
            ob, sb = brute_force_head(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h],
                                      beta[b, :, h], s0[b, h])
            assert np.max(np.abs(o[b, :, h] - ob)) <= 1e-12 * max(1.0, np.max(np.abs(ob)))
            assert np.max(np.abs(S_T[b, h] - sb)) <= 1e-12 * max(1.0, np.max(np.abs(sb)))


def test_per_channel_order_is_decay_then_erase():
    """[HLA] section 3 item 6 pseudocode: decay, then erase, then write.  With a
    per-channel gate the other order gives a different state; the oracle must
    follow decay-first and differ from erase-first."""
    B, T, H, dk, dv = 1, 9, 1, 5, 3
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, "channel", gscale=1.0)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate="channel")
    ob, sb = brute_force_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0],
                              s0[0, 0], order="decay_first")
    oe, se = brute_force_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0],
                              s0[0, 0], order="erase_first")
    assert rel_err(S_T[0, 0], sb) < 1e-12
    assert rel_err(S_T[0, 0], se) > 1e-3


def test_scalar_gate_order_immaterial():
    """[HLA] section 3 item 3: with one scalar alpha per head the decay commutes
    with the projector, so both orders give the oracle's result."""
    B, T, H, dk, dv = 1, 9, 1, 5, 3
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, "scalar", gscale=1.0)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate="scalar")
    oe, se = brute_force_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0],
                              s0[0, 0], order="erase_first")
    assert rel_err(o[0, :, 0], oe) < 1e-12
    assert rel_err(S_T[0, 0], se) < 1e-12


# ------------------------------------------------------------- closed forms

@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_beta_zero_is_pure_decay(gate):
    """[HLA] section 4: as beta -> 0 nothing is written.  Then
    S_t = S0 Diag(exp(g_1 + ... + g_t)) and o_t = S_t q_t."""
    B, T, H, dk, dv = 1, 13, 2, 6, 5
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, gate)
    beta[:] = 0.0
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate=gate)
    for h in range(H):
        G = np.cumsum(g[0, :, h].astype(np.float64), axis=0)
        for t in range(T):
            dec = np.exp(G[t]) * np.ones(dk) if gate == "scalar" else np.exp(G[t])
            want = (s0[0, h] * dec[None, :]) @ q[0, t, h].astype(np.float64)
            assert np.allclose(o[0, t, h], want, rtol=1e-12, atol=1e-14)
        dec = np.exp(G[-1]) * np.ones(dk) if gate == "scalar" else np.exp(G[-1])
        assert np.allclose(S_T[0, h], s0[0, h] * dec[None, :], rtol=1e-12, atol=1e-14)


def test_identity_gate_no_write_zero_state_gives_zero():
    """alpha = 1, beta = 0, S0 = 0: the state stays zero, so o is exactly 0."""
    q, k, v, g, beta, _ = _rand_inputs(2, 17, 3, 8, 8, "scalar")
    g[:] = 0.0
    beta[:] = 0.0
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, None)
    assert np.all(o == 0.0) and np.all(S_T == 0.0)


def test_orthonormal_keys_retrieve_written_values():
    """[HLA] sections 3-4: beta -> 1 replaces what is stored along k_t.  With
    alpha = 1, beta = 1 and orthonormal (standard-basis) keys written from a
    zero state, querying key k_j afterwards returns v_j exactly."""
    dk, dv, n = 8, 5, 6
    rng = np.random.default_rng(7)
    perm = rng.permutation(dk)[:n]
    T = 2 * n
    q = np.zeros((1, T, 1, dk), np.float32)
    k = np.zeros((1, T, 1, dk), np.float32)
    v = rng.standard_normal((1, T, 1, dv)).astype(np.float32)
    beta = np.zeros((1, T, 1), np.float32)
    g = np.zeros((1, T, 1), np.float32)
    for j in range(n):  # writes
        k[0, j, 0, perm[j]] = 1.0
        beta[0, j, 0] = 1.0
    for j in range(n):  # reads: beta = 0, query with key j
        k[0, n + j, 0, 0] = 1.0
        q[0, n + j, 0, perm[j]] = 1.0
    o, _ = oracle.gdr_fwd(q, k, v, g, beta, None)
    for j in range(n):
        assert np.array_equal(o[0, n + j, 0], v[0, j, 0].astype(np.float64))


def test_random_orthonormal_keys_retrieve_written_values():
    """Same statement with random orthonormal keys (QR): equal to 1e-12."""
    dk, dv, n = 16, 7, 10
    rng = np.random.default_rng(8)
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :n].T.astype(np.float32)
    # fp32 rounding leaves ||k|| = 1 +- 1e-7; make the fp64 widening exact unit
    # by using the fp32 vector itself as key and query (the identity needs
    # k^T k = 1 only to rounding, so the bound is the fp32 orthonormality).
    T = 2 * n
    q = np.zeros((1, T, 1, dk), np.float32)
    k = np.zeros((1, T, 1, dk), np.float32)
    v = rng.standard_normal((1, T, 1, dv)).astype(np.float32)
    beta = np.zeros((1, T, 1), np.float32)
    g = np.zeros((1, T, 1), np.float32)
    k[0, :n, 0] = keys
    beta[0, :n, 0] = 1.0
    k[0, n:, 0] = keys
    q[0, n:, 0] = keys
    o, _ = oracle.gdr_fwd(q, k, v, g, beta, None)
    kd = keys.astype(np.float64)
    ortho = np.max(np.abs(kd @ kd.T - np.eye(n)))
    for j in range(n):
        assert np.max(np.abs(o[0, n + j, 0] - v[0, j, 0])) <= 20 * ortho * np.max(np.abs(v)) + 1e-12


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_beta_one_unit_key_query_equal_key_returns_value(gate):
    """[HLA] section 4: with beta = 1 the stored value along k_t is replaced, so
    for ||k_t|| = 1 and q_t = k_t the read-out is o_t = v_t, whatever the state
    and the gate.  Keys are +-1/2 on four channels (exactly unit norm)."""
    rng = np.random.default_rng(9)
    B, T, H, dk, dv = 1, 20, 2, 8, 6
    _, _, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, gate, rng=rng)
    k = np.zeros((B, T, H, dk), np.float32)
    for t in range(T):
        for h in range(H):
            idx = rng.permutation(dk)[:4]
            k[0, t, h, idx] = 0.5 * rng.choice([-1.0, 1.0], size=4)
    q = k.copy()
    beta[:] = 1.0
    o, _ = oracle.gdr_fwd(q, k, v, g, beta, s0, gate=gate)
    assert np.max(np.abs(o - v.astype(np.float64))) < 1e-12


def test_alpha_one_is_deltanet():
    """[HLA] section 3 items 2 vs 3 and [LAV] DeltaNet: alpha = 1 reduces the
    gated rule to DeltaNet, here written in its projector form."""
    B, T, H, dk, dv = 1, 15, 2, 6, 4
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, "scalar")
    g[:] = 0.0
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0)
    for h in range(H):
        od, sd = deltanet_projector_head(q[0, :, h], k[0, :, h], v[0, :, h], beta[0, :, h],
                                         s0[0, h])
        assert rel_err(o[0, :, h], od) < 1e-12
        assert rel_err(S_T[0, h], sd) < 1e-12


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_alpha_zero_forgets_in_one_step(gate):
    """[HLA] section 4: a gate near 0 forgets in one step.  With g = -30 at
    every step, S_t = beta_t v_t k_t^T up to exp(-30); no NaN or Inf."""
    B, T, H, dk, dv = 1, 12, 1, 6, 5
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, gate)
    g[:] = -30.0
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate=gate)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S_T))
    kT = k[0, -1, 0].astype(np.float64)
    want = float(beta[0, -1, 0]) * np.outer(v[0, -1, 0].astype(np.float64), kT)
    assert np.max(np.abs(S_T[0, 0] - want)) < 1e-11


# -------------------------------------------------------------- invariants

def test_linearity_in_state_and_values():
    """For fixed q, k, alpha, beta the map (S0, V) -> (o, S_T) is linear
    (every equation in [HLA] section 3 is linear in S and v).  V1, V2 are
    multiples of 1/64 in [-4, 4], so V1 + V2 is exact in fp32."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 1, 19, 2, 6, 5
    q, k, _, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, "channel", rng=rng)
    V1 = (rng.integers(-256, 256, (B, T, H, dv)) / 64.0).astype(np.float32)
    V2 = (rng.integers(-256, 256, (B, T, H, dv)) / 64.0).astype(np.float32)
    o12, s12 = oracle.gdr_fwd(q, k, V1 + V2, g, beta, s0, gate="channel")
    o1, s1 = oracle.gdr_fwd(q, k, V1, g, beta, s0, gate="channel")
    o2, s2 = oracle.gdr_fwd(q, k, V2, g, beta, None, gate="channel")
    assert rel_err(o1 + o2, o12) < 1e-12
    assert rel_err(s1 + s2, s12) < 1e-12


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_split_and_resume(gate):
    """[HLA] sections 1 and 6: the fixed-size state is all that carries over, so
    running T1 tokens, then T2 tokens from S_T1, equals running T1 + T2."""
    B, T, H, dk, dv = 2, 23, 2, 5, 7
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, gate)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate=gate)
    t1 = 9
    oa, Sa = oracle.gdr_fwd(q[:, :t1], k[:, :t1], v[:, :t1], g[:, :t1], beta[:, :t1], s0,
                            gate=gate)
    ob, Sb = oracle.gdr_fwd(q[:, t1:], k[:, t1:], v[:, t1:], g[:, t1:], beta[:, t1:], Sa,
                            gate=gate)
    assert np.array_equal(np.concatenate([oa, ob], axis=1), o)
    assert np.array_equal(Sb, S_T)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_step_api_equals_sequence(gate):
    """The one-token step ([HLA] section 6, constant-cost update) applied T times
    equals the sequence forward."""
    N, T, H, dk, dv = 3, 7, 2, 4, 6
    q, k, v, g, beta, s0 = _rand_inputs(N, T, H, dk, dv, gate)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate=gate)
    S = s0.copy()
    for t in range(T):
        ot = oracle.gdr_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S, gate=gate)
        assert np.array_equal(ot, o[:, t])
    assert np.array_equal(S, S_T)


# ------------------------------------------------------ chunked restatement

@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T,C", [(64, 16), (53, 16), (40, 64), (130, 32)])
def test_chunked_form_matches_recurrence(gate, T, C):
    """[HLA] section 5 chunk equations (with the chunk-start decay on Q and K,
    inclusive output mask, strict A mask) reproduce the token recurrence."""
    B, H, dk, dv = 1, 2, 8, 6
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, gate)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, s0, gate=gate)
    oc, sc = chunked.chunk_fwd(q, k, v, g, beta, s0, C=C)
    assert rel_err(oc, o) < 1e-11
    assert rel_err(sc, S_T) < 1e-11


def test_chunked_stage_identities():
    """Per-chunk identities of the UT transform: (I + A) T = Diag(beta), and
    T is lower triangular."""
    B, T, H, dk, dv = 1, 32, 1, 8, 8
    q, k, v, g, beta, s0 = _rand_inputs(B, T, H, dk, dv, "scalar")
    _, _, st = chunked.chunk_fwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0],
                                      beta[0, :, 0], s0[0, 0], C=16, keep_stages=True)
    for s in st:
        L = s["A"].shape[0]
        bt = np.diag(s["T"]).copy()
        assert np.allclose((np.eye(L) + s["A"]) @ s["T"], np.diag(bt), atol=1e-12)
        assert np.allclose(np.triu(s["T"], 1), 0.0)


# ----------------------------------------------------- hand-worked examples

def test_hand_worked_scalar_example():
    """Two tokens, d_k = d_v = 2, worked by hand from [HLA] section 3 item 3.

    S0 = I.  t=1: alpha=1/2, beta=1/2, k=(1,0), v=(2,0), q=(1,0):
      decay S = I/2; p = S k = (1/2,0); S += 1/2 (v-p) k^T -> [[5/4,0],[0,1/2]];
      o_1 = (5/4, 0).
    t=2: alpha=1, beta=1, k=(0,1), v=(1,1), q=(1,1):
      p = (0,1/2); S += (v-p) k^T -> [[5/4,1],[0,1]]; o_2 = (9/4, 1).
    log(1/2) is rounded to fp32, hence the 1e-7 tolerance.
    """
    q = np.array([[1, 0], [1, 1]], np.float32).reshape(1, 2, 1, 2)
    k = np.array([[1, 0], [0, 1]], np.float32).reshape(1, 2, 1, 2)
    v = np.array([[2, 0], [1, 1]], np.float32).reshape(1, 2, 1, 2)
    g = np.array([math.log(0.5), 0.0], np.float32).reshape(1, 2, 1)
    beta = np.array([0.5, 1.0], np.float32).reshape(1, 2, 1)
    S0 = np.eye(2).reshape(1, 1, 2, 2)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, S0)
    assert np.allclose(o[0, :, 0], [[1.25, 0.0], [2.25, 1.0]], atol=1e-7)
    assert np.allclose(S_T[0, 0], [[1.25, 1.0], [0.0, 1.0]], atol=1e-7)


def test_hand_worked_per_channel_example():
    """One token, per-channel gate alpha = (1/2, 1), beta = 1, k = (1/2, 1/2),
    v = (1, 0), q = (1, 0), S0 = I ([HLA] section 3 item 6, decay first):
      S' = Diag(alpha) = [[1/2,0],[0,1]]; p = S' k = (1/4, 1/2);
      S = S' + (v - p) k^T = [[7/8, 3/8], [-1/4, 3/4]]; o = (7/8, -1/4).
    (Erase-first would give o = (7/8, -1/8).)"""
    q = np.array([1, 0], np.float32).reshape(1, 1, 1, 2)
    k = np.array([0.5, 0.5], np.float32).reshape(1, 1, 1, 2)
    v = np.array([1, 0], np.float32).reshape(1, 1, 1, 2)
    g = np.array([math.log(0.5), 0.0], np.float32).reshape(1, 1, 1, 2)
    beta = np.ones((1, 1, 1), np.float32)
    S0 = np.eye(2).reshape(1, 1, 2, 2)
    o, S_T = oracle.gdr_fwd(q, k, v, g, beta, S0, gate="channel")
    assert np.allclose(o[0, 0, 0], [0.875, -0.25], atol=1e-7)
    assert np.allclose(S_T[0, 0], [[0.875, 0.375], [-0.25, 0.75]], atol=1e-7)


def test_oracle_rejects_bad_arguments():
    q, k, v, g, beta, s0 = _rand_inputs(1, 4, 1, 4, 4, "scalar")
    with pytest.raises(ValueError):
        oracle.gdr_fwd(q, k, v, g[..., None].repeat(3, -1), beta, s0)
    with pytest.raises(TypeError):
        oracle.gdr_fwd(q.astype(np.float64), k, v, g, beta, s0)


def test_bf16_widening_is_exact():
    """bf16 inputs are widened by a 16-bit shift, identical to NumPy's."""
    x = np.array([1.0, -2.5, 3.140625, 1e-3], np.float32)
    u = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(widen(u), (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64))


def test_oracle_regression_fixture():
    """The oracle still reproduces the fixture its own script wrote."""
    import json
    import os

    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny.json")
    with open(path) as f:
        fx = json.load(f)
    for c in fx["cases"]:
        arr = {k: np.array(c[k], np.float32) for k in ("q", "k", "v", "g", "beta", "S0")}
        o, S_T = oracle.gdr_fwd(arr["q"], arr["k"], arr["v"], arr["g"], arr["beta"],
                                arr["S0"].astype(np.float64), gate=c["gate"], nthreads=1)
        assert np.allclose(o, np.array(c["o"]), rtol=0, atol=1e-14)
        assert np.allclose(S_T, np.array(c["S_T"]), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- gated linear attention
# [HLA] section 3 item 4: S_t = S_{t-1} Diag(alpha_t) + v_t k_t^T, o_t = S_t q_t.

def _gla_closed_form(q, k, v, g, S0, gate):
    """Unrolled: S_t[i, j] = S0[i, j] e^{G_t[j]} + sum_{s<=t} v_s[i] k_s[j] e^{G_t[j] - G_s[j]}
    with G_t = sum of g up to t (per key channel), computed from cumulative
    sums, independently of the oracle's loop."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gg = g.astype(np.float64)
    if gate == "scalar":
        gg = np.repeat(gg[..., None], dk, axis=-1)
    G = np.cumsum(gg, axis=1)  # [B,T,H,dk]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            for t in range(T):
                S = np.zeros((dv, dk)) if S0 is None else S0[b, h] * np.exp(G[b, t, h])[None, :]
                for s_ in range(t + 1):
                    S = S + np.outer(v[b, s_, h], k[b, s_, h] * np.exp(G[b, t, h] - G[b, s_, h]))
                o[b, t, h] = S @ q[b, t, h]
                if t == T - 1:
                    ST[b, h] = S
    return o, ST


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_gla_oracle_matches_closed_form(gate):
    q, k, v, g, _, s0 = _rand_inputs(2, 9, 2, 5, 3, gate)
    o, ST = oracle.gla_fwd(q, k, v, g, s0, gate=gate)
    ro, rS = _gla_closed_form(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64),
                              g, s0, gate)
    assert rel_err(o, ro) < 1e-12 and rel_err(ST, rS) < 1e-12


def test_gla_without_decay_is_linear_attention():
    """alpha = 1, S0 = 0: o_t = sum_{s<=t} v_s (k_s . q_t)  (causal linear
    attention without normaliser, [LAV] linear attention recurrence)."""
    q, k, v, g, _, _ = _rand_inputs(1, 12, 2, 6, 4, "scalar", S0=False)
    g[:] = 0.0
    o, _ = oracle.gla_fwd(q, k, v, g, None)
    qd, kd, vd = (x.astype(np.float64) for x in (q, k, v))
    scores = np.einsum("bthd,bshd->bhts", qd, kd)
    scores = np.tril(scores)
    want = np.einsum("bhts,bshv->bthv", scores, vd)
    assert rel_err(o, want) < 1e-12


def test_gla_write_is_additive_not_erasing():
    """Writing the same (k, v) twice with alpha = 1 doubles the state (the
    delta rule would overwrite: its second write adds nothing)."""
    q, k, v, g, beta, _ = _rand_inputs(1, 2, 1, 4, 3, "scalar", S0=False)
    k[0, 1] = k[0, 0]
    v[0, 1] = v[0, 0]
    g[:] = 0.0
    _, ST = oracle.gla_fwd(q, k, v, g, None)
    one = np.outer(v[0, 0, 0].astype(np.float64), k[0, 0, 0].astype(np.float64))
    assert rel_err(ST[0, 0], 2 * one) < 1e-12
    beta[:] = 1.0
    _, SD = oracle.gdr_fwd(q, k, v, g, beta, None)
    # k is unit length up to its fp32 rounding, so the erase is exact to ~1e-7
    assert rel_err(SD[0, 0], one) < 1e-6


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_gla_split_and_resume(gate):
    q, k, v, g, _, s0 = _rand_inputs(1, 20, 2, 8, 5, gate)
    o, ST = oracle.gla_fwd(q, k, v, g, s0, gate=gate)
    oa, Sa = oracle.gla_fwd(q[:, :7], k[:, :7], v[:, :7], g[:, :7], s0, gate=gate)
    ob, Sb = oracle.gla_fwd(q[:, 7:], k[:, 7:], v[:, 7:], g[:, 7:], Sa, gate=gate)
    assert rel_err(np.concatenate([oa, ob], axis=1), o) < 1e-12 and rel_err(Sb, ST) < 1e-12


def test_oracle_siblings_regression_fixture():
    """GLA, DPLR, backward and prologue still reproduce the fixture their own
    script wrote (guards against silent change; not an independent pin)."""
    import json
    import os
    import sys

    here = os.path.join(os.path.dirname(__file__), "golden")
    sys.path.insert(0, here)
    try:
        import make_golden_siblings as mg
    finally:
        sys.path.remove(here)
    with open(os.path.join(here, "oracle_siblings_tiny.json")) as f:
        fx = json.load(f)
    x = {k: np.array(v, np.float32) for k, v in fx["inputs"].items()}
    got = mg.results(x)
    for name, want in fx["results"].items():
        assert np.allclose(np.asarray(got[name]), np.array(want), rtol=0, atol=1e-13), name
