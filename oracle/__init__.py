"""Oracle for the gated delta-rule mixer: plain fp64 CPU code.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg may import this package.  The CUDA library
never calls, links or loads anything in here, and nothing in here imports the
CUDA library.

Contents
--------
``gdr_fwd`` / ``gdr_step``
    ctypes front-end of ``gdr_oracle.c``: the token-by-token recurrence
    S_t = S_{t-1} Diag(alpha_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t, in double precision, threaded over (batch, head).
    ("Decoding Hybrid Linear Attention Architectures", section 3 items 3 and
    6 with the single-step pseudocode; "Linear Attention Variants", section
    "DeltaNet: Error-Correcting Writes".)
``gla_fwd``
    The gated-linear-attention recurrence S_t = S_{t-1} Diag(alpha_t) +
    v_t k_t^T, o_t = S_t q_t (additive write, no erase), from its own plain
    loop in ``gdr_oracle.c`` ("Decoding Hybrid Linear Attention
    Architectures", section 3 item 4; "Linear Attention Variants", GLA
    section).
``gdr_fwd_f64`` / ``gdr_fwd_prologue``
    The same recurrence on fp64 inputs, and on the output of ``prologue``
    (raw q, k L2-normalised, beta = sigmoid(b), g = -s_h softplus(a)).
``gdr_bwd``
    The backward of the recurrence (reverse mode over tokens, every state
    kept): gradients of q, k, v, g, beta and S0 from dL/do and dL/dS_T.
``dplr_fwd``
    The diagonal-plus-low-rank transition S_t = S_{t-1}(Diag(alpha_t) +
    a_t b_t^T) + v_t k_t^T, o_t = S_t q_t ("Decoding Hybrid Linear Attention
    Architectures", section 3 item 5).
``chunked``
    A staged fp64 NumPy restatement of the chunkwise algorithm ("Decoding
    Hybrid Linear Attention Architectures", section 5, inter-chunk recursion
    and intra-chunk output equations, with the WY/UT transform named in
    "Linear Attention Variants", DeltaNet section).  It is a debugging aid
    that exposes per-stage values; it is pinned against ``gdr_fwd``.

Pins (closed forms, brute force, invariants) live in ``tests/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdr_oracle.so")
_lib = None
_lock = threading.Lock()

F32, BF16 = 0, 1
GATE_SCALAR, GATE_PER_CHANNEL = 0, 1


def build(force: bool = False) -> str:
    """Compile ``gdr_oracle.c`` into ``libgdr_oracle.so`` with gcc (no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            vp, i = ctypes.c_void_p, ctypes.c_int
            lib.oracle_gdr_fwd.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp, i, i, i, i, i, i]
            lib.oracle_gdr_fwd.restype = i
            lib.oracle_gdr_step.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, i, i, i, i, i]
            lib.oracle_gdr_step.restype = i
            lib.oracle_gla_fwd.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, i, i, i, i, i, i]
            lib.oracle_gla_fwd.restype = i
            lib.oracle_gdr_fwd_f64.argtypes = [vp, vp, vp, vp, i, vp, vp, vp, vp, i, i, i, i, i,
                                               i]
            lib.oracle_gdr_fwd_f64.restype = i
            lib.oracle_gdr_bwd.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp, vp, vp, vp, vp,
                                           vp, vp, i, i, i, i, i, i]
            lib.oracle_gdr_bwd.restype = i
            lib.oracle_dplr_fwd.argtypes = [vp, vp, vp, vp, vp, i, vp, i, vp, vp, vp, i, i, i, i,
                                            i, i]
            lib.oracle_dplr_fwd.restype = i
            _lib = lib
    return _lib


def default_threads() -> int:
    """Threads the oracle uses by default: every core this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _as_input(x, name):
    """Accept fp32 arrays, or bf16 given as raw uint16 bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"{name}: expected float32 or uint16 (bf16 bits), got {x.dtype}")


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def gdr_fwd(q, k, v, g, beta, S0=None, gate="scalar", nthreads=None):
    """fp64 recurrence over a whole sequence.

    q, k: [B,T,H,dk]; v: [B,T,H,dv] (float32, or uint16 holding bf16 bits,
    all three the same); g = log(alpha): [B,T,H] (scalar gate) or [B,T,H,dk]
    (per-channel gate), float32; beta: [B,T,H] float32; S0: [B,H,dv,dk] or
    None for a zero state.  Returns (o [B,T,H,dv] float64, S_T [B,H,dv,dk]
    float64).
    """
    q, dt = _as_input(q, "q")
    k, dt2 = _as_input(k, "k")
    v, dt3 = _as_input(v, "v")
    if not (dt == dt2 == dt3):
        raise TypeError("q, k, v must share one dtype")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or v.shape != (B, T, H, dv):
        raise ValueError("shape mismatch among q, k, v")
    gk = GATE_PER_CHANNEL if gate in ("channel", "per_channel", GATE_PER_CHANNEL) else GATE_SCALAR
    g = np.ascontiguousarray(g, dtype=np.float32)
    want_g = (B, T, H, dk) if gk == GATE_PER_CHANNEL else (B, T, H)
    if g.shape != want_g:
        raise ValueError(f"g has shape {g.shape}, expected {want_g}")
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    if beta.shape != (B, T, H):
        raise ValueError("beta must be [B,T,H]")
    S0d = None
    if S0 is not None:
        S0d = np.ascontiguousarray(S0, dtype=np.float64)
        if S0d.shape != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    o = np.zeros((B, T, H, dv), np.float64)
    S_T = np.zeros((B, H, dv, dk), np.float64)
    n = nthreads or default_threads()
    rc = _load().oracle_gdr_fwd(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(g), gk, _ptr(beta),
                                _ptr(S0d), _ptr(o), _ptr(S_T), B, T, H, dk, dv, n)
    if rc != 0:
        raise ValueError("oracle_gdr_fwd rejected its arguments")
    return o, S_T


def gla_fwd(q, k, v, g, S0=None, gate="scalar", nthreads=None):
    """fp64 gated linear attention over a whole sequence (additive write).

    q, k: [B,T,H,dk]; v: [B,T,H,dv] (float32 or uint16 bf16 bits); g = log
    alpha: [B,T,H] or [B,T,H,dk] float32; S0: [B,H,dv,dk] or None.  Returns
    (o [B,T,H,dv] float64, S_T [B,H,dv,dk] float64).
    """
    q, dt = _as_input(q, "q")
    k, dt2 = _as_input(k, "k")
    v, dt3 = _as_input(v, "v")
    if not (dt == dt2 == dt3):
        raise TypeError("q, k, v must share one dtype")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or v.shape != (B, T, H, dv):
        raise ValueError("shape mismatch among q, k, v")
    gk = GATE_PER_CHANNEL if gate in ("channel", "per_channel", GATE_PER_CHANNEL) else GATE_SCALAR
    g = np.ascontiguousarray(g, dtype=np.float32)
    want_g = (B, T, H, dk) if gk == GATE_PER_CHANNEL else (B, T, H)
    if g.shape != want_g:
        raise ValueError(f"g has shape {g.shape}, expected {want_g}")
    S0d = None
    if S0 is not None:
        S0d = np.ascontiguousarray(S0, dtype=np.float64)
        if S0d.shape != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    o = np.zeros((B, T, H, dv), np.float64)
    S_T = np.zeros((B, H, dv, dk), np.float64)
    n = nthreads or default_threads()
    rc = _load().oracle_gla_fwd(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(g), gk, _ptr(S0d), _ptr(o),
                                _ptr(S_T), B, T, H, dk, dv, n)
    if rc != 0:
        raise ValueError("oracle_gla_fwd rejected its arguments")
    return o, S_T


def gdr_step(q, k, v, g, beta, S, gate="scalar", nthreads=None):
    """One recurrent step for N states; S [N,H,dv,dk] float64 updated in place.

    q, k: [N,H,dk]; v: [N,H,dv]; g: [N,H] or [N,H,dk]; beta: [N,H].
    Returns o [N,H,dv] float64.
    """
    q, dt = _as_input(q, "q")
    k, _ = _as_input(k, "k")
    v, _ = _as_input(v, "v")
    N, H, dk = q.shape
    dv = v.shape[-1]
    gk = GATE_PER_CHANNEL if gate in ("channel", "per_channel", GATE_PER_CHANNEL) else GATE_SCALAR
    g = np.ascontiguousarray(g, dtype=np.float32)
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    if not (isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous):
        raise TypeError("S must be a C-contiguous float64 array (updated in place)")
    if S.shape != (N, H, dv, dk):
        raise ValueError("S must be [N,H,dv,dk]")
    o = np.zeros((N, H, dv), np.float64)
    n = nthreads or default_threads()
    rc = _load().oracle_gdr_step(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(g), gk, _ptr(beta),
                                 _ptr(S), _ptr(o), N, H, dk, dv, n)
    if rc != 0:
        raise ValueError("oracle_gdr_step rejected its arguments")
    return o


def gdr_fwd_f64(q, k, v, g, beta, S0=None, gate="scalar", nthreads=None):
    """``gdr_fwd`` with every input in float64 (same shapes)."""
    q, k, v, g, beta = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or v.shape != (B, T, H, dv):
        raise ValueError("shape mismatch among q, k, v")
    gk = GATE_PER_CHANNEL if gate in ("channel", "per_channel", GATE_PER_CHANNEL) else GATE_SCALAR
    want_g = (B, T, H, dk) if gk == GATE_PER_CHANNEL else (B, T, H)
    if g.shape != want_g or beta.shape != (B, T, H):
        raise ValueError("g / beta shape mismatch")
    S0d = None
    if S0 is not None:
        S0d = np.ascontiguousarray(S0, dtype=np.float64)
        if S0d.shape != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    o = np.zeros((B, T, H, dv), np.float64)
    S_T = np.zeros((B, H, dv, dk), np.float64)
    n = nthreads or default_threads()
    rc = _load().oracle_gdr_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(g), gk, _ptr(beta),
                                    _ptr(S0d), _ptr(o), _ptr(S_T), B, T, H, dk, dv, n)
    if rc != 0:
        raise ValueError("oracle_gdr_fwd_f64 rejected its arguments")
    return o, S_T


def gdr_fwd_prologue(q_raw, k_raw, v, a, b, gate_scale, S0=None, gate="scalar", norm_q=True,
                     norm_k=True, nthreads=None):
    """The forward from raw projections: ``prologue.prologue`` then
    ``gdr_fwd_f64``.  q_raw, k_raw, v fp32 or uint16 (bf16 bits); a [B,T,H]
    or [B,T,H,dk] and b [B,T,H] fp32 logits; gate_scale [H] > 0."""
    from . import prologue as _pro

    q, k, g, beta = _pro.prologue(q_raw, k_raw, a, b, gate_scale, norm_q, norm_k)
    return gdr_fwd_f64(q, k, _pro.widen(v), g, beta, S0, gate=gate, nthreads=nthreads)


def gdr_bwd(q, k, v, g, beta, dout, S0=None, dS_T=None, gate="scalar", nthreads=None):
    """fp64 gradients of the forward ``gdr_fwd`` for upstream dout = dL/do
    [B,T,H,dv] and dS_T = dL/dS_T [B,H,dv,dk] (None: 0).  Inputs as
    ``gdr_fwd``.  Returns dict dq, dk [B,T,H,dk], dv [B,T,H,dv], dg (shape of
    g), dbeta [B,T,H], dS0 [B,H,dv,dk] (float64)."""
    q, dt = _as_input(q, "q")
    k, dt2 = _as_input(k, "k")
    v, dt3 = _as_input(v, "v")
    if not (dt == dt2 == dt3):
        raise TypeError("q, k, v must share one dtype")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gk = GATE_PER_CHANNEL if gate in ("channel", "per_channel", GATE_PER_CHANNEL) else GATE_SCALAR
    g = np.ascontiguousarray(g, dtype=np.float32)
    beta = np.ascontiguousarray(beta, dtype=np.float32)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    if dout.shape != (B, T, H, dv):
        raise ValueError("dout must be [B,T,H,dv]")
    S0d = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
    dST = None if dS_T is None else np.ascontiguousarray(dS_T, dtype=np.float64)
    out = dict(dq=np.zeros((B, T, H, dk)), dk=np.zeros((B, T, H, dk)), dv=np.zeros((B, T, H, dv)),
               dg=np.zeros(g.shape), dbeta=np.zeros((B, T, H)), dS0=np.zeros((B, H, dv, dk)))
    n = nthreads or default_threads()
    rc = _load().oracle_gdr_bwd(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(g), gk, _ptr(beta),
                                _ptr(S0d), _ptr(dout), _ptr(dST), _ptr(out["dq"]),
                                _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                                _ptr(out["dbeta"]), _ptr(out["dS0"]), B, T, H, dk, dv, n)
    if rc != 0:
        raise ValueError("oracle_gdr_bwd rejected its arguments")
    return out


def dplr_fwd(q, k, v, a, b, g, S0=None, gate="scalar", nthreads=None):
    """fp64 DPLR recurrence S_t = S_{t-1}(Diag(alpha_t) + a_t b_t^T) + v_t k_t^T,
    o_t = S_t q_t.  q, k, a, b [B,T,H,dk] and v [B,T,H,dv] (float32, or
    uint16 bf16 bits, one dtype); g = log alpha [B,T,H] or [B,T,H,dk];
    S0 [B,H,dv,dk] or None.  Returns (o, S_T) float64."""
    arrs = [_as_input(x, n) for x, n in ((q, "q"), (k, "k"), (v, "v"), (a, "a"), (b, "b"))]
    dts = {dt for _, dt in arrs}
    if len(dts) != 1:
        raise TypeError("q, k, v, a, b must share one dtype")
    (q, dt), (k, _), (v, _), (a, _), (b, _) = arrs
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for x, n in ((k, "k"), (a, "a"), (b, "b")):
        if x.shape != (B, T, H, dk):
            raise ValueError(f"{n} must be [B,T,H,dk]")
    gk = GATE_PER_CHANNEL if gate in ("channel", "per_channel", GATE_PER_CHANNEL) else GATE_SCALAR
    g = np.ascontiguousarray(g, dtype=np.float32)
    S0d = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
    o = np.zeros((B, T, H, dv), np.float64)
    S_T = np.zeros((B, H, dv, dk), np.float64)
    n = nthreads or default_threads()
    rc = _load().oracle_dplr_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), dt, _ptr(g), gk,
                                 _ptr(S0d), _ptr(o), _ptr(S_T), B, T, H, dk, dv, n)
    if rc != 0:
        raise ValueError("oracle_dplr_fwd rejected its arguments")
    return o, S_T
