"""The mixer's prologue in fp64: inputs from raw projections.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Maps what a layer's projections produce to what the recurrence consumes:

* ``l2_normalise``: q, k rows scaled to unit length, x / sqrt(sum x^2 + eps).
  The delta rule's erase ``I - beta k k^T`` is the projector the pages
  describe ("replacement along the k_t direction", "Decoding Hybrid Linear
  Attention Architectures", section 3 item 2; "Linear Attention Variants",
  DeltaNet section) only for a unit key; q is treated the same way.  eps =
  1e-6 keeps an all-zero row at zero.
* ``sigmoid``: beta = 1 / (1 + e^{-b}) maps a logit onto the write strength's
  range (0, 1) ("Decoding Hybrid Linear Attention Architectures", section 4:
  beta near 0 writes almost nothing, near 1 replaces completely).
* ``softplus`` and ``log_decay``: g = log alpha = -s_h softplus(a), a
  forgetting rate alpha in (0, 1] per token, accumulated in log space
  (section 4, and section 5 on log-space gates), with a per-head scale s_h
  > 0; alpha -> 1 as a -> -inf (the identity-like gate initialisation of
  section 7's checklist).
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def widen(x):
    """fp32 array, or uint16 holding bf16 bits -> float64 (exact)."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def l2_normalise(x, eps=EPS):
    """Rows of the last axis scaled to unit length (x / sqrt(|x|^2 + eps))."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def sigmoid(b):
    b = np.asarray(b, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-b))


def softplus(a):
    """log(1 + e^a), written so that neither branch overflows."""
    a = np.asarray(a, dtype=np.float64)
    return np.maximum(a, 0.0) + np.log1p(np.exp(-np.abs(a)))


def log_decay(a, gate_scale):
    """g = -s_h softplus(a); a [B,T,H] or [B,T,H,dk], gate_scale [H]."""
    a = np.asarray(a, dtype=np.float64)
    s = np.asarray(gate_scale, dtype=np.float64)
    shape = (1, 1, -1) + ((1,) if a.ndim == 4 else ())
    return -s.reshape(shape) * softplus(a)


def prologue(q_raw, k_raw, a, b, gate_scale, norm_q=True, norm_k=True):
    """(q, k, g, beta) in fp64 from raw q, k (fp32 or bf16 bits), the gate
    logits a and the write-strength logits b (fp32)."""
    q = widen(q_raw)
    k = widen(k_raw)
    if norm_q:
        q = l2_normalise(q)
    if norm_k:
        k = l2_normalise(k)
    return q, k, log_decay(a, gate_scale), sigmoid(b)
