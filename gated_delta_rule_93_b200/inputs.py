"""Seeded synthetic inputs for the gated delta-rule mixer.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic, so both the CUDA path and the fp64 oracle consume the
exact same values from here.

Recipe (every workload, one CPU ``torch.Generator`` per call):
  * q, k ~ N(0, 1) in fp32, L2-normalised over d_k for each (b, t, h), then
    cast to the input dtype;
  * v ~ N(0, 1), cast to the input dtype;
  * g = log(alpha) = -0.1 * softplus(N(0, 1)), fp32, shape [B,T,H] for a
    scalar per-head gate or [B,T,H,d_k] for a per-channel gate;
  * beta = sigmoid(N(0, 1)), fp32;
  * S0 = N(0, 0.02^2) fp32 [B,H,d_v,d_k] where the workload has one, else None.
Draw order: q, k, v, g, beta, S0.  The decode workload draws its initial
state first, then the q, k, v, g, beta stacks of all steps (step-major).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    """A named shape + dtype recipe."""

    name: str
    kind: str  # "chunk" (gdr_chunk_fwd) or "step" (gdr_step)
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    gate: str  # "scalar" or "channel"
    with_S0: bool
    want_S_T: bool
    steps: int = 1  # decode workloads: consecutive steps
    C: int = 64
    mixer: str = "gdr"  # "gdr" (delta rule), "gla" (gated linear attention, beta unused)
    #                     or "dplr" (diagonal-plus-low-rank transition)
    prologue: bool = False  # raw projections in: q, k unnormalised, gate / beta logits
    backward: bool = False  # gradients (gdr_chunk_bwd) for a seeded dL/do
    note: str = field(default="", compare=False)

    @property
    def tokens(self) -> int:
        return self.B * self.T if self.kind == "chunk" else self.B * self.steps


# The workloads, named by what they are.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32", "chunk", 1, 256, 2, 32, 32, torch.float32, "scalar", False, True,
                 note="tiny Gated DeltaNet forward, fp32"),
        Workload("gdn_b8_t4096_h16_d128", "chunk", 8, 4096, 16, 128, 128, torch.bfloat16, "scalar",
                 False, True, note="Gated DeltaNet layer forward at 350M-model shape"),
        Workload("gdn_b1_t65536_h16_d128", "chunk", 1, 65536, 16, 128, 128, torch.bfloat16,
                 "scalar", True, True, note="long-sequence Gated DeltaNet forward"),
        Workload("kda_b8_t4096_h16_d128", "chunk", 8, 4096, 16, 128, 128, torch.bfloat16,
                 "channel", False, True, note="per-channel (Kimi-Delta-style) gate forward"),
        Workload("decode_n256_h16_d128_x1024", "step", 256, 1, 16, 128, 128, torch.bfloat16,
                 "scalar", True, True, steps=1024,
                 note="recurrent decode step, 256 sequences, 1024 consecutive steps"),
        Workload("gla_b8_t4096_h16_d128", "chunk", 8, 4096, 16, 128, 128, torch.bfloat16,
                 "scalar", False, True, mixer="gla",
                 note="gated linear attention forward at the same shape (additive writes)"),
        Workload("dplr_b8_t4096_h16_d128", "chunk", 8, 4096, 16, 128, 128, torch.bfloat16,
                 "scalar", False, True, mixer="dplr",
                 note="diagonal-plus-low-rank transition forward at the same shape"),
        Workload("gdn_bwd_b8_t4096_h16_d128", "chunk", 8, 4096, 16, 128, 128, torch.bfloat16,
                 "scalar", False, False, backward=True,
                 note="Gated DeltaNet backward at the 350M shape (dL/do ~ N(0, 1) fp32)"),
        Workload("gdn_prologue_b8_t4096_h16_d128", "chunk", 8, 4096, 16, 128, 128,
                 torch.bfloat16, "scalar", False, True, prologue=True,
                 note="Gated DeltaNet forward at the 350M shape from raw projections "
                      "(normalisation and gate maps inside the kernel)"),
    ]
}


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_chunk_inputs(B, T, H, dk, dv, dtype=torch.bfloat16, gate="scalar", with_S0=False,
                      seed=0):
    """Inputs for ``gdr_chunk_fwd`` on the CPU: dict of q,k,v,g,beta,S0 (S0 may be None)."""
    gen = torch.Generator().manual_seed(seed)
    q = _unit_rows(torch.randn(B, T, H, dk, generator=gen)).to(dtype)
    k = _unit_rows(torch.randn(B, T, H, dk, generator=gen)).to(dtype)
    v = torch.randn(B, T, H, dv, generator=gen).to(dtype)
    gshape = (B, T, H, dk) if gate == "channel" else (B, T, H)
    g = -0.1 * F.softplus(torch.randn(*gshape, generator=gen))
    beta = torch.sigmoid(torch.randn(B, T, H, generator=gen))
    S0 = 0.02 * torch.randn(B, H, dv, dk, generator=gen) if with_S0 else None
    return dict(q=q, k=k, v=v, g=g.float(), beta=beta.float(), S0=S0)


def make_dplr_inputs(B, T, H, d, dtype=torch.bfloat16, gate="scalar", with_S0=False, seed=0,
                     independent=False):
    """Inputs for ``gdr_dplr_fwd``: the ``make_chunk_inputs`` draws (q, k, v, g,
    beta, S0) plus an erase direction b (unit rows of N(0, 1), its own
    stream), and a = -beta e^{g} b (per channel, or the head's scalar gate),
    so that each transition Diag(alpha)(I - beta b b^T) is a contraction and
    long sequences stay bounded.  independent=True draws a on its own instead
    (unit rows of N(0, 1) times 0.5, a third stream): a general low-rank
    term, not tied to b (its transitions need not contract, so keep T short).
    Returns dict q, k, v, a, b, g, S0."""
    d_ = make_chunk_inputs(B, T, H, d, d, dtype, gate, with_S0, seed)
    gen = torch.Generator().manual_seed(seed + 15485863)
    b = _unit_rows(torch.randn(B, T, H, d, generator=gen))
    if independent:
        gen_a = torch.Generator().manual_seed(seed + 32452843)
        a = 0.5 * _unit_rows(torch.randn(B, T, H, d, generator=gen_a))
    else:
        al = torch.exp(d_["g"] if gate == "channel" else d_["g"][..., None])
        a = -d_["beta"][..., None] * al * b
    return dict(q=d_["q"], k=d_["k"], v=d_["v"], a=a.to(dtype), b=b.to(dtype), g=d_["g"],
                S0=d_["S0"])


def make_raw_chunk_inputs(B, T, H, dk, dv, dtype=torch.bfloat16, with_S0=False, seed=0,
                          gate_scale=None, gate="scalar"):
    """Raw-projection inputs for ``gdr_chunk_fwd_prologue``.

    Returns dict of q, k [B,T,H,dk] ~ N(0,1) not normalised, v [B,T,H,dv], a
    (gate logits) and b (beta logits) [B,T,H] ~ N(0,1) fp32, gate_scale [H]
    fp32 (default 0.1 for every head) and S0 (or None).  Same draws, in the
    same order, as ``make_chunk_inputs`` with the same seed, before its
    normalisation and gate maps: with gate_scale 0.1 the prologue yields that
    workload's distribution.  gate="channel": a is [B,T,H,dk] ~ N(0,1), drawn
    from a stream of its own (the other draws unchanged).
    """
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, H, dk, generator=gen).to(dtype)
    k = torch.randn(B, T, H, dk, generator=gen).to(dtype)
    v = torch.randn(B, T, H, dv, generator=gen).to(dtype)
    a = torch.randn(B, T, H, generator=gen)
    b = torch.randn(B, T, H, generator=gen)
    S0 = 0.02 * torch.randn(B, H, dv, dk, generator=gen) if with_S0 else None
    gs = torch.full((H,), 0.1) if gate_scale is None else torch.as_tensor(gate_scale).float()
    if gate == "channel":
        a = torch.randn(B, T, H, dk, generator=torch.Generator().manual_seed(seed + 49979687))
    return dict(q=q, k=k, v=v, a=a.float(), b=b.float(), gate_scale=gs.float().contiguous(),
                S0=S0)


def make_varlen_inputs(lens, H, dk, dv, dtype=torch.bfloat16, gate="scalar", with_S0=True,
                       seed=0):
    """Packed inputs for ``gdr_chunk_fwd_varlen``: len(lens) sequences back to back.

    Returns dict of q, k [total,H,dk], v [total,H,dv], g [total,H] (or
    [total,H,dk]), beta [total,H], S0 [N,H,dv,dk] fp32 (or None) and
    cu_seqlens int32 [N+1] (all on the CPU).  Token draws as
    ``make_chunk_inputs(1, total, ...)``; S0 from its own stream.
    """
    total = int(sum(lens))
    d = make_chunk_inputs(1, total, H, dk, dv, dtype, gate, False, seed=seed)
    out = {key: d[key][0] for key in ("q", "k", "v", "g", "beta")}
    gen = torch.Generator().manual_seed(seed + 7919)
    out["S0"] = 0.02 * torch.randn(len(lens), H, dv, dk, generator=gen) if with_S0 else None
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32)
    return out


def make_step_inputs(N, H, dk, dv, steps, dtype=torch.bfloat16, gate="scalar", seed=0):
    """Inputs for ``steps`` consecutive ``gdr_step`` calls.

    Returns dict with S0 [N,H,dv,dk] fp32 and per-step stacks q,k [steps,N,H,dk],
    v [steps,N,H,dv], g [steps,N,H] (or [steps,N,H,dk]), beta [steps,N,H].
    Draw order: S0, then the q, k, v, g, beta stacks (step-major).
    """
    gen = torch.Generator().manual_seed(seed)
    S0 = 0.02 * torch.randn(N, H, dv, dk, generator=gen)
    q = _unit_rows(torch.randn(steps, N, H, dk, generator=gen)).to(dtype)
    k = _unit_rows(torch.randn(steps, N, H, dk, generator=gen)).to(dtype)
    v = torch.randn(steps, N, H, dv, generator=gen).to(dtype)
    gshape = (steps, N, H, dk) if gate == "channel" else (steps, N, H)
    g = -0.1 * F.softplus(torch.randn(*gshape, generator=gen))
    beta = torch.sigmoid(torch.randn(steps, N, H, generator=gen))
    return dict(S0=S0.float(), q=q, k=k, v=v, g=g.float(), beta=beta.float())


def make_workload_inputs(w: Workload, seed=0, steps=None):
    if w.kind == "chunk" and w.prologue:
        return make_raw_chunk_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.with_S0, seed)
    if w.kind == "chunk" and w.mixer == "dplr":
        return make_dplr_inputs(w.B, w.T, w.H, w.dk, w.dtype, w.gate, w.with_S0, seed)
    if w.kind == "chunk" and w.backward:
        d = make_chunk_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.gate, w.with_S0, seed)
        gen = torch.Generator().manual_seed(seed + 104729)
        d["dout"] = torch.randn(w.B, w.T, w.H, w.dv, generator=gen)
        return d
    if w.kind == "chunk":
        return make_chunk_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.gate, w.with_S0, seed)
    return make_step_inputs(w.B, w.H, w.dk, w.dv, steps or w.steps, w.dtype, w.gate, seed)


def to_numpy_input(t: torch.Tensor):
    """CPU tensor -> numpy array the oracle accepts (float32, or uint16 bf16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.float().numpy()
