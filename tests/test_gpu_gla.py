"""GPU parity of gdr_chunk_fwd_gla (gated linear attention, the additive
sibling of the delta rule) against the fp64 oracle's recurrence.

Acceptance as for gdr_chunk_fwd: max|gpu - oracle| / max|oracle| <= 2e-2
(bf16 inputs, fp32 state), on o and on S_T separately.
"""
import pytest
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import make_chunk_inputs, to_numpy_input
from tests._gpu_util import assert_close

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _gpu(inp, dev, **kw):
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o, S_T = binding.chunk_fwd_gla(d["q"], d["k"], d["v"], d["g"], d["S0"], **kw)
    torch.cuda.synchronize(dev)
    return o, S_T


def _oracle(inp):
    gate = "channel" if inp["g"].dim() == 4 else "scalar"
    S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
    return oracle.gla_fwd(to_numpy_input(inp["q"]), to_numpy_input(inp["k"]),
                          to_numpy_input(inp["v"]), inp["g"].numpy(), S0, gate=gate)


# 4 full chunks + a ragged tail; one exact chunk; a single token
@pytest.mark.parametrize("T", [300, 64, 1])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("with_S0", [True, False])
def test_gla_matches_oracle(cuda_device, T, gate, with_S0):
    inp = make_chunk_inputs(2, T, 3, 128, 128, torch.bfloat16, gate, with_S0, seed=70 + T)
    o, S_T = _gpu(inp, cuda_device)
    assert binding.device_status() == 0
    ro, rS = _oracle(inp)
    assert_close(o, ro, TOL, "o")
    assert_close(S_T, rS, TOL, "S_T")


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_gla_strong_decay(cuda_device, gate):
    """Chunk decays beyond e^{-80} (the unfactored P form) and state scales
    below 2^-40 (the fold of the scale into the state)."""
    inp = make_chunk_inputs(1, 512, 2, 128, 128, torch.bfloat16, gate, True, seed=77)
    inp["g"] = inp["g"] * 20.0
    o, S_T = _gpu(inp, cuda_device)
    assert binding.device_status() == 0
    ro, rS = _oracle(inp)
    assert_close(o, ro, TOL, "o")
    assert_close(S_T, rS, TOL, "S_T")


def test_gla_no_decay_is_causal_linear_attention(cuda_device):
    """g = 0, S0 = 0: o_t = sum_{s<=t} v_s (k_s . q_t), also computed with torch
    matmuls on the same device in fp32."""
    inp = make_chunk_inputs(1, 200, 2, 128, 128, torch.bfloat16, "scalar", False, seed=78)
    inp["g"] = torch.zeros_like(inp["g"])
    o, _ = _gpu(inp, cuda_device)
    q, k, v = (inp[x].to(cuda_device).float() for x in ("q", "k", "v"))
    sc = torch.einsum("bthd,bshd->bhts", q, k).tril()
    want = torch.einsum("bhts,bshv->bthv", sc, v)
    ro, _ = _oracle(inp)
    assert_close(o, ro, TOL, "o vs oracle")
    assert_close(o, want.double().cpu().numpy(), TOL, "o vs causal linear attention")


def test_gla_state_in_place_and_split(cuda_device):
    """S_T may alias S0; running [0, 192) then [192, 300) from the first
    call's state gives the one-call output and final state."""
    inp = make_chunk_inputs(2, 300, 2, 128, 128, torch.bfloat16, "channel", True, seed=79)
    o, S_T = _gpu(inp, cuda_device)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    S = d["S0"].clone()
    sl = lambda t, a, b: t[:, a:b].contiguous()
    oa, _ = binding.chunk_fwd_gla(*(sl(d[x], 0, 192) for x in ("q", "k", "v", "g")), S, S_T=S)
    ob, _ = binding.chunk_fwd_gla(*(sl(d[x], 192, 300) for x in ("q", "k", "v", "g")), S, S_T=S)
    torch.cuda.synchronize()
    ro, rS = _oracle(inp)
    assert_close(torch.cat([oa, ob], dim=1), ro, TOL, "o of the split run")
    assert_close(S, rS, TOL, "S_T of the split run")
    assert_close(S_T, rS, TOL, "S_T")


def test_gla_empty_sequence_copies_state(cuda_device):
    inp = make_chunk_inputs(2, 0, 2, 128, 128, torch.bfloat16, "scalar", True, seed=80)
    _, S_T = _gpu(inp, cuda_device)
    assert torch.equal(S_T.cpu(), inp["S0"])
    inp["S0"] = None
    _, S_T = _gpu(inp, cuda_device)
    assert torch.count_nonzero(S_T).item() == 0


# the split-operand kernel: fp32 inputs (bar 1e-4) and other head dims
@pytest.mark.parametrize("dk,dv,dtype,gate", [(64, 64, torch.float32, "scalar"),
                                              (32, 128, torch.float32, "channel"),
                                              (128, 64, torch.bfloat16, "channel")])
def test_gla_split_operand_shapes(cuda_device, dk, dv, dtype, gate):
    inp = make_chunk_inputs(2, 150, 3, dk, dv, dtype, gate, True, seed=75 + dk + dv)
    o, S_T = _gpu(inp, cuda_device)
    assert binding.device_status() == 0
    ro, rS = _oracle(inp)
    tol = 1e-4 if dtype == torch.float32 else TOL
    assert_close(o, ro, tol, "o")
    assert_close(S_T, rS, tol, "S_T")
