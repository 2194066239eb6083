"""GPU parity of gdr_chunk_fwd_prologue (the chunked forward from raw
projections: q, k L2-normalised, beta = sigmoid(b), g = -s_h softplus(a)
inside the kernel) against the fp64 oracle's prologue + recurrence.

Acceptance as for gdr_chunk_fwd: max|gpu - oracle| / max|oracle| <= 2e-2
(bf16 inputs, fp32 state), on o and on S_T separately.
"""
import pytest
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import make_raw_chunk_inputs, to_numpy_input
from tests._gpu_util import assert_close, gpu_chunk, oracle_chunk

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _inputs(B, T, H, with_S0, seed):
    # distinct per-head scales, so that a head index mix-up shows
    return make_raw_chunk_inputs(B, T, H, 128, 128, torch.bfloat16, with_S0, seed,
                                 gate_scale=[0.05 + 0.1 * h for h in range(H)])


def _gpu(inp, dev, **kw):
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o, S_T = binding.chunk_fwd_prologue(d["q"], d["k"], d["v"], d["a"], d["b"], d["gate_scale"],
                                        d["S0"], **kw)
    torch.cuda.synchronize(dev)
    return o, S_T


def _oracle(inp, norm_q=True, norm_k=True):
    S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
    gate = "channel" if inp["a"].dim() == 4 else "scalar"
    return oracle.gdr_fwd_prologue(to_numpy_input(inp["q"]), to_numpy_input(inp["k"]),
                                   to_numpy_input(inp["v"]), inp["a"].numpy(), inp["b"].numpy(),
                                   inp["gate_scale"].numpy(), S0, gate=gate, norm_q=norm_q,
                                   norm_k=norm_k)


# several chunks + a ragged tail; one exact chunk; a single token
@pytest.mark.parametrize("T", [300, 64, 1])
@pytest.mark.parametrize("with_S0", [True, False])
def test_prologue_matches_oracle(cuda_device, T, with_S0):
    inp = _inputs(2, T, 3, with_S0, seed=90 + T)
    o, S_T = _gpu(inp, cuda_device)
    assert binding.device_status() == 0
    ro, rS = _oracle(inp)
    assert_close(o, ro, TOL, "o")
    assert_close(S_T, rS, TOL, "S_T")


@pytest.mark.parametrize("norm_q,norm_k", [(False, True), (True, False), (False, False)])
def test_prologue_normalisation_flags(cuda_device, norm_q, norm_k):
    """Each flag normalises its own tensor only (raw rows are scaled down so
    that the unnormalised runs stay in a sane range)."""
    inp = _inputs(1, 200, 2, True, seed=95)
    inp["q"] = (inp["q"].float() * 0.09).to(torch.bfloat16)
    inp["k"] = (inp["k"].float() * 0.09).to(torch.bfloat16)
    o, S_T = _gpu(inp, cuda_device, norm_q=norm_q, norm_k=norm_k)
    assert binding.device_status() == 0
    ro, rS = _oracle(inp, norm_q, norm_k)
    assert_close(o, ro, TOL, "o")
    assert_close(S_T, rS, TOL, "S_T")


def test_prologue_equals_separate_maps(cuda_device):
    """The fused call against gdr_chunk_fwd on inputs mapped beforehand by
    torch (normalise, sigmoid, -s softplus): the same result up to the
    rounding of the normalised q, k to bf16 (computed in another order)."""
    inp = _inputs(2, 256, 2, False, seed=96)
    o, S_T = _gpu(inp, cuda_device)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    nrm = lambda x: (x.float() * torch.rsqrt((x.float() ** 2).sum(-1, keepdim=True) + 1e-6))
    q = nrm(d["q"]).to(torch.bfloat16)
    k = nrm(d["k"]).to(torch.bfloat16)
    beta = torch.sigmoid(d["b"])
    g = -d["gate_scale"].view(1, 1, -1) * torch.nn.functional.softplus(d["a"])
    o2, S2 = binding.chunk_fwd(q, k, d["v"], g.contiguous(), beta.contiguous(), None)
    torch.cuda.synchronize()
    e_o = (o.float() - o2.float()).abs().max() / o2.float().abs().max()
    e_S = (S_T - S2).abs().max() / S2.abs().max()
    assert e_o < 1e-2 and e_S < 1e-2


def test_prologue_zero_query_row_gives_zero_output(cuda_device):
    """A query that is exactly zero stays zero through the normalisation
    (|q|^2 + eps > 0), so that token's output is exactly zero."""
    inp = _inputs(1, 130, 2, True, seed=97)
    inp["q"][:, 70] = 0
    o, _ = _gpu(inp, cuda_device)
    assert torch.count_nonzero(o[:, 70]).item() == 0
    assert torch.count_nonzero(o[:, 69]).item() > 0


def test_prologue_skipped_load_times_out_and_reports(cuda_device):
    """The prologue's own landing wait is bounded: a chunk whose load never
    goes out ends the call with a time-out status, and the context works."""
    inp = _inputs(1, 256, 2, False, seed=98)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    assert binding.device_status() == binding.GDR_OK
    binding.testing_skip_stage_load(1)
    binding.chunk_fwd_prologue(d["q"], d["k"], d["v"], d["a"], d["b"], d["gate_scale"], None)
    assert binding.device_status() == binding.GDR_ERR_TIMEOUT
    o, S_T = _gpu(inp, cuda_device)
    ro, rS = _oracle(inp)
    assert_close(o, ro, TOL, "o after recovery")
    assert binding.device_status() == binding.GDR_OK


# the split-operand kernel: fp32 inputs (bar 1e-4), other head dims, and
# per-channel gate logits (any dtype); several chunks and a ragged tail
@pytest.mark.parametrize("dk,dv,dtype,gate", [(128, 128, torch.bfloat16, "channel"),
                                              (64, 64, torch.float32, "scalar"),
                                              (32, 64, torch.float32, "channel"),
                                              (128, 32, torch.bfloat16, "scalar")])
def test_prologue_split_operand_shapes(cuda_device, dk, dv, dtype, gate):
    inp = make_raw_chunk_inputs(2, 150, 3, dk, dv, dtype, True, seed=98 + dk + dv,
                                gate_scale=[0.05 + 0.1 * h for h in range(3)], gate=gate)
    o, S_T = _gpu(inp, cuda_device)
    assert binding.device_status() == 0
    ro, rS = _oracle(inp)
    tol = 1e-4 if dtype == torch.float32 else TOL
    assert_close(o, ro, tol, "o")
    assert_close(S_T, rS, tol, "S_T")


def test_prologue_split_operand_flags(cuda_device):
    """norm_q only, fp32 d = 64: the flags on the split-operand kernel."""
    inp = make_raw_chunk_inputs(1, 100, 2, 64, 64, torch.float32, True, seed=99)
    inp["k"] = inp["k"] * 0.12
    o, S_T = _gpu(inp, cuda_device, norm_q=True, norm_k=False)
    ro, rS = _oracle(inp, norm_q=True, norm_k=False)
    assert_close(o, ro, 1e-4, "o")
    assert_close(S_T, rS, 1e-4, "S_T")
