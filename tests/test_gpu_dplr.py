"""GPU parity of gdr_dplr_fwd (the diagonal-plus-low-rank transition, chunked
on the tensor cores with split bf16 operands) against the fp64 oracle.  The
state is fp32 and every product is carried to near fp32 accuracy on the same
inputs; o is rounded to the input dtype.  Bars: o within 2e-2 for bf16
inputs (its rounding) and 1e-4 for fp32; S_T within 1e-4."""
import pytest
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import make_dplr_inputs, to_numpy_input
from tests._gpu_util import assert_close

pytestmark = pytest.mark.gpu


def _run(inp, dev):
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o, S_T = binding.dplr_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["g"], d["S0"])
    torch.cuda.synchronize(dev)
    return o, S_T


def _oracle(inp):
    gate = "channel" if inp["g"].dim() == 4 else "scalar"
    S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
    return oracle.dplr_fwd(*(to_numpy_input(inp[x]) for x in ("q", "k", "v", "a", "b")),
                           inp["g"].numpy(), S0, gate=gate)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("with_S0", [True, False])
def test_dplr_matches_oracle_d128_bf16(cuda_device, gate, with_S0):
    inp = make_dplr_inputs(2, 150, 2, 128, torch.bfloat16, gate, with_S0, seed=140)
    o, S_T = _run(inp, cuda_device)
    ro, rS = _oracle(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 1e-4, "S_T")


@pytest.mark.parametrize("d", [32, 64])
def test_dplr_matches_oracle_fp32(cuda_device, d):
    inp = make_dplr_inputs(2, 70, 3, d, torch.float32, "channel", True, seed=141 + d)
    o, S_T = _run(inp, cuda_device)
    ro, rS = _oracle(inp)
    assert_close(o, ro, 1e-4, "o")
    assert_close(S_T, rS, 1e-4, "S_T")


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("d,dtype,tol_o", [(128, torch.bfloat16, 2e-2), (64, torch.float32, 1e-4)])
def test_dplr_independent_low_rank_matches_oracle(cuda_device, gate, d, dtype, tol_o):
    """a and b drawn independently (a general low-rank read, not the delta
    rule's contraction a = -beta alpha b): 100 tokens, with S0."""
    inp = make_dplr_inputs(2, 100, 2, d, dtype, gate, True, seed=150 + d, independent=True)
    o, S_T = _run(inp, cuda_device)
    ro, rS = _oracle(inp)
    assert_close(o, ro, tol_o, "o")
    assert_close(S_T, rS, 1e-4, "S_T")


def test_dplr_with_delta_parameters_equals_chunked_delta_rule(cuda_device):
    """a = -beta (alpha . k), b = k, v -> beta v gives the gated delta rule:
    the recurrent DPLR kernel against the tensor-core chunked forward."""
    from gated_delta_rule_93_b200.inputs import make_chunk_inputs
    inp = make_chunk_inputs(2, 200, 2, 128, 128, torch.bfloat16, "scalar", True, seed=143)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    al = torch.exp(d["g"])[..., None]
    a = (-d["beta"][..., None] * al * d["k"].float()).to(torch.bfloat16)
    vb = (d["beta"][..., None] * d["v"].float()).to(torch.bfloat16)
    o, S_T = binding.dplr_fwd(d["q"], d["k"], vb, a, d["k"], d["g"], d["S0"])
    oc, Sc = binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    torch.cuda.synchronize()
    e_o = (o.float() - oc.float()).abs().max() / oc.float().abs().max()
    e_S = (S_T - Sc).abs().max() / Sc.abs().max()
    assert e_o < 2e-2 and e_S < 2e-2


def test_dplr_empty_sequence(cuda_device):
    inp = make_dplr_inputs(1, 0, 2, 64, torch.float32, "scalar", True, seed=144)
    _, S_T = _run(inp, cuda_device)
    assert torch.equal(S_T.cpu(), inp["S0"])


@pytest.mark.parametrize("dk,dv,dtype", [(64, 128, torch.float32), (128, 32, torch.bfloat16),
                                         (32, 64, torch.float32)])
def test_dplr_unequal_head_dims(cuda_device, dk, dv, dtype):
    """d_k != d_v: q, k, a, b [.., dk], v and o [.., dv], state [dv, dk];
    a ragged tail (130 = 2 x 64 + 2), per-channel gate, S0 given."""
    inp = make_dplr_inputs(2, 130, 2, dk, dtype, "channel", True, seed=160 + dk + dv)
    gen = torch.Generator().manual_seed(161 + dv)
    v = torch.randn(2, 130, 2, dv, generator=gen).to(dtype)
    S0 = 0.02 * torch.randn(2, 2, dv, dk, generator=gen)
    inp = dict(inp, v=v, S0=S0)
    o, S_T = _run(inp, cuda_device)
    ro, rS = _oracle(inp)
    assert_close(o, ro, 2e-2 if dtype == torch.bfloat16 else 1e-4, "o")
    assert_close(S_T, rS, 1e-4, "S_T")


def _one_channel_decay(inp, g_channel, channel=5, head=0):
    g = inp["g"].clone()
    g[:, :, head, channel] = g_channel
    return dict(inp, g=g.contiguous())


def test_dplr_per_channel_strong_decay_in_range(cuda_device):
    """One key channel at g = -2 per token (-62 over half a chunk, inside the
    split-operand range): oracle parity at the fp32 bar, clean status."""
    inp = _one_channel_decay(make_dplr_inputs(1, 200, 2, 64, torch.float32, "channel", True,
                                              seed=170), -2.0)
    o, S_T = _run(inp, cuda_device)
    assert binding.device_status() == binding.GDR_OK
    ro, rS = _oracle(inp)
    assert_close(o, ro, 1e-4, "o")
    assert_close(S_T, rS, 1e-4, "S_T")


def test_dplr_per_channel_rapid_forgetting_reports_range(cuda_device):
    """g = -30 per token in one channel is outside the factor range: the call
    records GDR_ERR_RANGE and its outputs stay finite."""
    inp = _one_channel_decay(make_dplr_inputs(1, 200, 2, 64, torch.float32, "channel", True,
                                              seed=171), -30.0)
    o, S_T = _run(inp, cuda_device)
    assert binding.device_status() == binding.GDR_ERR_RANGE
    assert torch.isfinite(o).all() and torch.isfinite(S_T).all()


def test_dplr_full_size_workload(cuda_device):
    """The DPLR workload (B8 T4096 H16 d128, bf16, scalar gate), whole
    tensors against the full oracle."""
    from gated_delta_rule_93_b200.inputs import WORKLOADS, make_workload_inputs
    inp = make_workload_inputs(WORKLOADS["dplr_b8_t4096_h16_d128"])
    o, S_T = _run(inp, cuda_device)
    assert binding.device_status() == binding.GDR_OK
    ro, rS = _oracle(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 1e-4, "S_T")
