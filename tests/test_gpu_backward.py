"""GPU parity of gdr_chunk_bwd (gradients of the recurrence) against the fp64
oracle's backward, which is pinned to finite differences of the forward.

Two paths.  bf16 inputs with d_k = d_v = 128 and a scalar gate run the
chunked backward on the tensor cores (bf16 operands, fp32 accumulation and
state gradient): the bar is the bf16 one, max|gpu - oracle| / max|oracle| <=
2e-2 on every gradient.  Every other shape runs the per-step recurrence in
fp32 on CUDA cores on the very same inputs: the bar is 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import make_chunk_inputs, to_numpy_input
from tests._gpu_util import assert_close

pytestmark = pytest.mark.gpu

def _tol(inp):
    tc = (inp["q"].dtype == torch.bfloat16 and inp["q"].shape[-1] == 128 and
          inp["g"].dim() == 3 and inp["q"].shape[1] > 0)
    return 2e-2 if tc else 1e-4


def _case(B, T, H, d, dtype, gate, with_S0, with_dST, seed):
    inp = make_chunk_inputs(B, T, H, d, d, dtype, gate, with_S0, seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(B, T, H, d, generator=gen)
    dST = torch.randn(B, H, d, d, generator=gen) if with_dST else None
    return inp, dout, dST


def _run(inp, dout, dST, dev):
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    out = binding.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout.to(dev), d["S0"],
                            dST.to(dev) if dST is not None else None)
    torch.cuda.synchronize(dev)
    return out


def _oracle(inp, dout, dST):
    gate = "channel" if inp["g"].dim() == 4 else "scalar"
    S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
    return oracle.gdr_bwd(to_numpy_input(inp["q"]), to_numpy_input(inp["k"]),
                          to_numpy_input(inp["v"]), inp["g"].numpy(), inp["beta"].numpy(),
                          dout.double().numpy(), S0,
                          None if dST is None else dST.double().numpy(), gate=gate)


def _check(out, ref, tol):
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert_close(out[name], ref[name], tol, name)


# d = 128 bf16 (the tensor-core forward's shape): two full 64-token chunks and a ragged tail
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("with_S0,with_dST", [(True, True), (False, False), (False, True)])
def test_backward_matches_oracle_d128(cuda_device, gate, with_S0, with_dST):
    inp, dout, dST = _case(2, 150, 2, 128, torch.bfloat16, gate, with_S0, with_dST, seed=120)
    _check(_run(inp, dout, dST, cuda_device), _oracle(inp, dout, dST), _tol(inp))
    assert binding.device_status() == 0


@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_backward_matches_oracle_small_heads_fp32(cuda_device, d, gate):
    inp, dout, dST = _case(2, 130, 3, d, torch.float32, gate, True, True, seed=121 + d)
    _check(_run(inp, dout, dST, cuda_device), _oracle(inp, dout, dST), _tol(inp))


@pytest.mark.parametrize("T", [1, 64])
def test_backward_short_sequences(cuda_device, T):
    inp, dout, dST = _case(1, T, 2, 128, torch.bfloat16, "scalar", True, True, seed=125 + T)
    _check(_run(inp, dout, dST, cuda_device), _oracle(inp, dout, dST), _tol(inp))


def test_backward_empty_sequence_passes_dST_through(cuda_device):
    inp, dout, dST = _case(2, 0, 2, 64, torch.float32, "scalar", True, True, seed=127)
    out = _run(inp, dout, dST, cuda_device)
    assert torch.equal(out["dS0"].cpu(), dST)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_backward_of_zero_upstream_is_zero(cuda_device, gate):
    inp, dout, _ = _case(1, 100, 2, 128, torch.bfloat16, gate, True, False, seed=128)
    out = _run(inp, torch.zeros_like(dout), None, cuda_device)
    for name, t in out.items():
        assert torch.count_nonzero(t).item() == 0, name


@pytest.mark.parametrize("B,T,H", [(1, 1024, 2), (2, 700, 3)])
def test_backward_tensor_cores_longer_sequences(cuda_device, B, T, H):
    """The chunked tensor-core backward over 11-16 chunks (the reverse pass
    carries dL/dS across all of them), with S0 and dL/dS_T."""
    inp, dout, dST = _case(B, T, H, 128, torch.bfloat16, "scalar", True, True, seed=130 + T)
    _check(_run(inp, dout, dST, cuda_device), _oracle(inp, dout, dST), 2e-2)
    assert binding.device_status() == 0


def test_backward_workload_agrees_with_cuda_core_backward(cuda_device):
    """The backward workload at the 350M shape (B8 T4096 H16 d128): the
    tensor-core chunked backward (scalar gate) against the fp32 CUDA-core
    recurrence on the same inputs with the gate given per channel (every
    channel the head's value: the same recurrence; its per-channel dg sums to
    the scalar one).  Bar: 2e-2 on every gradient."""
    from gated_delta_rule_93_b200.inputs import WORKLOADS, make_workload_inputs
    w = WORKLOADS["gdn_bwd_b8_t4096_h16_d128"]
    inp = make_workload_inputs(w)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    tc = binding.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dout"], d["S0"])
    gch = d["g"][..., None].expand(*d["g"].shape, 128).contiguous()
    ref = binding.chunk_bwd(d["q"], d["k"], d["v"], gch, d["beta"], d["dout"], d["S0"])
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    ref["dg"] = ref["dg"].sum(-1)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        e = ((tc[name] - ref[name]).abs().max() / ref[name].abs().max()).item()
        assert e <= 2e-2, f"{name}: {e:.3e}"
