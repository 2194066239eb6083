"""GPU parity of gdr_chunk_bwd (gradients of the recurrence) against the fp64
oracle's backward, which is pinned to finite differences of the forward.

The CUDA path computes in fp32 on the very same (bf16 or fp32) inputs, so
the bar is max|gpu - oracle| / max|oracle| <= 1e-4 on every gradient.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import make_chunk_inputs, to_numpy_input
from tests._gpu_util import assert_close

pytestmark = pytest.mark.gpu

TOL = 1e-4


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


def _check(out, ref):
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        assert_close(out[name], ref[name], TOL, name)


# d = 128 bf16 (the tensor-core forward's shape): two full 64-token chunks and a ragged tail
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("with_S0,with_dST", [(True, True), (False, False), (False, True)])
def test_backward_matches_oracle_d128(cuda_device, gate, with_S0, with_dST):
    inp, dout, dST = _case(2, 150, 2, 128, torch.bfloat16, gate, with_S0, with_dST, seed=120)
    _check(_run(inp, dout, dST, cuda_device), _oracle(inp, dout, dST))
    assert binding.device_status() == 0


@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_backward_matches_oracle_small_heads_fp32(cuda_device, d, gate):
    inp, dout, dST = _case(2, 130, 3, d, torch.float32, gate, True, True, seed=121 + d)
    _check(_run(inp, dout, dST, cuda_device), _oracle(inp, dout, dST))


@pytest.mark.parametrize("T", [1, 64])
def test_backward_short_sequences(cuda_device, T):
    inp, dout, dST = _case(1, T, 2, 128, torch.bfloat16, "scalar", True, True, seed=125 + T)
    _check(_run(inp, dout, dST, cuda_device), _oracle(inp, dout, dST))


def test_backward_empty_sequence_passes_dST_through(cuda_device):
    inp, dout, dST = _case(2, 0, 2, 64, torch.float32, "scalar", True, True, seed=127)
    out = _run(inp, dout, dST, cuda_device)
    assert torch.equal(out["dS0"].cpu(), dST)


def test_backward_of_zero_upstream_is_zero(cuda_device):
    inp, dout, _ = _case(1, 100, 2, 128, torch.bfloat16, "channel", True, False, seed=128)
    out = _run(inp, torch.zeros_like(dout), None, cuda_device)
    for name, t in out.items():
        assert torch.count_nonzero(t).item() == 0, name
