"""GPU parity of gdr_step (recurrent decode step) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import (WORKLOADS, make_chunk_inputs, make_step_inputs,
                                             to_numpy_input)
from tests._gpu_util import TOL, assert_close, gpu_chunk, oracle_chunk
from tests._pins import rel_err

pytestmark = pytest.mark.gpu


def _run_steps(inp, device, steps):
    S = inp["S0"].to(device).clone()
    outs = []
    for i in range(steps):
        o = binding.step(inp["q"][i].to(device), inp["k"][i].to(device), inp["v"][i].to(device),
                         inp["g"][i].to(device), inp["beta"][i].to(device), S)
        outs.append(o)
    torch.cuda.synchronize()
    return torch.stack(outs), S


def _oracle_steps(inp, steps, gate):
    S = inp["S0"].double().numpy().copy()
    outs = []
    for i in range(steps):
        outs.append(oracle.gdr_step(to_numpy_input(inp["q"][i]), to_numpy_input(inp["k"][i]),
                                    to_numpy_input(inp["v"][i]), inp["g"][i].numpy(),
                                    inp["beta"][i].numpy(), S, gate=gate))
    return np.stack(outs), S


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (64, 128), (128, 32)])
def test_step_small(cuda_device, dtype, gate, dk, dv):
    inp = make_step_inputs(5, 3, dk, dv, steps=12, dtype=dtype, gate=gate, seed=dk + dv)
    o, S = _run_steps(inp, cuda_device, 12)
    ro, rS = _oracle_steps(inp, 12, gate)
    assert_close(o, ro, TOL[dtype], "o")
    assert_close(S, rS, TOL[dtype], "S")


def test_decode_workload_1024_steps(cuda_device):
    """256 sequences x 16 heads x d128, 1024 consecutive steps, whole output
    and final state checked against 1024 oracle steps."""
    w = WORKLOADS["decode_n256_h16_d128_x1024"]
    inp = make_step_inputs(w.B, w.H, w.dk, w.dv, steps=w.steps, dtype=w.dtype, gate=w.gate)
    o, S = _run_steps(inp, cuda_device, w.steps)
    ro, rS = _oracle_steps(inp, w.steps, w.gate)
    assert_close(o, ro, 2e-2, "o (all steps)")
    assert_close(S, rS, 2e-2, "S after 1024 steps")


def test_prefill_then_decode_handoff(cuda_device):
    """Chunked prefill over T tokens, then gdr_step on the next tokens from the
    returned S_T, equals the oracle over the whole sequence."""
    T, n = 200, 6
    inp = make_chunk_inputs(2, T + n, 2, 128, 128, torch.bfloat16, "scalar", True, seed=11)
    pre = {k: (v[:, :T].contiguous() if k != "S0" else v) for k, v in inp.items()}
    o_pre, S_T = gpu_chunk(pre, cuda_device)
    S = S_T.clone()
    outs = []
    for t in range(T, T + n):
        outs.append(binding.step(*(inp[x][:, t].contiguous().to(cuda_device)
                                   for x in ("q", "k", "v", "g", "beta")), S))
    torch.cuda.synchronize()
    ro, rS = oracle_chunk(inp)
    assert_close(o_pre, ro[:, :T], 2e-2, "prefill o")
    assert_close(torch.stack(outs, dim=1), ro[:, T:], 2e-2, "decode o")
    assert_close(S, rS, 2e-2, "final state")


def test_step_beta_one_replaces(cuda_device):
    """beta = 1, ||k|| = 1, q = k: o = v for any state and gate."""
    N, H, d = 8, 4, 128
    g = torch.Generator().manual_seed(3)
    k = torch.zeros(N, H, d)
    idx = torch.randint(0, d, (N, H), generator=g)
    k.scatter_(2, idx[..., None], 1.0)
    v = torch.randn(N, H, d, generator=g)
    S = torch.randn(N, H, d, d, generator=g).cuda()
    o = binding.step(k.cuda(), k.cuda(), v.cuda(), -torch.rand(N, H).cuda(),
                     torch.ones(N, H).cuda(), S)
    torch.cuda.synchronize()
    assert (o.cpu() - v).abs().max().item() < 1e-5
