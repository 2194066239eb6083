"""GPU parity of gdr_chunk_fwd_varlen (packed sequences of different lengths)
against the fp64 oracle sequence by sequence, against the dense entry point
on each sequence alone, and the prefill -> decode hand-off to gdr_step.

Acceptance as for gdr_chunk_fwd: max|gpu - oracle| / max|oracle| <= 2e-2
(bf16 inputs, fp32 state), on o and on S_T separately.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import make_varlen_inputs, to_numpy_input
from tests._gpu_util import assert_close

pytestmark = pytest.mark.gpu

# empty, single-token, exact-chunk, ragged and several-chunk sequences
LENS = [100, 0, 64, 1, 257, 31, 128, 190]


def _run(inp, dev, **kw):
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o, S_T = binding.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                                      d["S0"], **kw)
    torch.cuda.synchronize(dev)
    return o, S_T


def _oracle_seq(inp, i):
    """The fp64 oracle on sequence i alone (a batch of one)."""
    cu = inp["cu_seqlens"].tolist()
    s0, s1 = cu[i], cu[i + 1]
    gate = "channel" if inp["g"].dim() == 3 else "scalar"
    S0 = None if inp["S0"] is None else inp["S0"][i:i + 1].double().numpy()
    sl = lambda t: t[s0:s1].unsqueeze(0)
    return oracle.gdr_fwd(to_numpy_input(sl(inp["q"])), to_numpy_input(sl(inp["k"])),
                          to_numpy_input(sl(inp["v"])), sl(inp["g"]).numpy(),
                          sl(inp["beta"]).numpy(), S0, gate=gate)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("with_S0", [True, False])
def test_varlen_matches_oracle(cuda_device, gate, with_S0):
    inp = make_varlen_inputs(LENS, 2, 128, 128, torch.bfloat16, gate, with_S0, seed=40)
    o, S_T = _run(inp, cuda_device)
    assert binding.device_status() == 0
    cu = inp["cu_seqlens"].tolist()
    for i, n in enumerate(LENS):
        ro, rS = _oracle_seq(inp, i)
        if n:
            assert_close(o[cu[i]:cu[i + 1]].unsqueeze(0), ro, 2e-2, f"o of sequence {i}")
        assert_close(S_T[i:i + 1], rS, 2e-2, f"S_T of sequence {i}")


def test_varlen_empty_sequence_keeps_initial_state(cuda_device):
    inp = make_varlen_inputs(LENS, 2, 128, 128, torch.bfloat16, "scalar", True, seed=41)
    _, S_T = _run(inp, cuda_device)
    assert torch.equal(S_T[1].cpu(), inp["S0"][1])


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_varlen_equals_dense_calls(cuda_device, gate):
    """Each packed sequence gives what gdr_chunk_fwd gives on it alone: the
    rows past a sequence's end enter with beta = 0 and g = 0, so they add
    exact zeros."""
    inp = make_varlen_inputs(LENS, 2, 128, 128, torch.bfloat16, gate, True, seed=42)
    o, S_T = _run(inp, cuda_device)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    cu = inp["cu_seqlens"].tolist()
    for i, n in enumerate(LENS):
        if n == 0:
            continue
        sl = lambda t: t[cu[i]:cu[i + 1]].unsqueeze(0).clone()  # own (aligned) storage
        od, Sd = binding.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]),
                                   sl(d["beta"]), d["S0"][i:i + 1].clone())
        torch.cuda.synchronize()
        assert torch.equal(o[cu[i]:cu[i + 1]], od[0]), f"o of sequence {i}"
        assert torch.equal(S_T[i], Sd[0]), f"S_T of sequence {i}"


def test_prefill_then_decode(cuda_device):
    """Prefill each sequence's first tokens with gdr_chunk_fwd_varlen, then
    decode its next token with gdr_step from S_T: the same as the oracle over
    the longer sequence."""
    full = [71, 130, 1, 64]
    inp = make_varlen_inputs([n + 1 for n in full], 2, 128, 128, torch.bfloat16, "scalar", True,
                             seed=43)
    cu = inp["cu_seqlens"].tolist()
    pre = torch.cat([torch.arange(cu[i], cu[i] + n) for i, n in enumerate(full)])
    last = torch.tensor([cu[i] + n for i, n in enumerate(full)])
    pre_inp = {k: inp[k][pre] for k in ("q", "k", "v", "g", "beta")}
    pre_inp["S0"] = inp["S0"]
    cu_pre = [0]
    for n in full:
        cu_pre.append(cu_pre[-1] + n)
    pre_inp["cu_seqlens"] = torch.tensor(cu_pre, dtype=torch.int32)
    _, S = _run(pre_inp, cuda_device)
    step = {k: inp[k][last].to(cuda_device) for k in ("q", "k", "v", "g", "beta")}
    o1 = binding.step(step["q"], step["k"], step["v"], step["g"], step["beta"], S)
    torch.cuda.synchronize()
    for i in range(len(full)):
        ro, rS = _oracle_seq(inp, i)
        assert_close(o1[i:i + 1], ro[:, -1], 2e-2, f"decoded o of sequence {i}")
        assert_close(S[i:i + 1], rS, 2e-2, f"state after decode of sequence {i}")


def test_varlen_rejects_unsupported_shapes(cuda_device):
    inp = make_varlen_inputs([10, 20], 2, 48, 48, torch.bfloat16, "scalar", False, seed=44)
    with pytest.raises(binding.GdrError) as ei:
        _run(inp, cuda_device)
    assert ei.value.status == binding.GDR_ERR_UNSUPPORTED


# the split-operand kernel: fp32 inputs (bar 1e-4) and other head dims
@pytest.mark.parametrize("dk,dv,dtype,gate", [(64, 64, torch.float32, "scalar"),
                                              (32, 64, torch.float32, "channel"),
                                              (128, 64, torch.bfloat16, "scalar")])
def test_varlen_split_operand_shapes(cuda_device, dk, dv, dtype, gate):
    inp = make_varlen_inputs(LENS, 2, dk, dv, dtype, gate, True, seed=45 + dk + dv)
    o, S_T = _run(inp, cuda_device)
    assert binding.device_status() == 0
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    cu = inp["cu_seqlens"].tolist()
    for i, n in enumerate(LENS):
        ro, rS = _oracle_seq(inp, i)
        if n:
            assert_close(o[cu[i]:cu[i + 1]].unsqueeze(0), ro, tol, f"o of sequence {i}")
        assert_close(S_T[i:i + 1], rS, tol, f"S_T of sequence {i}")
