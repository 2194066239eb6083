"""GPU parity of gdr_chunk_fwd against the fp64 oracle (element by element).

Acceptance: max|gpu - oracle| / max|oracle| <= 1e-4 for fp32 inputs and
<= 2e-2 for bf16 inputs with an fp32 state, on o and on S_T separately.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import WORKLOADS, make_chunk_inputs, make_workload_inputs
from tests._gpu_util import TOL, assert_close, gpu_chunk, oracle_chunk

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("T,with_S0", [(256, False), (200, True), (1, True), (64, False)])
def test_chunk_small_shapes(cuda_device, dtype, gate, d, T, with_S0):
    """Several chunks, ragged tails (200 = 3 x 64 + 8, 1), every head size."""
    inp = make_chunk_inputs(2, T, 3, d, d, dtype, gate, with_S0, seed=T + d)
    o, S_T = gpu_chunk(inp, cuda_device)
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, TOL[dtype], "o")
    assert_close(S_T, rS, TOL[dtype], "S_T")


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 32), (32, 64)])
def test_chunk_unequal_head_dims(cuda_device, dk, dv):
    inp = make_chunk_inputs(1, 150, 2, dk, dv, torch.bfloat16, "scalar", True, seed=5)
    o, S_T = gpu_chunk(inp, cuda_device)
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 2e-2, "S_T")


def test_tiny_fp32_workload(cuda_device):
    """Tiny Gated DeltaNet forward, fp32: B1 H2 T256 d32, S0 = 0."""
    w = WORKLOADS["tiny_fp32"]
    inp = make_workload_inputs(w)
    o, S_T = gpu_chunk(inp, cuda_device)
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 1e-4, "o")
    assert_close(S_T, rS, 1e-4, "S_T")


@pytest.mark.parametrize("name", ["gdn_b8_t4096_h16_d128", "gdn_b1_t65536_h16_d128",
                                  "kda_b8_t4096_h16_d128"])
def test_full_size_workloads(cuda_device, name):
    """The full-size workloads, whole tensors compared with the full oracle."""
    w = WORKLOADS[name]
    inp = make_workload_inputs(w)
    o, S_T = gpu_chunk(inp, cuda_device)
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, TOL[w.dtype], f"{name} o")
    assert_close(S_T, rS, TOL[w.dtype], f"{name} S_T")


def test_empty_sequence_returns_initial_state(cuda_device):
    inp = make_chunk_inputs(2, 0, 2, 64, 64, torch.bfloat16, "scalar", True, seed=1)
    o, S_T = gpu_chunk(inp, cuda_device)
    assert o.numel() == 0
    assert torch.equal(S_T.cpu(), inp["S0"])


def test_no_final_state_and_zero_initial_state(cuda_device):
    inp = make_chunk_inputs(1, 130, 2, 128, 128, torch.bfloat16, "scalar", False, seed=2)
    o, S_T = gpu_chunk(inp, cuda_device, output_final_state=False)
    assert S_T is None
    ro, _ = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o")


def test_initial_state_may_alias_final_state(cuda_device):
    inp = make_chunk_inputs(2, 100, 2, 128, 128, torch.bfloat16, "channel", True, seed=3)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    S = d["S0"].clone()
    o, S_T = binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, S_T=S)
    torch.cuda.synchronize()
    ro, rS = oracle_chunk(inp)
    assert S_T.data_ptr() == S.data_ptr()
    assert_close(o, ro, 2e-2, "o")
    assert_close(S, rS, 2e-2, "S_T (aliased)")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_strong_scalar_forgetting_has_no_nan(cuda_device, dtype):
    """g = -30 at every step (alpha ~ 1e-13): history is erased in one step and
    nothing overflows (every exponent the scalar path forms is <= 0)."""
    inp = make_chunk_inputs(1, 192, 2, 64, 64, dtype, "scalar", True, seed=4)
    inp["g"][:] = -30.0
    o, S_T = gpu_chunk(inp, cuda_device)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S_T).all()
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, TOL[dtype], "o")
    assert_close(S_T, rS, TOL[dtype], "S_T")


def test_strong_per_channel_decay_tensor_cores(cuda_device):
    """Per-channel gates 20x the usual recipe (alpha ~ 0.2 per token): the
    log decay over a 32-token half chunk reaches about -72 in some channel.
    The operand factors e^{gc - m} stay inside bf16's range there, and the
    state's change of frame between chunks is applied as two factors (their
    product would underflow fp32)."""
    inp = make_chunk_inputs(1, 512, 2, 128, 128, torch.bfloat16, "channel", True, seed=77)
    inp["g"] = inp["g"] * 20.0
    o, S_T = gpu_chunk(inp, cuda_device)
    assert binding.device_status() == 0
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 2e-2, "S_T")


def test_beta_zero_is_pure_decay(cuda_device):
    """beta = 0: no write, so S_T = S0 Diag(exp(sum g)) (closed form)."""
    inp = make_chunk_inputs(1, 160, 2, 64, 32, torch.float32, "channel", True, seed=6)
    inp["beta"][:] = 0.0
    o, S_T = gpu_chunk(inp, cuda_device)
    G = inp["g"].double().sum(dim=1)  # [B,H,dk]
    want = inp["S0"].double() * torch.exp(G)[:, :, None, :]
    e = (S_T.cpu().double() - want).abs().max() / want.abs().max()
    assert e < 1e-5


def test_split_and_resume_on_gpu(cuda_device):
    """fwd(T1) then fwd(T2, S0 = S_T1) equals fwd(T1 + T2)."""
    inp = make_chunk_inputs(2, 320, 2, 128, 128, torch.bfloat16, "scalar", True, seed=7)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    o, S_T = binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    t1 = 192
    oa, Sa = binding.chunk_fwd(d["q"][:, :t1].contiguous(), d["k"][:, :t1].contiguous(),
                               d["v"][:, :t1].contiguous(), d["g"][:, :t1].contiguous(),
                               d["beta"][:, :t1].contiguous(), d["S0"])
    ob, Sb = binding.chunk_fwd(d["q"][:, t1:].contiguous(), d["k"][:, t1:].contiguous(),
                               d["v"][:, t1:].contiguous(), d["g"][:, t1:].contiguous(),
                               d["beta"][:, t1:].contiguous(), Sa)
    torch.cuda.synchronize()
    ro, rS = oracle_chunk(inp)
    assert_close(torch.cat([oa, ob], dim=1), ro, 2e-2, "o split")
    assert_close(Sb, rS, 2e-2, "S_T split")


def test_linearity_in_values(cuda_device):
    """o(S0, V1 + V2) = o(S0, V1) + o(0, V2) for fixed q, k, gates (fp32).
    Three runs of the split-operand path, each within a few 2^-18 per product
    of exact (two bf16 terms per operand, three MMAs per product): bar 5e-5."""
    a = make_chunk_inputs(1, 130, 2, 64, 64, torch.float32, "scalar", True, seed=8)
    b = make_chunk_inputs(1, 130, 2, 64, 64, torch.float32, "scalar", True, seed=9)
    d = {k: v.to(cuda_device) for k, v in a.items()}
    v2 = b["v"].to(cuda_device)
    o1, s1 = binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    o2, s2 = binding.chunk_fwd(d["q"], d["k"], v2, d["g"], d["beta"], None)
    o12, s12 = binding.chunk_fwd(d["q"], d["k"], d["v"] + v2, d["g"], d["beta"], d["S0"])
    torch.cuda.synchronize()
    assert ((o1 + o2 - o12).abs().max() / o12.abs().max()).item() < 5e-5
    assert ((s1 + s2 - s12).abs().max() / s12.abs().max()).item() < 5e-5


def test_misaligned_pointer_is_rejected(cuda_device):
    inp = make_chunk_inputs(1, 64, 1, 64, 64, torch.bfloat16, "scalar", False, seed=10)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    buf = torch.empty(64 * 64 + 1, dtype=torch.bfloat16, device=cuda_device)
    q_bad = buf[1:].view(1, 64, 1, 64)
    with pytest.raises(binding.GdrError, match="aligned"):
        binding.chunk_fwd(q_bad, d["k"], d["v"], d["g"], d["beta"])
    assert binding.device_status() == 0


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("with_S0", [True, False])
def test_segment_path_matches_oracle(cuda_device, gate, with_S0):
    """A long sequence with few heads runs as segments (two passes, a combine
    of the segments' states, a final pass): B1 H2 T4096 d128 is 4 segments of
    16 chunks on a B200."""
    B, T, H, d = 1, 4096, 2, 128
    assert binding.chunk_fwd_kernel_launches(B, T, H, d, d, gate=gate) == 4
    assert binding.chunk_fwd_workspace_bytes(B, T, H, d, d, gate=gate) == 3 * B * 4 * H * d * d * 4
    inp = make_chunk_inputs(B, T, H, d, d, torch.bfloat16, gate, with_S0, seed=11)
    o, S_T = gpu_chunk(inp, cuda_device)
    assert binding.device_status() == 0
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 2e-2, "S_T")


@pytest.mark.parametrize("gscale", [0.0, 0.0125])
@pytest.mark.parametrize("P", [None, 8])
def test_segment_path_weak_decay(cuda_device, gscale, P):
    """Weak decay, where a segment's transition M_p is far from zero: g = 0
    (the delta rule, "Decoding Hybrid Linear Attention Architectures",
    section 3 item 2) and g of about -0.001 per token (the default gates
    times 0.0125).  The segment path recovers M_p = (M_p + E_p) - E_p from
    two runs; here that difference is not damped.  B1 H2 T4096 d128 with S0,
    the automatic segment path (4 segments) and the segmented entry point
    with 8 segments."""
    B, T, H, d = 1, 4096, 2, 128
    inp = make_chunk_inputs(B, T, H, d, d, torch.bfloat16, "scalar", True, seed=17)
    inp["g"] = (inp["g"] * gscale).contiguous()
    dd = {k: v.to(cuda_device) for k, v in inp.items()}
    if P is None:
        assert binding.chunk_fwd_kernel_launches(B, T, H, d, d) == 4
        o, S_T = binding.chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"])
    else:
        ws = torch.empty(3 * B * P * H * d * d * 4, dtype=torch.uint8, device=cuda_device)
        o, S_T = binding.chunk_fwd_segmented(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                             dd["S0"], segments=P, workspace=ws)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 2e-2, "S_T")


def test_segment_path_initial_state_may_alias_final_state(cuda_device):
    inp = make_chunk_inputs(1, 4096, 2, 128, 128, torch.bfloat16, "scalar", True, seed=12)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    S = d["S0"].clone()
    o, S_T = binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], S, S_T=S)
    torch.cuda.synchronize()
    ro, rS = oracle_chunk(inp)
    assert S_T.data_ptr() == S.data_ptr()
    assert_close(o, ro, 2e-2, "o")
    assert_close(S, rS, 2e-2, "S_T (aliased)")


def test_segment_path_rejects_short_workspace(cuda_device):
    inp = make_chunk_inputs(1, 4096, 2, 128, 128, torch.bfloat16, "scalar", False, seed=13)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    small = torch.empty(16, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(binding.GdrError) as ei:
        binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, workspace=small)
    assert ei.value.status == binding.GDR_ERR_WORKSPACE


def test_segment_rule_leaves_wide_batches_alone(cuda_device):
    """B*H large enough to fill the SMs, short sequences, fp32 inputs or other
    head sizes: one launch, no workspace."""
    for args, kw in [((8, 4096, 16, 128, 128), {}), ((1, 512, 2, 128, 128), {}),
                     ((1, 65536, 16, 128, 128), {"dtype": torch.float32}),
                     ((1, 65536, 2, 64, 64), {})]:
        assert binding.chunk_fwd_kernel_launches(*args, **kw) == 1, args
        assert binding.chunk_fwd_workspace_bytes(*args, **kw) == 0, args


@pytest.mark.parametrize("gate,P", [("scalar", 2), ("scalar", 8), ("channel", 4),
                                    ("scalar", 3)])
def test_segmented_entry_point_matches_oracle(cuda_device, gate, P):
    """gdr_chunk_fwd_segmented with the caller's P and workspace (nothing is
    allocated by the call): B2 H2 T1536 (24 chunks) with S0."""
    B, T, H, d = 2, 1536, 2, 128
    inp = make_chunk_inputs(B, T, H, d, d, torch.bfloat16, gate, True, seed=20 + P)
    dd = {k: v.to(cuda_device) for k, v in inp.items()}
    ws = torch.empty(3 * B * P * H * d * d * 4, dtype=torch.uint8, device=cuda_device)
    o, S_T = binding.chunk_fwd_segmented(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                                         dd["S0"], segments=P, workspace=ws)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 2e-2, "S_T")


def test_segmented_entry_point_rejects_short_workspace(cuda_device):
    inp = make_chunk_inputs(1, 1024, 2, 128, 128, torch.bfloat16, "scalar", False, seed=30)
    dd = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    ws = torch.empty(3 * 4 * 2 * 128 * 128 * 4 - 16, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(binding.GdrError) as ei:
        binding.chunk_fwd_segmented(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], None,
                                    segments=4, workspace=ws)
    assert ei.value.status == binding.GDR_ERR_WORKSPACE


def _one_channel_decay(inp, g_channel, channel=5, head=0):
    g = inp["g"].clone()
    g[:, :, head, channel] = g_channel
    return dict(inp, g=g.contiguous())


def test_per_channel_strong_decay_within_range(cuda_device):
    """One key channel forgetting fast, e^{-2.5} per token (-80 over half a
    chunk), inside the tensor-core path's range: oracle parity, clean status."""
    inp = _one_channel_decay(make_chunk_inputs(1, 256, 2, 128, 128, torch.bfloat16, "channel",
                                               True, seed=61), -2.5)
    o, S_T = gpu_chunk(inp, cuda_device)
    assert binding.device_status() == binding.GDR_OK
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o")
    assert_close(S_T, rS, 2e-2, "S_T")


def test_per_channel_rapid_forgetting_reports_range(cuda_device):
    """One key channel at g = -30 per token ("one-step rapid forgetting",
    "Decoding Hybrid Linear Attention Architectures", section 4) is beyond
    what the tensor-core path's tile scaling represents: the call records
    GDR_ERR_RANGE in the device status word and its outputs stay finite."""
    inp = _one_channel_decay(make_chunk_inputs(1, 256, 2, 128, 128, torch.bfloat16, "channel",
                                               True, seed=62), -30.0)
    o, S_T = gpu_chunk(inp, cuda_device)
    assert binding.device_status() == binding.GDR_ERR_RANGE
    assert torch.isfinite(o.float()).all() and torch.isfinite(S_T).all()
    # the status word was cleared by the read; a call within range is clean
    inp2 = make_chunk_inputs(1, 128, 2, 128, 128, torch.bfloat16, "channel", False, seed=63)
    gpu_chunk(inp2, cuda_device)
    assert binding.device_status() == binding.GDR_OK


@pytest.mark.parametrize("d,dtype", [(64, torch.bfloat16), (128, torch.float32), (32, torch.float32)])
def test_per_channel_strong_decay_split_path(cuda_device, d, dtype):
    """The split-operand path (d < 128 or fp32 inputs): one key channel at
    g = -2 per token (-62 over half a chunk, inside its 2^100 factor range)
    matches the oracle at the dtype's bar, with a clean status."""
    inp = _one_channel_decay(make_chunk_inputs(1, 200, 2, d, d, dtype, "channel", True,
                                               seed=64), -2.0)
    o, S_T = gpu_chunk(inp, cuda_device)
    assert binding.device_status() == binding.GDR_OK
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, TOL[dtype], "o")
    assert_close(S_T, rS, TOL[dtype], "S_T")


@pytest.mark.parametrize("d,dtype", [(64, torch.bfloat16), (128, torch.float32)])
def test_per_channel_rapid_forgetting_split_path_reports_range(cuda_device, d, dtype):
    """g = -30 per token in one channel is beyond the split-operand path's
    factor range too: GDR_ERR_RANGE in the status word, finite outputs."""
    inp = _one_channel_decay(make_chunk_inputs(1, 200, 2, d, d, dtype, "channel", True,
                                               seed=65), -30.0)
    o, S_T = gpu_chunk(inp, cuda_device)
    assert binding.device_status() == binding.GDR_ERR_RANGE
    assert torch.isfinite(o.float()).all() and torch.isfinite(S_T).all()
