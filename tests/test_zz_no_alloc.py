"""The entry point that allocates nothing: gdr_chunk_fwd_segmented_noalloc.

Some callers cannot allocate device memory while they run the mixer (a
plugin inside a host framework that owns the device's memory pool and gives
it no allocator, or a serving loop that must not stall on cudaMalloc /
cudaFree, which can synchronise the whole device).  This entry point runs
the segment path of the chunked forward with its scratch in a fixed array
built into the library.  Here it is called through the C ABI (ctypes) and
compared with gdr_chunk_fwd_segmented, which takes the same scratch from a
caller's workspace, on two calls in a row (so the second call starts from
whatever the first one left in the shared array).

The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.build import build
from gated_delta_rule_93_b200.inputs import make_chunk_inputs
from tests._gpu_util import TOL, assert_close

D = 128


def _noalloc(L, d, o, S_T, P):
    """Call the C entry point directly: raw device pointers, the current stream."""
    B, T, H, _ = d["q"].shape
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.gdr_chunk_fwd_segmented_noalloc(
        p(d["q"]), p(d["k"]), p(d["v"]), binding.GDR_BF16, p(d["g"]),
        binding.GDR_GATE_PER_CHANNEL if d["g"].dim() == 4 else binding.GDR_GATE_SCALAR,
        p(d["beta"]), p(d["S0"]), p(o), p(S_T), B, T, H, D, D, 64, P, stream)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device):
    L = binding.lib()
    # first call: 32 segment-heads with S0; second: 8 segment-heads without
    # S0 and another gate, reading a region the first call left behind
    cases = [(1, 8192, 4, 8, "scalar", True, 41), (2, 2048, 2, 2, "channel", False, 42)]
    for B, T, H, P, gate, with_S0, seed in cases:
        inp = make_chunk_inputs(B, T, H, D, D, torch.bfloat16, gate, with_S0, seed=seed)
        d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
        o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=cuda_device)
        S_T = torch.empty((B, H, D, D), dtype=torch.float32, device=cuda_device)
        rc = _noalloc(L, d, o, S_T, P)
        assert rc == binding.GDR_OK, L.gdr_last_error_message().decode()
        ws = torch.empty(3 * B * P * H * D * D * 4, dtype=torch.uint8, device=cuda_device)
        ro, rS = binding.chunk_fwd_segmented(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"],
                                             segments=P, workspace=ws)
        torch.cuda.synchronize()
        assert binding.device_status() == 0
        assert torch.isfinite(o.float()).all() and torch.isfinite(S_T).all()
        ref_o, ref_S = ro.double().cpu().numpy(), rS.double().cpu().numpy()
        assert_close(o, ref_o, TOL[torch.bfloat16], f"o (B{B} T{T} H{H} P{P})")
        assert_close(S_T, ref_S, TOL[torch.bfloat16], f"S_T (B{B} T{T} H{H} P{P})")


def test_noalloc_refuses_more_than_its_scratch():
    """B*P*H above what the fixed array holds is refused before anything is
    enqueued (fake pointers: nothing may touch them)."""
    build()
    L = binding.lib()
    fake = ctypes.c_void_p(0x10000)
    per_unit = 3 * D * D * 4
    assert binding.NOALLOC_SCRATCH_BYTES // per_unit == 128

    def call(B, H, P, T=65536):
        return L.gdr_chunk_fwd_segmented_noalloc(fake, fake, fake, binding.GDR_BF16, fake,
                                                 binding.GDR_GATE_SCALAR, fake, None, fake, None,
                                                 B, T, H, D, D, 64, P, None)

    assert call(1, 32, 8) == binding.GDR_ERR_WORKSPACE
    assert "scratch" in L.gdr_last_error_message().decode()
    assert call(2, 16, 8) == binding.GDR_ERR_WORKSPACE
    assert call(1, 16, 3) == binding.GDR_ERR_UNSUPPORTED  # segments of whole chunks
    assert call(0, 16, 8) == binding.GDR_OK               # empty: nothing to do
