"""Failure reporting on the GPU without faulting it: a bounded wait that runs
out sets the device status word; the kernel unwinds and the context stays
usable."""
import pytest
import torch

from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import make_chunk_inputs
from tests._gpu_util import assert_close, gpu_chunk, oracle_chunk

pytestmark = pytest.mark.gpu


def test_skipped_stage_load_times_out_and_reports(cuda_device):
    inp = make_chunk_inputs(1, 256, 2, 128, 128, torch.bfloat16, "scalar", False, seed=13)
    d = {k: (v.to(cuda_device) if v is not None else None) for k, v in inp.items()}
    assert binding.device_status() == binding.GDR_OK
    binding.testing_skip_stage_load(1)  # chunk 1's inputs never arrive
    binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None)
    assert binding.device_status() == binding.GDR_ERR_TIMEOUT
    # the status word was cleared by the read, and the context still works
    o, S_T = gpu_chunk(inp, cuda_device)
    ro, rS = oracle_chunk(inp)
    assert_close(o, ro, 2e-2, "o after recovery")
    assert_close(S_T, rS, 2e-2, "S_T after recovery")
    assert binding.device_status() == binding.GDR_OK


def test_skip_hook_rejects_negative_chunk():
    with pytest.raises(binding.GdrError):
        binding.testing_skip_stage_load(-1)
