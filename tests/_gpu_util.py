"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding and the fp64 oracle on the very same (rounded) inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.inputs import to_numpy_input
from tests._pins import rel_err

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def gpu_chunk(inp, device, output_final_state=True):
    d = {k: (v.to(device) if v is not None else None) for k, v in inp.items()}
    o, S_T = binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"],
                               output_final_state=output_final_state)
    torch.cuda.synchronize(device)
    return o, S_T


def oracle_chunk(inp, nthreads=None):
    gate = "channel" if inp["g"].dim() == 4 else "scalar"
    S0 = None if inp["S0"] is None else inp["S0"].double().numpy()
    return oracle.gdr_fwd(to_numpy_input(inp["q"]), to_numpy_input(inp["k"]),
                          to_numpy_input(inp["v"]), inp["g"].numpy(), inp["beta"].numpy(), S0,
                          gate=gate, nthreads=nthreads)


def err(gpu_t, ref):
    return rel_err(gpu_t.detach().float().cpu().double().numpy(), ref)


def assert_close(gpu_t, ref, tol, what):
    e = err(gpu_t, ref)
    assert np.isfinite(e) and e <= tol, f"{what}: max|d|/max|ref| = {e:.3e} > {tol:.1e}"
    return e
