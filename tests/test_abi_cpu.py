"""Host-side checks of the C-ABI library (no GPU, no compute calls)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_93_b200 import binding
from gated_delta_rule_93_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return binding.lib()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"\b(gdr_\w+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert "gdr_chunk_fwd" in declared and "gdr_step" in declared
    for name in declared:
        assert hasattr(L, name), f"{name} declared in include/ but not exported"
    assert set(binding.EXPORTS) <= set(declared)


def test_no_driver_dependency(L):
    """The library links the CUDA runtime statically and needs no libcuda at
    load time (it loads on this GPU-less host)."""
    assert L.gdr_version() == 100


def test_status_strings(L):
    for code, name in enumerate(["GDR_OK", "GDR_ERR_INVALID_ARG", "GDR_ERR_UNSUPPORTED",
                                 "GDR_ERR_WORKSPACE", "GDR_ERR_CUDA", "GDR_ERR_TIMEOUT",
                                 "GDR_ERR_RANGE"]):
        assert binding.status_string(code) == name


def test_workspace_query(L):
    assert L.gdr_chunk_fwd_workspace_bytes(8, 4096, 16, 128, 128, 64, 1, 0) == 0
    # the segment path depends on the device's SM count: none without a GPU,
    # three fp32 states per segment and head with one
    import torch

    ws = L.gdr_chunk_fwd_workspace_bytes(1, 65536, 16, 128, 128, 64, 1, 0)
    if torch.cuda.is_available():
        assert ws > 0 and ws % (3 * 16 * 128 * 128 * 4) == 0
    else:
        assert ws == 0
    assert L.gdr_chunk_fwd_kernel_launches(8, 4096, 16, 128, 128, 64, 1, 0) == 1
    assert L.gdr_chunk_fwd_kernel_launches(0, 4096, 16, 128, 128, 64, 1, 0) == 0


def _fake_ptr(off=0):
    return ctypes.c_void_p(0x10000 + off)


def test_validation_rejects_before_any_launch(L):
    p = _fake_ptr()
    args = lambda **kw: dict(dict(q=p, k=p, v=p, dt=1, g=p, gate=0, beta=p, S0=None, o=p,
                                  ST=None, B=1, T=64, H=1, dk=128, dv=128, C=64, ws=None,
                                  wsb=0, st=None), **kw)

    def call(**kw):
        a = args(**kw)
        return L.gdr_chunk_fwd(a["q"], a["k"], a["v"], a["dt"], a["g"], a["gate"], a["beta"],
                               a["S0"], a["o"], a["ST"], a["B"], a["T"], a["H"], a["dk"],
                               a["dv"], a["C"], a["ws"], a["wsb"], a["st"])

    assert call(C=32) == binding.GDR_ERR_UNSUPPORTED
    assert call(dk=48) == binding.GDR_ERR_UNSUPPORTED
    assert call(dv=256) == binding.GDR_ERR_UNSUPPORTED
    assert call(dt=7) == binding.GDR_ERR_INVALID_ARG
    assert call(gate=3) == binding.GDR_ERR_INVALID_ARG
    assert call(B=-1) == binding.GDR_ERR_INVALID_ARG
    assert call(q=None) == binding.GDR_ERR_INVALID_ARG
    assert call(o=_fake_ptr(4)) == binding.GDR_ERR_INVALID_ARG
    assert "aligned" in L.gdr_last_error_message().decode()
    assert call(S0=_fake_ptr(8)) == binding.GDR_ERR_INVALID_ARG
    # empty problems succeed without touching the device
    assert call(B=0) == binding.GDR_OK
    assert call(H=0) == binding.GDR_OK

    def step(**kw):
        d = dict(q=p, k=p, v=p, dt=1, g=p, gate=0, beta=p, S=p, o=p, N=4, H=2, dk=128, dv=128,
                 st=None)
        d.update(kw)
        return L.gdr_step(d["q"], d["k"], d["v"], d["dt"], d["g"], d["gate"], d["beta"],
                          d["S"], d["o"], d["N"], d["H"], d["dk"], d["dv"], d["st"])

    assert step(dk=100) == binding.GDR_ERR_UNSUPPORTED
    assert step(S=None) == binding.GDR_ERR_INVALID_ARG
    assert step(S=_fake_ptr(4)) == binding.GDR_ERR_INVALID_ARG
    assert step(N=-2) == binding.GDR_ERR_INVALID_ARG
    assert step(N=0) == binding.GDR_OK


def test_segmented_validation_rejects_before_any_launch(L):
    """gdr_chunk_fwd_segmented: caller-chosen segments, caller's workspace."""
    p = _fake_ptr()
    need = 3 * 2 * 4 * 3 * 128 * 128 * 4  # B=2, P=4, H=3

    def call(**kw):
        a = dict(q=p, k=p, v=p, dt=1, g=p, gate=0, beta=p, S0=None, o=p, ST=None, B=2, T=1024,
                 H=3, dk=128, dv=128, C=64, P=4, ws=p, wsb=need, st=None)
        a.update(kw)
        return L.gdr_chunk_fwd_segmented(a["q"], a["k"], a["v"], a["dt"], a["g"], a["gate"],
                                         a["beta"], a["S0"], a["o"], a["ST"], a["B"], a["T"],
                                         a["H"], a["dk"], a["dv"], a["C"], a["P"], a["ws"],
                                         a["wsb"], a["st"])

    assert call(P=1) == binding.GDR_ERR_UNSUPPORTED
    assert call(P=3) == binding.GDR_ERR_UNSUPPORTED      # 1024 is not 3 x whole chunks
    assert call(T=1000) == binding.GDR_ERR_UNSUPPORTED   # ragged segments
    assert call(dt=0) == binding.GDR_ERR_UNSUPPORTED     # fp32 inputs: single pass only
    assert call(dk=64, dv=64) == binding.GDR_ERR_UNSUPPORTED
    assert call(wsb=need - 1) == binding.GDR_ERR_WORKSPACE
    assert call(ws=None) == binding.GDR_ERR_WORKSPACE
    assert call(ws=_fake_ptr(8)) == binding.GDR_ERR_INVALID_ARG
    assert call(q=None) == binding.GDR_ERR_INVALID_ARG
    assert call(B=0) == binding.GDR_OK


def test_binding_refuses_cpu_tensors(L):
    import torch

    x = torch.zeros(1, 64, 1, 32)
    with pytest.raises(ValueError, match="CUDA"):
        binding.chunk_fwd(x, x, x, torch.zeros(1, 64, 1), torch.zeros(1, 64, 1))


def test_varlen_validation_rejects_before_any_launch(L):
    """gdr_chunk_fwd_varlen: packed sequences, the shapes gdr_chunk_fwd takes."""
    p = _fake_ptr()

    def call(**kw):
        a = dict(q=p, k=p, v=p, dt=1, g=p, gate=0, beta=p, cu=p, S0=None, o=p, ST=None, N=3,
                 total=500, H=2, dk=128, dv=128, C=64, st=None)
        a.update(kw)
        return L.gdr_chunk_fwd_varlen(a["q"], a["k"], a["v"], a["dt"], a["g"], a["gate"],
                                      a["beta"], a["cu"], a["S0"], a["o"], a["ST"], a["N"],
                                      a["total"], a["H"], a["dk"], a["dv"], a["C"], a["st"])

    assert call(N=-1) == binding.GDR_ERR_INVALID_ARG
    assert call(cu=None) == binding.GDR_ERR_INVALID_ARG
    assert call(dt=5) == binding.GDR_ERR_INVALID_ARG
    assert call(dk=48, dv=64) == binding.GDR_ERR_UNSUPPORTED
    assert call(C=32) == binding.GDR_ERR_UNSUPPORTED
    assert call(q=None) == binding.GDR_ERR_INVALID_ARG
    assert call(o=_fake_ptr(2)) == binding.GDR_ERR_INVALID_ARG
    assert call(N=0) == binding.GDR_OK


def test_gla_validation_rejects_before_any_launch(L):
    """gdr_chunk_fwd_gla: no beta; the shapes gdr_chunk_fwd takes."""
    p = _fake_ptr()

    def call(**kw):
        a = dict(q=p, k=p, v=p, dt=1, g=p, gate=0, S0=None, o=p, ST=None, B=2, T=300, H=2,
                 dk=128, dv=128, C=64, st=None)
        a.update(kw)
        return L.gdr_chunk_fwd_gla(a["q"], a["k"], a["v"], a["dt"], a["g"], a["gate"], a["S0"],
                                   a["o"], a["ST"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                   a["C"], a["st"])

    assert call(B=-1) == binding.GDR_ERR_INVALID_ARG
    assert call(gate=7) == binding.GDR_ERR_INVALID_ARG
    assert call(dt=5) == binding.GDR_ERR_INVALID_ARG
    assert call(dk=48, dv=64) == binding.GDR_ERR_UNSUPPORTED
    assert call(C=32) == binding.GDR_ERR_UNSUPPORTED
    assert call(q=None) == binding.GDR_ERR_INVALID_ARG
    assert call(g=None) == binding.GDR_ERR_INVALID_ARG
    assert call(o=_fake_ptr(2)) == binding.GDR_ERR_INVALID_ARG
    assert call(H=0) == binding.GDR_OK


def test_prologue_validation_rejects_before_any_launch(L):
    """gdr_chunk_fwd_prologue: raw projections; the shapes gdr_chunk_fwd takes."""
    p = _fake_ptr()

    def call(**kw):
        a = dict(q=p, k=p, v=p, dt=1, a=p, gate=0, gs=p, b=p, S0=None, o=p, ST=None, B=2, T=300,
                 H=2, dk=128, dv=128, C=64, flags=3, st=None)
        a.update(kw)
        return L.gdr_chunk_fwd_prologue(a["q"], a["k"], a["v"], a["dt"], a["a"], a["gate"],
                                        a["gs"], a["b"], a["S0"], a["o"], a["ST"], a["B"], a["T"],
                                        a["H"], a["dk"], a["dv"], a["C"], a["flags"], a["st"])

    assert call(B=-1) == binding.GDR_ERR_INVALID_ARG
    assert call(flags=4) == binding.GDR_ERR_INVALID_ARG
    assert call(dt=5) == binding.GDR_ERR_INVALID_ARG
    assert call(gate=7) == binding.GDR_ERR_INVALID_ARG
    assert call(dk=48, dv=64) == binding.GDR_ERR_UNSUPPORTED
    assert call(C=32) == binding.GDR_ERR_UNSUPPORTED
    assert call(gs=None) == binding.GDR_ERR_INVALID_ARG
    assert call(b=None) == binding.GDR_ERR_INVALID_ARG
    assert call(q=None) == binding.GDR_ERR_INVALID_ARG
    assert call(H=0) == binding.GDR_OK


def test_backward_validation_rejects_before_any_launch(L):
    """gdr_chunk_bwd: square heads of 32, 64 or 128; workspace required."""
    p = _fake_ptr()
    # CUDA cores (fp32 inputs, or a per-channel gate): every 8th state + an 8-token stash
    ws = L.gdr_chunk_bwd_workspace_bytes(2, 300, 2, 128, 128, 0, 0)
    assert ws == 2 * 2 * (38 + 1 + 8) * 128 * 128 * 4
    assert L.gdr_chunk_bwd_workspace_bytes(2, 300, 2, 128, 128, 1, 1) == ws
    # tensor cores (bf16, d = 128, scalar gate): 104 KB of bf16 stash per chunk and head
    assert L.gdr_chunk_bwd_workspace_bytes(2, 300, 2, 128, 128, 1, 0) == 2 * 2 * 5 * 122880
    assert L.gdr_chunk_bwd_workspace_bytes(2, 300, 2, 128, 64, 1, 0) == 0

    def call(**kw):
        a = dict(q=p, k=p, v=p, dt=0, g=p, gate=0, beta=p, S0=None, do=p, dST=None, dq=p, dk=p,
                 dv=p, dg=p, db=p, dS0=None, B=2, T=300, H=2, dk_=128, dv_=128, ws=p, wsb=ws,
                 st=None)
        a.update(kw)
        return L.gdr_chunk_bwd(a["q"], a["k"], a["v"], a["dt"], a["g"], a["gate"], a["beta"],
                               a["S0"], a["do"], a["dST"], a["dq"], a["dk"], a["dv"], a["dg"],
                               a["db"], a["dS0"], a["B"], a["T"], a["H"], a["dk_"], a["dv_"],
                               a["ws"], a["wsb"], a["st"])

    assert call(B=-1) == binding.GDR_ERR_INVALID_ARG
    assert call(dt=5) == binding.GDR_ERR_INVALID_ARG
    assert call(gate=3) == binding.GDR_ERR_INVALID_ARG
    assert call(dk_=128, dv_=64) == binding.GDR_ERR_UNSUPPORTED
    assert call(dk_=96, dv_=96) == binding.GDR_ERR_UNSUPPORTED
    assert call(do=None) == binding.GDR_ERR_INVALID_ARG
    assert call(dg=None) == binding.GDR_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == binding.GDR_ERR_WORKSPACE
    assert call(ws=None) == binding.GDR_ERR_WORKSPACE
    assert call(ws=_fake_ptr(4)) == binding.GDR_ERR_INVALID_ARG
    assert call(H=0) == binding.GDR_OK


def test_dplr_validation_rejects_before_any_launch(L):
    p = _fake_ptr()

    def call(**kw):
        a = dict(q=p, k=p, v=p, a=p, b=p, dt=1, g=p, gate=0, S0=None, o=p, ST=None, B=2, T=100,
                 H=2, dk=64, dv=64, st=None)
        a.update(kw)
        return L.gdr_dplr_fwd(a["q"], a["k"], a["v"], a["a"], a["b"], a["dt"], a["g"], a["gate"],
                              a["S0"], a["o"], a["ST"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                              a["st"])

    assert call(T=-1) == binding.GDR_ERR_INVALID_ARG
    assert call(dt=7) == binding.GDR_ERR_INVALID_ARG
    assert call(gate=2) == binding.GDR_ERR_INVALID_ARG
    assert call(dk=64, dv=48) == binding.GDR_ERR_UNSUPPORTED
    assert call(dk=48, dv=48) == binding.GDR_ERR_UNSUPPORTED
    assert call(a=None) == binding.GDR_ERR_INVALID_ARG
    assert call(a=_fake_ptr(4)) == binding.GDR_ERR_INVALID_ARG
    assert call(S0=_fake_ptr(8)) == binding.GDR_ERR_INVALID_ARG
    assert call(b=None) == binding.GDR_ERR_INVALID_ARG
    assert call(B=0) == binding.GDR_OK


def test_every_binding_refuses_cpu_tensors(L):
    """No entry has a CPU path: each raises before reaching the library."""
    import torch

    x = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16)
    g = torch.zeros(1, 64, 1)
    calls = [
        lambda: binding.chunk_fwd_gla(x, x, x, g),
        lambda: binding.chunk_fwd_prologue(x, x, x, g, g, torch.ones(1)),
        lambda: binding.chunk_bwd(x, x, x, g, g, torch.zeros(1, 64, 1, 128)),
        lambda: binding.dplr_fwd(x, x, x, x, x, g),
        lambda: binding.chunk_fwd_segmented(x, x, x, g, g, segments=2,
                                            workspace=torch.zeros(16, dtype=torch.uint8)),
        lambda: binding.step(x[:, 0], x[:, 0], x[:, 0], g[:, 0], g[:, 0],
                             torch.zeros(1, 1, 128, 128)),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(ValueError, match="CUDA"):
            call()
