"""Thin Python binding of ``libgdr.so`` (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this
module checks tensor devices, dtypes, shapes and contiguity, then passes
raw device pointers and the current CUDA stream through ctypes.  There is no
CPU fallback: if the library is missing, or a tensor is not on a CUDA
device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdr.so")
_lib = None
_lock = threading.Lock()

GDR_OK, GDR_ERR_INVALID_ARG, GDR_ERR_UNSUPPORTED, GDR_ERR_WORKSPACE, GDR_ERR_CUDA, \
    GDR_ERR_TIMEOUT, GDR_ERR_RANGE = range(7)
GDR_F32, GDR_BF16 = 0, 1
GDR_GATE_SCALAR, GDR_GATE_PER_CHANNEL = 0, 1

EXPORTS = (
    "gdr_chunk_fwd_workspace_bytes",
    "gdr_chunk_fwd_kernel_launches",
    "gdr_chunk_fwd",
    "gdr_chunk_fwd_segmented",
    "gdr_chunk_fwd_segmented_noalloc",
    "gdr_chunk_fwd_varlen",
    "gdr_chunk_fwd_gla",
    "gdr_chunk_fwd_prologue",
    "gdr_chunk_bwd_workspace_bytes",
    "gdr_chunk_bwd",
    "gdr_dplr_fwd",
    "gdr_step",
    "gdr_get_device_status",
    "gdr_status_string",
    "gdr_last_error_message",
    "gdr_version",
    "gdr_testing_skip_stage_load",
)


class GdrError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{status_string(status)}: {msg}")
        self.status = status


def lib():
    """Load ``libgdr.so`` once; raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m gated_delta_rule_93_b200.build` (no CPU fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            L.gdr_chunk_fwd_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
            L.gdr_chunk_fwd_workspace_bytes.restype = sz
            L.gdr_chunk_fwd_kernel_launches.argtypes = [i, i, i, i, i, i, i, i]
            L.gdr_chunk_fwd_kernel_launches.restype = i
            L.gdr_chunk_fwd.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp, i, i, i, i, i, i,
                                        vp, sz, vp]
            L.gdr_chunk_fwd.restype = i
            L.gdr_chunk_fwd_segmented.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp, i, i, i, i,
                                                  i, i, i, vp, sz, vp]
            L.gdr_chunk_fwd_segmented.restype = i
            L.gdr_chunk_fwd_segmented_noalloc.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp,
                                                          i, i, i, i, i, i, i, vp]
            L.gdr_chunk_fwd_segmented_noalloc.restype = i
            L.gdr_chunk_fwd_varlen.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp, vp, i, i, i,
                                               i, i, i, vp]
            L.gdr_chunk_fwd_varlen.restype = i
            L.gdr_chunk_fwd_gla.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, i, i, i, i, i, i,
                                            vp]
            L.gdr_chunk_fwd_gla.restype = i
            L.gdr_chunk_fwd_prologue.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp, vp, i, i,
                                                 i, i, i, i, i, vp]
            L.gdr_chunk_fwd_prologue.restype = i
            L.gdr_chunk_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
            L.gdr_chunk_bwd_workspace_bytes.restype = sz
            L.gdr_chunk_bwd.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        vp, i, i, i, i, i, vp, sz, vp]
            L.gdr_chunk_bwd.restype = i
            L.gdr_dplr_fwd.argtypes = [vp, vp, vp, vp, vp, i, vp, i, vp, vp, vp, i, i, i, i, i,
                                       vp]
            L.gdr_dplr_fwd.restype = i
            L.gdr_step.argtypes = [vp, vp, vp, i, vp, i, vp, vp, vp, i, i, i, i, vp]
            L.gdr_step.restype = i
            L.gdr_get_device_status.argtypes = [vp]
            L.gdr_get_device_status.restype = i
            L.gdr_status_string.argtypes = [i]
            L.gdr_status_string.restype = ctypes.c_char_p
            L.gdr_last_error_message.argtypes = []
            L.gdr_last_error_message.restype = ctypes.c_char_p
            L.gdr_version.argtypes = []
            L.gdr_version.restype = i
            L.gdr_testing_skip_stage_load.argtypes = [i]
            L.gdr_testing_skip_stage_load.restype = i
            _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().gdr_status_string(int(s)).decode()


def _check(rc):
    if rc != GDR_OK:
        raise GdrError(rc, lib().gdr_last_error_message().decode())


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (no CPU path exists)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _in_dtype(dt):
    if dt == torch.bfloat16:
        return GDR_BF16
    if dt == torch.float32:
        return GDR_F32
    raise TypeError(f"q/k/v dtype must be bfloat16 or float32, got {dt}")


def chunk_fwd_workspace_bytes(B, T, H, dk, dv, C=64, dtype=torch.bfloat16, gate="scalar"):
    gk = GDR_GATE_PER_CHANNEL if gate == "channel" else GDR_GATE_SCALAR
    return int(lib().gdr_chunk_fwd_workspace_bytes(B, T, H, dk, dv, C, _in_dtype(dtype), gk))


def chunk_fwd_kernel_launches(B, T, H, dk, dv, C=64, dtype=torch.bfloat16, gate="scalar"):
    """Kernels one ``chunk_fwd`` call launches on the current device."""
    gk = GDR_GATE_PER_CHANNEL if gate == "channel" else GDR_GATE_SCALAR
    return int(lib().gdr_chunk_fwd_kernel_launches(B, T, H, dk, dv, C, _in_dtype(dtype), gk))


def chunk_fwd(q, k, v, g, beta, S0=None, *, output_final_state=True, o=None, S_T=None, C=64,
              workspace=None, stream=None):
    """Chunkwise forward, ``gdr_chunk_fwd``.  Returns (o, S_T or None).

    q, k [B,T,H,dk]; v [B,T,H,dv] (bf16 or fp32, one dtype); g [B,T,H] (scalar
    gate) or [B,T,H,dk] (per-channel gate) fp32 log alpha; beta [B,T,H] fp32;
    S0 [B,H,dv,dk] fp32 or None.
    """
    _need(q, "q")
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (B, T, H, dk), dev)
    _need(v, "v", dt, (B, T, H, dv), dev)
    if g.dim() == 4:
        _need(g, "g", torch.float32, (B, T, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (B, T, H), dev)
        gk = GDR_GATE_SCALAR
    _need(beta, "beta", torch.float32, (B, T, H), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _need(o, "o", dt, (B, T, H, dv), dev)
    if output_final_state and S_T is None:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dv, dk), dev)
    with torch.cuda.device(dev):
        # the segment rule depends on the SM count of q's device, which the
        # library reads from the current device
        ws = chunk_fwd_workspace_bytes(B, T, H, dk, dv, C, dt, "channel" if gk else "scalar")
        if ws and workspace is None:
            workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        rc = lib().gdr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(g), gk,
                                 _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, C,
                                 _ptr(workspace), workspace.numel() if workspace is not None
                                 else 0, _stream_handle(stream))
    _check(rc)
    return o, S_T


def step(q, k, v, g, beta, S, *, o=None, stream=None):
    """One decode step, ``gdr_step``: S [N,H,dv,dk] fp32 is updated in place.

    q, k [N,H,dk]; v [N,H,dv]; g [N,H] or [N,H,dk]; beta [N,H].  Returns o.
    """
    _need(q, "q")
    dev = q.device
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (N, H, dk), dev)
    _need(v, "v", dt, (N, H, dv), dev)
    if g.dim() == 3:
        _need(g, "g", torch.float32, (N, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (N, H), dev)
        gk = GDR_GATE_SCALAR
    _need(beta, "beta", torch.float32, (N, H), dev)
    _need(S, "S", torch.float32, (N, H, dv, dk), dev)
    if o is None:
        o = torch.empty((N, H, dv), dtype=dt, device=dev)
    _need(o, "o", dt, (N, H, dv), dev)
    with torch.cuda.device(dev):
        rc = lib().gdr_step(_ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(g), gk, _ptr(beta),
                            _ptr(S), _ptr(o), N, H, dk, dv, _stream_handle(stream))
    _check(rc)
    return o


def testing_skip_stage_load(chunk):
    """Test-only: the next tensor-core chunked forward on this thread skips the
    input load of `chunk`, so its bounded waits time out (see gdr_testing.h)."""
    _check(lib().gdr_testing_skip_stage_load(int(chunk)))


def device_status(stream=None):
    """Synchronise and read/clear the library's device status word (0 = OK)."""
    return int(lib().gdr_get_device_status(_stream_handle(stream)))


def chunk_fwd_segmented(q, k, v, g, beta, S0=None, *, segments, workspace,
                        output_final_state=True, o=None, S_T=None, C=64, stream=None):
    """``gdr_chunk_fwd_segmented``: the chunked forward as ``segments`` segments
    per sequence in the caller's ``workspace`` (a uint8 CUDA tensor of at least
    3*B*segments*H*dv*dk*4 bytes).  Returns (o, S_T or None)."""
    _need(q, "q")
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (B, T, H, dk), dev)
    _need(v, "v", dt, (B, T, H, dv), dev)
    if g.dim() == 4:
        _need(g, "g", torch.float32, (B, T, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (B, T, H), dev)
        gk = GDR_GATE_SCALAR
    _need(beta, "beta", torch.float32, (B, T, H), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    if not isinstance(workspace, torch.Tensor) or workspace.device != dev:
        raise ValueError("workspace must be a tensor on the inputs' device")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _need(o, "o", dt, (B, T, H, dv), dev)
    if output_final_state and S_T is None:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dv, dk), dev)
    with torch.cuda.device(dev):
        rc = lib().gdr_chunk_fwd_segmented(
            _ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(g), gk, _ptr(beta), _ptr(S0),
            _ptr(o), _ptr(S_T), B, T, H, dk, dv, C, int(segments), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check(rc)
    return o, S_T


# Bytes of the scratch array built into the library (GDR_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 24 * 1024 * 1024


def chunk_fwd_segmented_noalloc(q, k, v, g, beta, S0=None, *, segments, o, S_T=None, C=64,
                                stream=None):
    """``gdr_chunk_fwd_segmented_noalloc``: the segment path with its scratch in
    the library's fixed array, for callers that cannot allocate device memory
    while they run the mixer.  The caller passes every output (``o``, and
    ``S_T`` or None); nothing is allocated here or in the library.  Calls
    that overlap on the GPU race on the shared array.  Returns (o, S_T)."""
    _need(q, "q")
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (B, T, H, dk), dev)
    _need(v, "v", dt, (B, T, H, dv), dev)
    if g.dim() == 4:
        _need(g, "g", torch.float32, (B, T, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (B, T, H), dev)
        gk = GDR_GATE_SCALAR
    _need(beta, "beta", torch.float32, (B, T, H), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    _need(o, "o", dt, (B, T, H, dv), dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dv, dk), dev)
    with torch.cuda.device(dev):
        rc = lib().gdr_chunk_fwd_segmented_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(g), gk, _ptr(beta), _ptr(S0),
            _ptr(o), _ptr(S_T), B, T, H, dk, dv, C, int(segments), _stream_handle(stream))
    _check(rc)
    return o, S_T


def chunk_fwd_varlen(q, k, v, g, beta, cu_seqlens, S0=None, *, output_final_state=True, o=None,
                     S_T=None, C=64, stream=None):
    """``gdr_chunk_fwd_varlen``: N packed sequences of different lengths.

    q, k [total, H, dk]; v [total, H, dv] (bf16); g [total, H] or
    [total, H, dk] fp32; beta [total, H] fp32; cu_seqlens int32 CUDA tensor
    [N + 1] (sequence i = tokens cu_seqlens[i] .. cu_seqlens[i + 1] - 1);
    S0 [N, H, dv, dk] fp32 or None.  Returns (o [total, H, dv], S_T or None).
    """
    _need(q, "q")
    dev = q.device
    total, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (total, H, dk), dev)
    _need(v, "v", dt, (total, H, dv), dev)
    if g.dim() == 3:
        _need(g, "g", torch.float32, (total, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (total, H), dev)
        gk = GDR_GATE_SCALAR
    _need(beta, "beta", torch.float32, (total, H), dev)
    if not isinstance(cu_seqlens, torch.Tensor) or cu_seqlens.dtype != torch.int32 or \
            cu_seqlens.device != dev or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 tensor [N + 1] on the inputs' device")
    N = cu_seqlens.numel() - 1
    if S0 is not None:
        _need(S0, "S0", torch.float32, (N, H, dv, dk), dev)
    if o is None:
        o = torch.empty((total, H, dv), dtype=dt, device=dev)
    _need(o, "o", dt, (total, H, dv), dev)
    if output_final_state and S_T is None:
        S_T = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (N, H, dv, dk), dev)
    with torch.cuda.device(dev):
        rc = lib().gdr_chunk_fwd_varlen(
            _ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(g), gk, _ptr(beta), _ptr(cu_seqlens),
            _ptr(S0), _ptr(o), _ptr(S_T), N, total, H, dk, dv, C, _stream_handle(stream))
    _check(rc)
    return o, S_T


def chunk_fwd_gla(q, k, v, g, S0=None, *, output_final_state=True, o=None, S_T=None, C=64,
                  stream=None):
    """``gdr_chunk_fwd_gla``: gated linear attention, S_t = S_{t-1} Diag(alpha_t)
    + v_t k_t^T, o_t = S_t q_t (no beta).  q, k [B,T,H,dk]; v [B,T,H,dv] (bf16);
    g [B,T,H] or [B,T,H,dk] fp32 log alpha; S0 [B,H,dv,dk] fp32 or None.
    Returns (o, S_T or None)."""
    _need(q, "q")
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (B, T, H, dk), dev)
    _need(v, "v", dt, (B, T, H, dv), dev)
    if g.dim() == 4:
        _need(g, "g", torch.float32, (B, T, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (B, T, H), dev)
        gk = GDR_GATE_SCALAR
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _need(o, "o", dt, (B, T, H, dv), dev)
    if output_final_state and S_T is None:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dv, dk), dev)
    with torch.cuda.device(dev):
        rc = lib().gdr_chunk_fwd_gla(_ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(g), gk,
                                     _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, C,
                                     _stream_handle(stream))
    _check(rc)
    return o, S_T


def chunk_fwd_prologue(q, k, v, a, b, gate_scale, S0=None, *, norm_q=True, norm_k=True,
                       output_final_state=True, o=None, S_T=None, C=64, stream=None):
    """``gdr_chunk_fwd_prologue``: the chunked forward from raw projections.

    q, k [B,T,H,dk] (raw; bf16 or fp32); v [B,T,H,dv]; a [B,T,H] (scalar
    gate) or [B,T,H,dk] (per-channel gate) and b [B,T,H] fp32 gate and beta
    logits; gate_scale [H] fp32.  In the kernel: q, k L2-normalised (per the
    flags), beta = sigmoid(b), g = -gate_scale[h] softplus(a).
    Returns (o, S_T or None)."""
    _need(q, "q")
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (B, T, H, dk), dev)
    _need(v, "v", dt, (B, T, H, dv), dev)
    if a.dim() == 4:
        _need(a, "a", torch.float32, (B, T, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(a, "a", torch.float32, (B, T, H), dev)
        gk = GDR_GATE_SCALAR
    _need(b, "b", torch.float32, (B, T, H), dev)
    _need(gate_scale, "gate_scale", torch.float32, (H,), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _need(o, "o", dt, (B, T, H, dv), dev)
    if output_final_state and S_T is None:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dv, dk), dev)
    flags = (1 if norm_q else 0) | (2 if norm_k else 0)
    with torch.cuda.device(dev):
        rc = lib().gdr_chunk_fwd_prologue(_ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(a),
                                          gk, _ptr(gate_scale), _ptr(b), _ptr(S0),
                                          _ptr(o), _ptr(S_T), B, T, H, dk, dv, C, flags,
                                          _stream_handle(stream))
    _check(rc)
    return o, S_T


def chunk_bwd_workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16, gate="scalar"):
    """Workspace ``chunk_bwd`` needs for this shape, input dtype and gate kind."""
    gk = GDR_GATE_PER_CHANNEL if gate == "channel" else GDR_GATE_SCALAR
    return int(lib().gdr_chunk_bwd_workspace_bytes(B, T, H, dk, dv, _in_dtype(dtype), gk))


def chunk_bwd(q, k, v, g, beta, dout, S0=None, dS_T=None, *, want_dS0=True, workspace=None,
              out=None, stream=None):
    """``gdr_chunk_bwd``: gradients of the chunked forward.

    Inputs as ``chunk_fwd``; dout [B,T,H,dv] fp32; dS_T [B,H,dv,dk] fp32 or
    None.  Returns dict dq, dk, dv, dg, dbeta, dS0 (fp32; dS0 None unless
    want_dS0)."""
    _need(q, "q")
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    _need(k, "k", dt, (B, T, H, dk), dev)
    _need(v, "v", dt, (B, T, H, dv), dev)
    if g.dim() == 4:
        _need(g, "g", torch.float32, (B, T, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (B, T, H), dev)
        gk = GDR_GATE_SCALAR
    _need(beta, "beta", torch.float32, (B, T, H), dev)
    _need(dout, "dout", torch.float32, (B, T, H, dv), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    if dS_T is not None:
        _need(dS_T, "dS_T", torch.float32, (B, H, dv, dk), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    if out is None:  # (or the caller's preallocated dict of the same tensors)
        out = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
                   dv=torch.empty((B, T, H, dv), **f32), dg=torch.empty(tuple(g.shape), **f32),
                   dbeta=torch.empty((B, T, H), **f32),
                   dS0=torch.empty((B, H, dv, dk), **f32) if want_dS0 else None)
    for name, shape in (("dq", (B, T, H, dk)), ("dk", (B, T, H, dk)), ("dv", (B, T, H, dv)),
                        ("dg", tuple(g.shape)), ("dbeta", (B, T, H))):
        _need(out[name], name, torch.float32, shape, dev)
    if out.get("dS0") is not None:
        _need(out["dS0"], "dS0", torch.float32, (B, H, dv, dk), dev)
    ws = chunk_bwd_workspace_bytes(B, T, H, dk, dv, dt, "channel" if gk else "scalar")
    if workspace is None and ws:
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = lib().gdr_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _in_dtype(dt), _ptr(g), gk,
                                 _ptr(beta), _ptr(S0), _ptr(dout), _ptr(dS_T), _ptr(out["dq"]),
                                 _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                                 _ptr(out["dbeta"]), _ptr(out.get("dS0")), B, T, H, dk, dv,
                                 _ptr(workspace),
                                 workspace.numel() * workspace.element_size()
                                 if workspace is not None else 0, _stream_handle(stream))
    _check(rc)
    return out


def dplr_fwd(q, k, v, a, b, g, S0=None, *, output_final_state=True, o=None, S_T=None,
             stream=None):
    """``gdr_dplr_fwd``: S_t = S_{t-1}(Diag(alpha_t) + a_t b_t^T) + v_t k_t^T,
    o_t = S_t q_t.  q, k, a, b [B,T,H,d]; v [B,T,H,d] (one dtype); g [B,T,H]
    or [B,T,H,d] fp32; S0 [B,H,d,d] fp32 or None.  Returns (o, S_T or None)."""
    _need(q, "q")
    dev = q.device
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    for t_, n_ in ((k, "k"), (a, "a"), (b, "b")):
        _need(t_, n_, dt, (B, T, H, dk), dev)
    _need(v, "v", dt, (B, T, H, dv), dev)
    if g.dim() == 4:
        _need(g, "g", torch.float32, (B, T, H, dk), dev)
        gk = GDR_GATE_PER_CHANNEL
    else:
        _need(g, "g", torch.float32, (B, T, H), dev)
        gk = GDR_GATE_SCALAR
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _need(o, "o", dt, (B, T, H, dv), dev)
    if output_final_state and S_T is None:
        S_T = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dv, dk), dev)
    with torch.cuda.device(dev):
        rc = lib().gdr_dplr_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _in_dtype(dt),
                                _ptr(g), gk, _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv,
                                _stream_handle(stream))
    _check(rc)
    return o, S_T
