"""Causal kernelized linear attention for B200 (sm_100a).

Thin Python binding over the C ABI in ``include/la.h`` (``libla.so``, built
in-tree by ``causal_kernelized_linear_la_b200.build``).  This module only
marshals arguments: it checks devices, dtypes and shapes of torch tensors,
allocates outputs with torch, and passes raw device pointers and the current
CUDA stream to the library.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback.  If libla.so is
missing or no GPU is present, calls raise.

Entry points (same names as the C ABI):

* ``la_prefill(q, k, v, mode=..., gamma=..., alpha=..., g=..., S0=..., z0=..., eps=...)``
  -> ``(o, S, z)`` (``z`` is None in gated-delta mode)
* ``la_prefill_varlen(q, k, v, seq_lens, mode=..., ...)`` -> ``(o, S, z)`` for a
  right-padded batch of sequences of different lengths
* ``la_decode_step(q, k, v, S, z, eps=...)`` -> ``o``; S and z updated in place
* ``la_gated_delta_decode_step(q, k, v, alpha, g, S)`` -> ``o``; S updated in place
* ``la_prefill_workspace_bytes(...)``, ``la_prefill_kernel_count(...)``,
  ``la_prefill_varlen_workspace_bytes(...)``,
  ``la_status_string(code)``, ``lib()``
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libla.so")

LA_OK, LA_ERR_INVALID, LA_ERR_UNSUPPORTED, LA_ERR_ALIGN, LA_ERR_CUDA, LA_ERR_TIMEOUT, LA_ERR_WORKSPACE = range(7)
LA_F32, LA_BF16 = 0, 1
MODES = {"plain": 0, "decay": 1, "gated_delta": 2, "gla": 3}

# Symbols the library exports; the header include/la.h declares exactly these.
EXPORTS = ("la_prefill", "la_prefill_noalloc", "la_prefill_workspace_bytes", "la_prefill_kernel_count",
           "la_prefill_varlen",
           "la_prefill_varlen_workspace_bytes", "la_decode_step", "la_gated_delta_decode_step",
           "la_set_stage_events", "la_causal_conv", "la_selftest_wait_timeout",
           "la_prefill_check", "la_status_string", "la_version")


class LaConfig(ctypes.Structure):
    """Mirror of ``la_config`` in include/la.h."""
    _fields_ = [("dtype", ctypes.c_int), ("mode", ctypes.c_int), ("eps", ctypes.c_float),
                ("stream", ctypes.c_void_p), ("S0", ctypes.c_void_p), ("z0", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


class LaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {la_status_string(code)}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with causal_kernelized_linear_la_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, cfgp = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(LaConfig)
        L.la_prefill.argtypes = [vp] * 8 + [i] * 5 + [cfgp]
        L.la_prefill.restype = i
        L.la_prefill_noalloc.argtypes = [vp] * 8 + [i] * 5 + [cfgp]
        L.la_prefill_noalloc.restype = i
        L.la_prefill_workspace_bytes.argtypes = [i] * 5 + [cfgp]
        L.la_prefill_workspace_bytes.restype = ctypes.c_size_t
        L.la_prefill_kernel_count.argtypes = [i] * 5 + [cfgp]
        L.la_prefill_kernel_count.restype = i
        ip = ctypes.POINTER(ctypes.c_int)
        L.la_prefill_varlen.argtypes = [vp] * 8 + [ip] + [i] * 5 + [cfgp]
        L.la_prefill_varlen.restype = i
        L.la_prefill_varlen_workspace_bytes.argtypes = [ip] + [i] * 4 + [cfgp]
        L.la_prefill_varlen_workspace_bytes.restype = ctypes.c_size_t
        L.la_decode_step.argtypes = [vp] * 6 + [i] * 4 + [cfgp]
        L.la_decode_step.restype = i
        L.la_gated_delta_decode_step.argtypes = [vp] * 7 + [i] * 4 + [cfgp]
        L.la_gated_delta_decode_step.restype = i
        L.la_prefill_check.argtypes = [vp, vp]
        L.la_prefill_check.restype = i
        L.la_selftest_wait_timeout.argtypes = [vp]
        L.la_selftest_wait_timeout.restype = i
        L.la_causal_conv.argtypes = [vp] * 5 + [i] * 5 + [cfgp]
        L.la_causal_conv.restype = i
        L.la_set_stage_events.argtypes = [ctypes.POINTER(vp), i]
        L.la_set_stage_events.restype = i
        L.la_status_string.argtypes = [i]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_version.argtypes = []
        L.la_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def la_status_string(code: int) -> str:
    return lib().la_status_string(int(code)).decode()


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return LA_F32
    if t.dtype == torch.bfloat16:
        return LA_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _check_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (the library has no CPU path)")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")


def _stream_handle(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def la_prefill_workspace_bytes(B, H, N, d, dv, dtype="bf16", mode="plain") -> int:
    cfg = LaConfig(LA_BF16 if dtype == "bf16" else LA_F32, MODES[mode], 0.0, None, None, None, None, 0)
    return int(lib().la_prefill_workspace_bytes(B, H, N, d, dv, ctypes.byref(cfg)))


def la_prefill_kernel_count(B, H, N, d, dv, dtype="bf16", mode="plain") -> int:
    """Kernels one la_prefill call with these sizes launches (host-only)."""
    cfg = LaConfig(LA_BF16 if dtype == "bf16" else LA_F32, MODES[mode], 0.0, None, None, None, None, 0)
    return int(lib().la_prefill_kernel_count(B, H, N, d, dv, ctypes.byref(cfg)))


def la_prefill(q, k, v, mode="plain", gamma=None, alpha=None, g=None, S0=None, z0=None, eps=1e-6,
               out=None, S_out=None, z_out=None, workspace=None, stream=None):
    """Causal prefill over [B,H,N,*] tensors; returns ``(o, S_N, z_N)``.

    mode "plain" (gamma = 1), "decay" (gamma [H] fp32), "gated_delta"
    (alpha, g [B,H,N] fp32; k L2-normalised; returns z_N = None), or "gla"
    (alpha [B,H,N,d] fp32, the per-key-channel gate; returns z_N = None)."""
    torch = _torch()
    if mode not in MODES:
        raise ValueError(f"mode must be one of {list(MODES)}")
    B, H, N, d = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, N) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k must be [B,H,N,d] and v [B,H,N,dv], all of one dtype")
    delta = mode in ("gated_delta", "gla")   # the modes without a normaliser
    dev = q.device
    if out is None:
        out = torch.empty((B, H, N, dv), device=dev, dtype=q.dtype)
    if S_out is None:
        S_out = torch.empty((B, H, d, dv), device=dev, dtype=torch.float32)
    if not delta and z_out is None:
        z_out = torch.empty((B, H, d), device=dev, dtype=torch.float32)
    if delta:
        z_out = None
    first = alpha if delta else gamma
    for t in (first, g, S0, z0, S_out, z_out):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("gamma/alpha/g/S0/z0/S_out/z_out must be float32")
    _check_cuda(q, k, v, first, g, S0, z0, out, S_out, z_out, workspace)
    need = la_prefill_workspace_bytes(B, H, N, d, dv, "bf16" if q.dtype == torch.bfloat16 else "f32", mode)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    cfg = LaConfig(_dtype_code(q), MODES[mode], float(eps), _stream_handle(stream), _ptr(S0), _ptr(z0),
                   _ptr(workspace), ws_bytes)
    rc = lib().la_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(first), _ptr(g), _ptr(out), _ptr(S_out), _ptr(z_out),
                          B, H, N, d, dv, ctypes.byref(cfg))
    if rc != LA_OK:
        raise LaError(rc, "la_prefill")
    return out, S_out, z_out


def _host_lens(seq_lens):
    """The sequence lengths as a C int array (host memory)."""
    lens = [int(n) for n in (seq_lens.tolist() if hasattr(seq_lens, "tolist") else seq_lens)]
    return (ctypes.c_int * max(len(lens), 1))(*lens), len(lens)


def la_prefill_varlen_workspace_bytes(seq_lens, H, d, dv, dtype="bf16", mode="plain") -> int:
    arr, B = _host_lens(seq_lens)
    cfg = LaConfig(LA_BF16 if dtype == "bf16" else LA_F32, MODES[mode], 0.0, None, None, None, None, 0)
    return int(lib().la_prefill_varlen_workspace_bytes(arr, B, H, d, dv, ctypes.byref(cfg)))


def la_prefill_varlen(q, k, v, seq_lens, mode="plain", gamma=None, alpha=None, g=None, S0=None, z0=None,
                      eps=1e-6, out=None, S_out=None, z_out=None, workspace=None, stream=None):
    """Prefill of a right-padded batch: q, k [B,H,N,d], v [B,H,N,dv] with
    sequence b in rows 0..seq_lens[b]-1 (seq_lens: host ints).  Returns
    ``(o, S, z)`` with each sequence's final state; rows of o past a
    sequence's length are not written (uninitialised when o is allocated
    here).  Other arguments as in ``la_prefill``."""
    torch = _torch()
    if mode not in MODES:
        raise ValueError(f"mode must be one of {list(MODES)}")
    B, H, N, d = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, N) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k must be [B,H,N,d] and v [B,H,N,dv], all of one dtype")
    arr, nl = _host_lens(seq_lens)
    if nl != B:
        raise ValueError(f"seq_lens has {nl} entries for a batch of {B}")
    delta = mode in ("gated_delta", "gla")   # the modes without a normaliser
    dev = q.device
    if out is None:
        out = torch.empty((B, H, N, dv), device=dev, dtype=q.dtype)
    if S_out is None:
        S_out = torch.empty((B, H, d, dv), device=dev, dtype=torch.float32)
    if not delta and z_out is None:
        z_out = torch.empty((B, H, d), device=dev, dtype=torch.float32)
    if delta:
        z_out = None
    first = alpha if delta else gamma
    for t in (first, g, S0, z0, S_out, z_out):
        if t is not None and t.dtype != torch.float32:
            raise TypeError("gamma/alpha/g/S0/z0/S_out/z_out must be float32")
    _check_cuda(q, k, v, first, g, S0, z0, out, S_out, z_out, workspace)
    cfg = LaConfig(_dtype_code(q), MODES[mode], float(eps), _stream_handle(stream), _ptr(S0), _ptr(z0), None, 0)
    need = int(lib().la_prefill_varlen_workspace_bytes(arr, B, H, d, dv, ctypes.byref(cfg)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    cfg.workspace = _ptr(workspace)
    cfg.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().la_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(first), _ptr(g), _ptr(out), _ptr(S_out),
                                 _ptr(z_out), arr, B, H, N, d, dv, ctypes.byref(cfg))
    if rc != LA_OK:
        raise LaError(rc, "la_prefill_varlen")
    return out, S_out, z_out


def la_decode_step(q, k, v, S, z, eps=1e-6, out=None, stream=None):
    """One decode step; q,k [B,H,d], v [B,H,dv]; S [B,H,d,dv], z [B,H,d]
    (fp32, updated in place).  Returns o [B,H,dv]."""
    torch = _torch()
    B, H, d = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, dv), device=q.device, dtype=q.dtype)
    _check_cuda(q, k, v, S, z, out)
    cfg = LaConfig(_dtype_code(q), MODES["plain"], float(eps), _stream_handle(stream), None, None, None, 0)
    rc = lib().la_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(z), _ptr(out), B, H, d, dv,
                              ctypes.byref(cfg))
    if rc != LA_OK:
        raise LaError(rc, "la_decode_step")
    return out


def la_gated_delta_decode_step(q, k, v, alpha, g, S, out=None, stream=None):
    """One gated-delta decode step; alpha, g [B,H] fp32; S updated in place."""
    torch = _torch()
    B, H, d = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, dv), device=q.device, dtype=q.dtype)
    _check_cuda(q, k, v, alpha, g, S, out)
    cfg = LaConfig(_dtype_code(q), MODES["gated_delta"], 0.0, _stream_handle(stream), None, None, None, 0)
    rc = lib().la_gated_delta_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(g), _ptr(S), _ptr(out),
                                          B, H, d, dv, ctypes.byref(cfg))
    if rc != LA_OK:
        raise LaError(rc, "la_gated_delta_decode_step")
    return out


def la_causal_conv(x, weight, cache=None, out=None, cache_out=None, stream=None):
    """Short causal convolution with conv cache on device tensors.
    x [B,H,N,d] bf16/fp32, weight [H,d,w] fp32, cache [B,H,w-1,d] or None.
    Returns (out, cache_out); cache_out is allocated when not given."""
    if x.dim() != 4 or weight.dim() != 3:
        raise ValueError("x must be [B,H,N,d] and weight [H,d,w]")
    torch = _torch()
    B, H, N, d = x.shape
    w = weight.shape[-1]
    if weight.shape != (H, d, w) or weight.dtype != torch.float32:
        raise ValueError("weight must be fp32 [H,d,w]")
    dev = x.device
    if out is None:
        out = torch.empty_like(x)
    if cache_out is None and w > 1:
        cache_out = torch.empty((B, H, w - 1, d), device=dev, dtype=x.dtype)
    _check_cuda(x, weight, cache, out, cache_out)
    cfg = LaConfig(_dtype_code(x), 0, 0.0, _stream_handle(stream), None, None, None, 0)
    rc = lib().la_causal_conv(_ptr(x), _ptr(weight), _ptr(cache), _ptr(out), _ptr(cache_out),
                              B, H, N, d, w, ctypes.byref(cfg))
    if rc != LA_OK:
        raise LaError(rc, "la_causal_conv")
    return out, cache_out


def la_set_stage_events(events=None):
    """Profiling hook: record torch.cuda.Event events[i] after the i-th kernel
    of every later call (None or [] turns it off).  The events must have been
    recorded once (so that they exist) and stay alive while the hook is set."""
    events = list(events or [])
    arr = (ctypes.c_void_p * max(1, len(events)))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    rc = lib().la_set_stage_events(arr, len(events))
    if rc != LA_OK:
        raise LaError(rc, "la_set_stage_events")


def la_selftest_wait_timeout(stream=None):
    """Enqueue the bounded-wait failure self-test; the next la_prefill_check
    on the stream raises LaError with code LA_ERR_TIMEOUT."""
    rc = lib().la_selftest_wait_timeout(_stream_handle(stream))
    if rc != LA_OK:
        raise LaError(rc, "la_selftest_wait_timeout")


def la_prefill_check(workspace=None, stream=None):
    """Synchronise the stream and report device-side errors of the last prefill."""
    rc = lib().la_prefill_check(_ptr(workspace), _stream_handle(stream))
    if rc != LA_OK:
        raise LaError(rc, "la_prefill_check")
