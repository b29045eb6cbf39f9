"""Float64 CPU oracle for causal kernelized linear attention.

TEST INFRASTRUCTURE ONLY.  The product path never imports this package; only
the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
(and its ``--impl reference`` arm) call it.  It shares no code with the CUDA
path: the arithmetic lives in ``la_oracle.c`` (plain C, float64, OpenMP over
independent chains), built here with gcc and loaded through ctypes.

Functions take host numpy arrays (any float dtype; converted to float64) and
return float64 arrays:

* ``kernelized(q, k, v, gamma=None, S0=None, z0=None, eps=1e-6, apply_phi=True)``
  -> ``(o, S, z)``: the write-then-read recurrence with normaliser
  ("What Is Linear Attention?" §4, §5.1; "Efficient attention variants" §5, §7.1).
* ``gated_delta(q, k, v, alpha, g, S0=None)`` -> ``(o, S)``
  ("Efficient attention variants" §7.4).
* ``decode_step(q, k, v, S, z, eps)`` -> ``(o, S, z)``: one application of the
  kernelized loop body (gamma = 1) to a given state and one token.
* ``gla(q, k, v, alpha, S0=None)`` -> ``(o, S)``: the per-key-channel gated
  recurrence ("Efficient attention variants" §7.2).
* ``causal_conv(x, w, cache=None)`` -> ``(y, cache_out)``: the short causal
  convolution with its conv cache ("What Is Linear Attention?" §5.4).

Parity status: every function is pinned by tests under ``tests/`` (none is
"parity unpinned").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB = os.path.join(_HERE, "liblaoracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile la_oracle.c into liblaoracle.so (gcc, -O2, OpenMP, IEEE math)."""
    stale = not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "la_oracle.h")))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                        "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        _bind(lib)
        _lib = lib
    return _lib


def _use_library(path):
    """Load a different build of la_oracle.c (the mutation tests use this to
    plant mistakes in a copy of the oracle); None restores the default."""
    global _lib
    _lib = None
    if path is not None:
        lib = ctypes.CDLL(path)
        _bind(lib)
        _lib = lib


def _bind(lib):
    P = ctypes.POINTER(ctypes.c_double)
    I = ctypes.c_int
    lib.la_oracle_kernelized.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, ctypes.c_double, I]
    lib.la_oracle_kernelized.restype = None
    lib.la_oracle_gated_delta.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I]
    lib.la_oracle_gated_delta.restype = None
    lib.la_oracle_gla.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I]
    lib.la_oracle_gla.restype = None
    lib.la_oracle_causal_conv.argtypes = [P, P, P, P, P, I, I, I, I, I]
    lib.la_oracle_causal_conv.restype = None
    lib.la_oracle_threads.argtypes = []
    lib.la_oracle_threads.restype = I


def threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return _load().la_oracle_threads()


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def kernelized(q, k, v, gamma=None, S0=None, z0=None, eps=1e-6, apply_phi=True):
    """q,k [B,H,N,d], v [B,H,N,dv] -> o [B,H,N,dv], S [B,H,d,dv], z [B,H,d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, N, d) and v.shape == (B, H, N, dv)
    gamma, S0, z0 = _f64(gamma), _f64(S0), _f64(z0)
    if gamma is not None:
        assert gamma.shape == (H,)
    if S0 is not None:
        assert S0.shape == (B, H, d, dv)
    if z0 is not None:
        assert z0.shape == (B, H, d)
    o = np.empty((B, H, N, dv))
    S = np.empty((B, H, d, dv))
    z = np.empty((B, H, d))
    _load().la_oracle_kernelized(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(S0), _ptr(z0),
                                 _ptr(o), _ptr(S), _ptr(z), B, H, N, d, dv, float(eps), int(bool(apply_phi)))
    return o, S, z


def gated_delta(q, k, v, alpha, g, S0=None):
    """q,k [B,H,N,d], v [B,H,N,dv], alpha,g [B,H,N] -> o [B,H,N,dv], S [B,H,d,dv]."""
    q, k, v, alpha, g, S0 = _f64(q), _f64(k), _f64(v), _f64(alpha), _f64(g), _f64(S0)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, N, d) and v.shape == (B, H, N, dv)
    assert alpha.shape == (B, H, N) and g.shape == (B, H, N)
    if S0 is not None:
        assert S0.shape == (B, H, d, dv)
    o = np.empty((B, H, N, dv))
    S = np.empty((B, H, d, dv))
    _load().la_oracle_gated_delta(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(g), _ptr(S0),
                                  _ptr(o), _ptr(S), B, H, N, d, dv)
    return o, S


def decode_step(q, k, v, S, z, eps=1e-6):
    """One decode step: q,k [Bs,H,d], v [Bs,H,dv], S [Bs,H,d,dv], z [Bs,H,d]
    -> (o [Bs,H,dv], S_new, z_new); the kernelized loop body with gamma = 1."""
    o, S1, z1 = kernelized(np.asarray(q)[:, :, None, :], np.asarray(k)[:, :, None, :],
                           np.asarray(v)[:, :, None, :], None, S, z, eps, True)
    return o[:, :, 0, :], S1, z1


def gated_delta_step(q, k, v, alpha, g, S):
    """One gated-delta decode step: q,k [Bs,H,d], v [Bs,H,dv], alpha,g [Bs,H]."""
    o, S1 = gated_delta(np.asarray(q)[:, :, None, :], np.asarray(k)[:, :, None, :],
                        np.asarray(v)[:, :, None, :], np.asarray(alpha)[:, :, None],
                        np.asarray(g)[:, :, None], S)
    return o[:, :, 0, :], S1


def gla(q, k, v, alpha, S0=None):
    """q,k,alpha [B,H,N,d], v [B,H,N,dv] -> o [B,H,N,dv], S [B,H,d,dv]."""
    q, k, v, alpha, S0 = _f64(q), _f64(k), _f64(v), _f64(alpha), _f64(S0)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, N, d) and alpha.shape == (B, H, N, d) and v.shape == (B, H, N, dv)
    if S0 is not None:
        assert S0.shape == (B, H, d, dv)
    o = np.empty((B, H, N, dv))
    S = np.empty((B, H, d, dv))
    _load().la_oracle_gla(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(S0), _ptr(o), _ptr(S), B, H, N, d, dv)
    return o, S


def causal_conv(x, w, cache=None):
    """x [B,H,N,d], w [H,d,W], cache [B,H,W-1,d] or None (zero history)
    -> (y [B,H,N,d], cache_out [B,H,W-1,d])."""
    x, w, cache = _f64(x), _f64(w), _f64(cache)
    B, H, N, d = x.shape
    W = w.shape[-1]
    assert w.shape == (H, d, W) and W >= 1
    if cache is not None:
        assert cache.shape == (B, H, W - 1, d)
    y = np.empty((B, H, N, d))
    cache_out = np.empty((B, H, W - 1, d))
    _load().la_oracle_causal_conv(_ptr(x), _ptr(w), _ptr(cache), _ptr(y), _ptr(cache_out) if W > 1 else None,
                                  B, H, N, d, W)
    return y, cache_out
