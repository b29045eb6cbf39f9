"""Seeded synthetic inputs for causal kernelized linear attention.

This module is the one piece shared by the CPU oracle's tests and the CUDA
path's tests and benchmark.  It builds inputs only: it holds none of the
method's arithmetic (no feature map, no recurrence, no chunk algebra).

Workloads (all synthetic; the pages measure on no dataset):

* ``plain_f32``   1 sequence x 1 head, N=256, d=dv=64, fp32 q,k,v ~ N(0,1),
                  plain causal (gamma = 1), eps = 1e-6.
* ``plain_bf16``  B=4, H=8, N=4096, d=dv=64, q,k,v ~ N(0,1)/sqrt(d) rounded to
                  bf16, gamma = 1.
* ``decay_bf16``  B=2, H=16, N=32768, d=dv=128, q,k,v ~ N(0,1)/sqrt(d) in bf16,
                  per-head decay gamma_h = 1 - 2^(-5 - 3h/15), h = 0..15.
* ``decode``      256 sequences x 32 heads, d=dv=128, fp32 state
                  S ~ 0.1*N(0,1), z = |N(0,1)| + 1; each step one bf16 token
                  q,k,v ~ N(0,1)/sqrt(d) drawn from ``default_rng([seed, step])``.
* ``gdelta_bf16`` B=1, H=32, N=65536, d=dv=128, q,v ~ N(0,1) in bf16,
                  k ~ N(0,1) L2-normalised per token (fp32) then bf16,
                  g = sigmoid(N(0,1)), alpha = exp(-0.1*softplus(N(0,1))),
                  per head and token, fp32.

Rounding to bf16 is round-to-nearest-even, done here once; both the oracle and
the GPU consume the same rounded numbers, so input quantisation is never
counted as kernel error.  Scalars computed from a formula (gamma_h, g, alpha)
are evaluated in float64 and rounded to float32 once.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BASE_SEED = 42  # the seed of the pages' own verification program


def bf16_round(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 ``x`` to bfloat16 (round to nearest, ties to even).

    Returns ``(bits, values)``: the bf16 bit patterns as uint16 and the same
    numbers widened back to float32 (exact)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bits = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    values = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return bits, values


def decay_gammas(H: int) -> np.ndarray:
    """Per-head decay gamma_h = 1 - 2^(-5 - 3h/15), h = 0..H-1 (0-based),
    evaluated in float64 and rounded to float32 once."""
    h = np.arange(H, dtype=np.float64)
    return (1.0 - np.exp2(-5.0 - 3.0 * h / 15.0)).astype(np.float32)


@dataclasses.dataclass
class PrefillInputs:
    """Host-side inputs of one prefill call.

    ``q``/``k``: [B,H,N,d]; ``v``: [B,H,N,dv].  ``dtype`` is "f32" or "bf16".
    For bf16, ``*_bits`` hold the uint16 patterns the device receives and the
    float32 arrays hold the same (exactly representable) numbers.
    ``gamma`` [H] (decay mode), ``alpha``/``g`` [B,H,N] (gated delta) and
    ``alpha`` [B,H,N,d] (gla) are fp32.
    """
    name: str
    mode: str  # "plain" | "decay" | "gated_delta" | "gla"
    dtype: str  # "f32" | "bf16"
    B: int
    H: int
    N: int
    d: int
    dv: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_bits: np.ndarray | None = None
    k_bits: np.ndarray | None = None
    v_bits: np.ndarray | None = None
    gamma: np.ndarray | None = None
    alpha: np.ndarray | None = None
    g: np.ndarray | None = None
    eps: float = 1e-6

    @property
    def tokens(self) -> int:
        return self.B * self.N

    @property
    def token_heads(self) -> int:
        return self.B * self.H * self.N


def _normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def _finish(p: PrefillInputs) -> PrefillInputs:
    if p.dtype == "bf16":
        p.q_bits, p.q = bf16_round(p.q)
        p.k_bits, p.k = bf16_round(p.k)
        p.v_bits, p.v = bf16_round(p.v)
    return p


def make_kernelized(B, H, N, d, dv, *, dtype="bf16", mode="plain", seed=BASE_SEED,
                    scale=None, eps=1e-6, name="custom") -> PrefillInputs:
    """q,k,v ~ N(0,1)*scale (scale defaults to 1/sqrt(d) for bf16, 1 for f32);
    plain (gamma = 1) or per-head decay ``decay_gammas(H)``."""
    if scale is None:
        scale = 1.0 / math.sqrt(d) if dtype == "bf16" else 1.0
    rng = np.random.default_rng(seed)
    q = _normal(rng, (B, H, N, d), scale)
    k = _normal(rng, (B, H, N, d), scale)
    v = _normal(rng, (B, H, N, dv), scale)
    gamma = decay_gammas(H) if mode == "decay" else None
    return _finish(PrefillInputs(name, mode, dtype, B, H, N, d, dv, q, k, v, gamma=gamma, eps=eps))


def make_gated_delta(B, H, N, d, dv, *, dtype="bf16", seed=BASE_SEED, name="custom") -> PrefillInputs:
    """q,v ~ N(0,1); k ~ N(0,1) then L2-normalised per token in fp32;
    g = sigmoid(x), alpha = exp(-0.1*softplus(y)) with x,y ~ N(0,1) per (b,h,t),
    evaluated in float64 and rounded to float32 once."""
    rng = np.random.default_rng(seed)
    q = _normal(rng, (B, H, N, d))
    k = _normal(rng, (B, H, N, d))
    v = _normal(rng, (B, H, N, dv))
    k /= np.sqrt(np.sum(k.astype(np.float64) ** 2, axis=-1, keepdims=True)).astype(np.float32)
    x = rng.standard_normal((B, H, N)).astype(np.float64)
    y = rng.standard_normal((B, H, N)).astype(np.float64)
    g = (1.0 / (1.0 + np.exp(-x))).astype(np.float32)
    softplus = np.log1p(np.exp(-np.abs(y))) + np.maximum(y, 0.0)
    alpha = np.exp(-0.1 * softplus).astype(np.float32)
    return _finish(PrefillInputs(name, "gated_delta", dtype, B, H, N, d, dv, q, k, v, alpha=alpha, g=g))


def make_gla(B, H, N, d, dv, *, dtype="bf16", seed=BASE_SEED, name="custom") -> PrefillInputs:
    """q,v ~ N(0,1); k ~ N(0,1)/sqrt(d); per-key-channel gate
    alpha = exp(-0.1*softplus(y)) with y ~ N(0,1) per (b,h,t,channel),
    evaluated in float64 and rounded to float32 once."""
    rng = np.random.default_rng(seed)
    q = _normal(rng, (B, H, N, d))
    k = _normal(rng, (B, H, N, d), 1.0 / np.sqrt(d))
    v = _normal(rng, (B, H, N, dv))
    y = rng.standard_normal((B, H, N, d)).astype(np.float64)
    softplus = np.log1p(np.exp(-np.abs(y))) + np.maximum(y, 0.0)
    alpha = np.exp(-0.1 * softplus).astype(np.float32)
    return _finish(PrefillInputs(name, "gla", dtype, B, H, N, d, dv, q, k, v, alpha=alpha))


# The five named workloads, each with its own seed (base seed + index), and a
# sixth for the per-key-channel gate (not one of the five benchmark configs).
WORKLOADS = {
    "plain_f32": dict(kind="kernelized", B=1, H=1, N=256, d=64, dv=64, dtype="f32", mode="plain", seed=BASE_SEED + 1),
    "plain_bf16": dict(kind="kernelized", B=4, H=8, N=4096, d=64, dv=64, dtype="bf16", mode="plain", seed=BASE_SEED + 2),
    "decay_bf16": dict(kind="kernelized", B=2, H=16, N=32768, d=128, dv=128, dtype="bf16", mode="decay", seed=BASE_SEED + 3),
    "decode": dict(kind="decode", S=256, H=32, d=128, dv=128, steps=1000, seed=BASE_SEED + 4),
    "gdelta_bf16": dict(kind="gated_delta", B=1, H=32, N=65536, d=128, dv=128, dtype="bf16", seed=BASE_SEED + 5),
    "gla_bf16": dict(kind="gla", B=1, H=32, N=8192, d=128, dv=128, dtype="bf16", seed=BASE_SEED + 6),
    "gdelta_decode": dict(kind="decode_gated_delta", S=256, H=32, d=128, dv=128, steps=1000, seed=BASE_SEED + 7),
}


def make_workload(name: str, **override) -> PrefillInputs:
    """Build one of the named prefill workloads; keyword overrides (e.g. N)
    shrink it for quick tests while keeping the recipe and seed."""
    spec = dict(WORKLOADS[name])
    spec.update(override)
    kind = spec.pop("kind")
    if kind == "kernelized":
        return make_kernelized(spec["B"], spec["H"], spec["N"], spec["d"], spec["dv"], dtype=spec["dtype"],
                               mode=spec["mode"], seed=spec["seed"], name=name)
    if kind == "gated_delta":
        return make_gated_delta(spec["B"], spec["H"], spec["N"], spec["d"], spec["dv"], dtype=spec["dtype"],
                                seed=spec["seed"], name=name)
    if kind == "gla":
        return make_gla(spec["B"], spec["H"], spec["N"], spec["d"], spec["dv"], dtype=spec["dtype"],
                        seed=spec["seed"], name=name)
    raise ValueError(f"{name} is not a prefill workload")


@dataclasses.dataclass
class DecodeState:
    """Initial decode state: S [Bs,H,d,dv] fp32 ~ 0.1*N(0,1), z [Bs,H,d] = |N(0,1)|+1."""
    S: np.ndarray
    z: np.ndarray


def make_decode_state(Bs=256, H=32, d=128, dv=128, seed=BASE_SEED + 4) -> DecodeState:
    rng = np.random.default_rng(seed)
    S = _normal(rng, (Bs, H, d, dv), 0.1)
    z = np.abs(rng.standard_normal((Bs, H, d), dtype=np.float32)) + np.float32(1.0)
    return DecodeState(S, z)


@dataclasses.dataclass
class DecodeToken:
    """One decode token per (sequence, head): q,k [Bs,H,d], v [Bs,H,dv] in bf16."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_bits: np.ndarray
    k_bits: np.ndarray
    v_bits: np.ndarray


def make_decode_token(step: int, Bs=256, H=32, d=128, dv=128, seed=BASE_SEED + 4) -> DecodeToken:
    """Token of decode step ``step`` from ``default_rng([seed, step])``, so any
    step can be regenerated without storing the chain."""
    rng = np.random.default_rng([seed, step])
    s = 1.0 / math.sqrt(d)
    qb, q = bf16_round(_normal(rng, (Bs, H, d), s))
    kb, k = bf16_round(_normal(rng, (Bs, H, d), s))
    vb, v = bf16_round(_normal(rng, (Bs, H, dv), s))
    return DecodeToken(q, k, v, qb, kb, vb)


@dataclasses.dataclass
class GatedDeltaDecodeToken:
    """One gated-delta decode token per (sequence, head): q,k [Bs,H,d],
    v [Bs,H,dv] in bf16 (k L2-normalised), alpha, g [Bs,H] fp32."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_bits: np.ndarray
    k_bits: np.ndarray
    v_bits: np.ndarray
    alpha: np.ndarray
    g: np.ndarray


def make_gated_delta_decode_token(step: int, Bs=256, H=32, d=128, dv=128,
                                  seed=BASE_SEED + 7) -> GatedDeltaDecodeToken:
    """Token of gated-delta decode step ``step`` from ``default_rng([seed, step])``,
    drawn like the gated-delta prefill workload's tokens: q, v ~ N(0,1), k ~ N(0,1)
    L2-normalised in fp32, g = sigmoid(x), alpha = exp(-0.1*softplus(y))."""
    rng = np.random.default_rng([seed, step])
    q = _normal(rng, (Bs, H, d))
    k = _normal(rng, (Bs, H, d))
    v = _normal(rng, (Bs, H, dv))
    k /= np.sqrt(np.sum(k.astype(np.float64) ** 2, axis=-1, keepdims=True)).astype(np.float32)
    x = rng.standard_normal((Bs, H)).astype(np.float64)
    y = rng.standard_normal((Bs, H)).astype(np.float64)
    g = (1.0 / (1.0 + np.exp(-x))).astype(np.float32)
    softplus = np.log1p(np.exp(-np.abs(y))) + np.maximum(y, 0.0)
    alpha = np.exp(-0.1 * softplus).astype(np.float32)
    qb, q = bf16_round(q)
    kb, k = bf16_round(k)
    vb, v = bf16_round(v)
    return GatedDeltaDecodeToken(q, k, v, qb, kb, vb, alpha, g)
