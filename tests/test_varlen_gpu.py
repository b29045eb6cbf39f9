"""GPU parity of la_prefill_varlen: a right-padded batch whose sequences have
different lengths ("Efficient attention variants" §10, closing remarks: real
batches carry padding and chunk boundaries that the single-sequence examples
leave out).

Every padding row of q, k, v (and alpha, g) is NaN or inf, so a kernel that
let one into a result would spread a non-finite value into that sequence's
outputs or state; out is pre-filled with a sentinel, and its padding rows
must still hold it afterwards.  Each sequence is checked against the oracle
over its own length, and against la_prefill on that sequence alone: bit for
bit where the batch runs one sequence at a time (the same kernels and segment
plan), within the oracle tolerance where the bf16 kernelized batch runs as one
launch set (its segment length is chosen for the whole batch).
"""
import numpy as np
import pytest

from causal_kernelized_linear_la_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


def _make(mode, dtype, B, H_, N, d, dv, seed):
    if mode == "gated_delta":
        return inputs.make_gated_delta(B, H_, N, d, dv, dtype=dtype, seed=seed)
    if mode == "gla":
        return inputs.make_gla(B, H_, N, d, dv, dtype=dtype, seed=seed)
    return inputs.make_kernelized(B, H_, N, d, dv, dtype=dtype, mode=mode, seed=seed)


def _device(p, lens, torch):
    """Device tensors with NaN, +inf or -inf in every padding row."""
    q, k, v = H.device_inputs(p)
    a = None if p.alpha is None else H.dev(p.alpha, torch)
    g = None if p.g is None else H.dev(p.g, torch)
    junk = (float("nan"), float("inf"), float("-inf"))
    for b, n in enumerate(lens):
        for t in (q, k, v, a, g):
            if t is not None:
                for r in range(n, t.shape[2]):
                    t[b, :, r] = junk[(r + b) % 3]
    return q, k, v, a, g


def _one_launch_set(mode, dtype, B):
    return dtype == "bf16" and mode in ("plain", "decay") and B <= 64


def _kw(p, a, g, torch):
    kw = {"mode": p.mode, "eps": p.eps}
    if p.mode == "decay":
        kw["gamma"] = H.dev(p.gamma, torch)
    if p.mode in ("gated_delta", "gla"):
        kw["alpha"] = a
    if p.mode == "gated_delta":
        kw["g"] = g
    return kw


def _oracle_seq(p, b, n, S0=None, z0=None):
    """Oracle results of every head of sequence b over its first n tokens."""
    import oracle
    sl = (slice(b, b + 1), slice(None), slice(0, n))
    s0 = None if S0 is None else S0[b:b + 1]
    z0_ = None if z0 is None else z0[b:b + 1]
    if p.mode == "gated_delta":
        o, S = oracle.gated_delta(p.q[sl], p.k[sl], p.v[sl], p.alpha[sl], p.g[sl], s0)
        return o[0], S[0], None
    if p.mode == "gla":
        o, S = oracle.gla(p.q[sl], p.k[sl], p.v[sl], p.alpha[sl], s0)
        return o[0], S[0], None
    o, S, z = oracle.kernelized(p.q[sl], p.k[sl], p.v[sl], p.gamma, s0, z0_, p.eps)
    return o[0], S[0], z[0]


def _check_seq(p, got, b, n, S0=None, z0=None):
    o, S, z = got
    o_r, S_r, z_r = _oracle_seq(p, b, n, S0, z0)
    tol = H.TOL_O[p.dtype]
    if n > 0:
        e = H.rel_max(o[b, :, :n], o_r)
        assert e <= tol, f"o mismatch, sequence {b} (length {n}): {e:.3e}"
    es = H.rel_fro(S[b], S_r)
    assert es <= H.TOL_STATE if n > 0 or S0 is not None else es == 0.0, f"S mismatch, sequence {b}: {es:.3e}"
    if z_r is not None:
        ez = H.rel_fro(z[b], z_r)
        assert ez <= H.TOL_STATE if n > 0 or z0 is not None else ez == 0.0, f"z mismatch, sequence {b}"


CASES = [
    # mode, dtype, d, dv, padded N, lengths (0, 1, chunk edges, ragged, full)
    ("plain", "bf16", 64, 64, 700, [700, 0, 65, 1, 300, 64]),
    ("decay", "bf16", 128, 128, 520, [129, 520, 0, 63, 400]),
    ("plain", "bf16", 64, 128, 300, [300, 17, 128]),
    ("gated_delta", "bf16", 128, 128, 400, [400, 1, 0, 130, 257]),
    ("gated_delta", "bf16", 64, 64, 200, [64, 200, 33]),
    ("plain", "f32", 64, 64, 160, [160, 5, 0, 64]),
    ("decay", "f32", 128, 128, 100, [31, 100]),
    ("gated_delta", "f32", 64, 64, 90, [90, 0, 45]),
    ("gla", "bf16", 128, 128, 150, [150, 2, 0, 77]),
    ("gla", "f32", 64, 64, 60, [13, 60]),
]


LARGE_CASES = [
    # 16 heads: the batch's 1,184 segments of 128 tokens are too many for one
    # wave, so the segment length grows to 1,408 tokens (not a power of two)
    ("decay", "bf16", 128, 128, 4096, [4096, 3000, 1, 0, 2049], 16),
    # 40 sequences of scattered lengths, two segments per SM
    ("plain", "bf16", 64, 64, 640, [(37 * i * i + 11 * i) % 641 for i in range(40)], 4),
    # 65 sequences: more than one launch set takes, one sequence at a time
    ("plain", "bf16", 64, 64, 80, [(7 * i) % 81 for i in range(65)], 1),
]


@pytest.mark.parametrize("mode,dtype,d,dv,N,lens", CASES)
def test_varlen_matches_oracle_and_solo_calls(mode, dtype, d, dv, N, lens):
    _run_case(mode, dtype, d, dv, N, lens, 3)


@pytest.mark.parametrize("mode,dtype,d,dv,N,lens,heads", LARGE_CASES)
def test_varlen_large_batches(mode, dtype, d, dv, N, lens, heads):
    _run_case(mode, dtype, d, dv, N, lens, heads)


def _run_case(mode, dtype, d, dv, N, lens, H_):
    import torch
    import causal_kernelized_linear_la_b200 as la
    B = len(lens)
    p = _make(mode, dtype, B, H_, N, d, dv, seed=1300 + N + d)
    q, k, v, a, g = _device(p, lens, torch)
    kw = _kw(p, a, g, torch)
    out = torch.full((B, H_, N, dv), SENTINEL, device="cuda", dtype=q.dtype)
    o, S, z = la.la_prefill_varlen(q, k, v, lens, out=out, **kw)
    la.la_prefill_check()
    o_h = o.float().cpu().numpy().astype(np.float64)
    S_h = S.cpu().numpy().astype(np.float64)
    z_h = None if z is None else z.cpu().numpy().astype(np.float64)
    for b, n in enumerate(lens):
        assert np.all(o_h[b, :, n:] == SENTINEL), f"padding rows of sequence {b} were written"
        assert np.all(np.isfinite(o_h[b, :, :n])) and np.all(np.isfinite(S_h[b])), f"sequence {b} read padding"
        _check_seq(p, (o_h, S_h, z_h), b, n)
    # each sequence alone through la_prefill
    exact = not _one_launch_set(mode, dtype, B)
    for b, n in enumerate(lens):
        sub = lambda t: None if t is None else t[b:b + 1, :, :n].contiguous()
        kw1 = dict(kw)
        if "alpha" in kw1:
            kw1["alpha"] = sub(a)
        if "g" in kw1:
            kw1["g"] = sub(g)
        o1, S1, z1 = la.la_prefill(sub(q), sub(k), sub(v), **kw1)
        if exact:
            assert torch.equal(o1[0], o[b, :, :n]), f"sequence {b}: o differs from the solo call"
            assert torch.equal(S1[0], S[b]), f"sequence {b}: S differs from the solo call"
            if z is not None:
                assert torch.equal(z1[0], z[b]), f"sequence {b}: z differs from the solo call"
            continue
        if n > 0:
            e = H.rel_max(o1[0].float().cpu().numpy(), o_h[b, :, :n])
            assert e <= H.TOL_O[dtype], f"sequence {b}: o differs from the solo call by {e:.3e}"
        es = H.rel_fro(S1[0].cpu().numpy(), S_h[b])
        assert es <= H.TOL_STATE, f"sequence {b}: S differs from the solo call by {es:.3e}"


@pytest.mark.parametrize("mode", ["plain", "decay", "gated_delta"])
def test_varlen_chunked_continuation(mode):
    """Chunked prefill of a mixed batch: each sequence's first part, then its
    second part from the returned states, equals the oracle over the whole
    sequence (parts of different lengths per sequence, some empty)."""
    import torch
    import causal_kernelized_linear_la_b200 as la
    first, total = [100, 0, 250, 64], [300, 90, 250, 200]
    B, H_, N, d = len(total), 2, max(total), 128
    p = _make(mode, "bf16", B, H_, N, d, d, seed=1400)
    q, k, v, a, g = H.device_inputs(p) + (None if p.alpha is None else H.dev(p.alpha, torch),
                                          None if p.g is None else H.dev(p.g, torch))
    kw = _kw(p, a, g, torch)
    o1, S1, z1 = la.la_prefill_varlen(q, k, v, first, **kw)
    # the second parts, moved to the start of each sequence's block
    second = [t - f for f, t in zip(first, total)]
    N2 = max(second)
    def shift(t):
        if t is None:
            return None
        s = torch.zeros((B, H_, N2) + tuple(t.shape[3:]), device="cuda", dtype=t.dtype)
        for b in range(B):
            s[b, :, :second[b]] = t[b, :, first[b]:total[b]]
        return s
    kw2 = dict(kw)
    if "alpha" in kw2:
        kw2["alpha"] = shift(a)
    if "g" in kw2:
        kw2["g"] = shift(g)
    o2, S2, z2 = la.la_prefill_varlen(shift(q), shift(k), shift(v), second, S0=S1,
                                      z0=None if z1 is None else z1, **kw2)
    la.la_prefill_check()
    o = np.zeros((B, H_, N, d))
    o1h, o2h = o1.float().cpu().numpy(), o2.float().cpu().numpy()
    for b in range(B):
        o[b, :, :first[b]] = o1h[b, :, :first[b]]
        o[b, :, first[b]:total[b]] = o2h[b, :, :second[b]]
    S = S2.cpu().numpy().astype(np.float64)
    z = None if z2 is None else z2.cpu().numpy().astype(np.float64)
    for b, n in enumerate(total):
        _check_seq(p, (o, S, z), b, n)
