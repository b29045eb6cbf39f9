"""Shared test plumbing: move seeded inputs to the GPU, run the library and
the oracle on the same numbers, and compare with the stated tolerances."""
import numpy as np

import oracle

TOL_O = {"f32": 1e-4, "bf16": 2e-2}  # max|do| / max|o_ref|
TOL_STATE = 1e-2                     # relative Frobenius error of S and z


def dev(t_np, torch, dtype=None):
    import torch as _t
    if t_np is None:
        return None
    if t_np.dtype == np.uint16:
        return _t.from_numpy(np.ascontiguousarray(t_np).view(np.int16)).view(_t.bfloat16).cuda()
    x = _t.from_numpy(np.ascontiguousarray(t_np)).cuda()
    return x if dtype is None else x.to(dtype)


def device_inputs(p):
    import torch
    if p.dtype == "bf16":
        q, k, v = dev(p.q_bits, torch), dev(p.k_bits, torch), dev(p.v_bits, torch)
    else:
        q, k, v = dev(p.q, torch), dev(p.k, torch), dev(p.v, torch)
    return q, k, v


def run_library(p, S0=None, z0=None):
    import torch
    import causal_kernelized_linear_la_b200 as la
    q, k, v = device_inputs(p)
    kw = {}
    if p.mode == "decay":
        kw["gamma"] = dev(p.gamma, torch)
    if p.mode == "gated_delta":
        kw["alpha"], kw["g"] = dev(p.alpha, torch), dev(p.g, torch)
    if p.mode == "gla":
        kw["alpha"] = dev(p.alpha, torch)
    o, S, z = la.la_prefill(q, k, v, mode=p.mode, eps=p.eps, S0=None if S0 is None else dev(S0, torch),
                            z0=None if z0 is None else dev(z0, torch), **kw)
    la.la_prefill_check()
    o = o.float().cpu().numpy().astype(np.float64)
    S = S.cpu().numpy().astype(np.float64)
    z = None if z is None else z.cpu().numpy().astype(np.float64)
    return o, S, z


def run_oracle(p, chains=None, S0=None, z0=None):
    """Oracle on all chains, or on a list of (b, h) pairs; returns arrays with
    a leading axis over the selected chains when `chains` is given."""
    sel = [(b, h) for b in range(p.B) for h in range(p.H)] if chains is None else chains
    outs = []
    for b, h in sel:
        sl = (slice(b, b + 1), slice(h, h + 1))
        s0 = None if S0 is None else S0[sl]
        if p.mode == "gated_delta":
            o, S = oracle.gated_delta(p.q[sl], p.k[sl], p.v[sl], p.alpha[sl], p.g[sl], s0)
            z = None
        elif p.mode == "gla":
            o, S = oracle.gla(p.q[sl], p.k[sl], p.v[sl], p.alpha[sl], s0)
            z = None
        else:
            gam = None if p.gamma is None else p.gamma[h:h + 1]
            o, S, z = oracle.kernelized(p.q[sl], p.k[sl], p.v[sl], gam, s0, None if z0 is None else z0[sl], p.eps)
        outs.append((o[0, 0], S[0, 0], None if z is None else z[0, 0]))
    return outs


def rel_max(a, ref):
    return float(np.max(np.abs(a - ref)) / max(np.max(np.abs(ref)), 1e-30))


def rel_fro(a, ref):
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-30))


def assert_close(p, got, ref_list, chains, tok=None):
    o, S, z = got
    tol = TOL_O[p.dtype]
    for (b, h), (o_r, S_r, z_r) in zip(chains, ref_list):
        og = o[b, h] if tok is None else o[b, h][tok]
        orf = o_r if tok is None else o_r[tok]
        e = rel_max(og, orf)
        assert e <= tol, f"o mismatch chain ({b},{h}): {e:.3e} > {tol}"
        es = rel_fro(S[b, h], S_r)
        assert es <= TOL_STATE, f"S mismatch chain ({b},{h}): {es:.3e}"
        if z_r is not None:
            ez = rel_fro(z[b, h], z_r)
            assert ez <= TOL_STATE, f"z mismatch chain ({b},{h}): {ez:.3e}"
