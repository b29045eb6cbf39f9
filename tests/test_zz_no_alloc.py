"""la_prefill_noalloc: the tensor-core prefill for callers that cannot
allocate device memory while they run (for example a server that plans all
of its device memory up front, or a plugin host that offers no workspace).
It keeps its segment summaries in a fixed 16 MiB device array inside the
library instead of a caller workspace.

The GPU test calls the entry point through the C ABI, twice in a row, and
compares it with la_prefill (the same computation with a caller workspace)
within the tolerances the parity tests use.  This file is collected last so
a run that stops at the first failure has already run every other test; it
passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest

import causal_kernelized_linear_la_b200 as la
from causal_kernelized_linear_la_b200 import LaConfig, inputs
from tests import helpers as H


def _raw_noalloc(q, k, v, gamma, out, S_out, z_out, mode, eps=1e-6, stream=None):
    import torch
    B, Hh, N, d = q.shape
    dv = v.shape[-1]
    s = stream if stream is not None else torch.cuda.current_stream()
    cfg = LaConfig(la.LA_BF16, la.MODES[mode], eps, ctypes.c_void_p(s.cuda_stream), None, None, None, 0)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return la.lib().la_prefill_noalloc(p(q), p(k), p(v), p(gamma), None, p(out), p(S_out), p(z_out),
                                       B, Hh, N, d, dv, ctypes.byref(cfg))


def _usual_split(B, Hh, N, d, dv, chunk=64, max_seg=4096):
    """The segment split la_prefill picks (whole waves of resident CTAs,
    segments of at most 4096 tokens), restated to size the test cases."""
    chains = B * Hh
    sms = 2 * 148 if (d == 64 and dv == 64) else 148
    waves = 1
    while True:
        G = max(1, waves * sms // chains)
        L = -(-N // G)
        L = -(-L // chunk) * chunk
        if L <= max_seg or L <= chunk:
            break
        waves += 1
    L = max(L, 2 * chunk)
    return L, -(-N // L)


def test_full_decay_workload_needs_longer_segments():
    """The decay workload's usual split does not fit the fixed scratch, so the
    no-allocation call lengthens its segments (host arithmetic only)."""
    B, Hh, N, d, dv = 2, 16, 32768, 128, 128
    L, G = _usual_split(B, Hh, N, d, dv)
    gmax = (16 << 20) // (B * Hh * (d * dv + d) * 4)
    assert (L, G) == (3648, 9) and gmax == 7 and G > gmax


@pytest.mark.gpu
def test_noalloc_lengthened_segments_match_the_oracle():
    """The full decay workload (B=2, H=16, N=32768, d=dv=128) through the
    no-allocation entry point, whose segments are lengthened to fit: every
    output against la_prefill, and two chains against the float64 oracle."""
    import torch
    p = inputs.make_workload("decay_bf16")
    q, k, v = H.device_inputs(p)
    gamma = H.dev(p.gamma, torch)
    out = torch.full_like(v, float("nan"))
    S_out = torch.full((p.B, p.H, p.d, p.dv), float("nan"), device="cuda")
    z_out = torch.full((p.B, p.H, p.d), float("nan"), device="cuda")
    rc = _raw_noalloc(q, k, v, gamma, out, S_out, z_out, "decay", p.eps)
    assert rc == la.LA_OK, la.la_status_string(rc)
    la.la_prefill_check()
    got = (out.float().cpu().numpy().astype(np.float64), S_out.cpu().numpy().astype(np.float64),
           z_out.cpu().numpy().astype(np.float64))
    del out, S_out, z_out
    o_ref, S_ref, z_ref = la.la_prefill(q, k, v, mode="decay", gamma=gamma, eps=p.eps)
    la.la_prefill_check()
    assert H.rel_max(got[0], o_ref.float().cpu().numpy()) <= H.TOL_O["bf16"]
    assert H.rel_fro(got[1], S_ref.cpu().numpy()) <= H.TOL_STATE
    chains = [(0, 0), (1, 15)]
    H.assert_close(p, got, H.run_oracle(p, chains), chains)


@pytest.mark.gpu
def test_noalloc_gla_matches_la_prefill():
    """bf16 GLA keeps its segment summaries in the fixed scratch too; two calls
    in a row against la_prefill with a caller workspace."""
    import torch
    p = inputs.make_gla(2, 4, 1000, 128, 128, dtype="bf16", seed=34)
    q, k, v = H.device_inputs(p)
    al = H.dev(p.alpha, torch)
    o_ref, S_ref, _ = la.la_prefill(q, k, v, mode="gla", alpha=al)
    la.la_prefill_check()
    s = torch.cuda.current_stream()
    cfg = LaConfig(la.LA_BF16, la.MODES["gla"], 0.0, ctypes.c_void_p(s.cuda_stream), None, None, None, 0)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    for _ in range(2):
        out = torch.full_like(v, float("nan"))
        S_out = torch.full_like(S_ref, float("nan"))
        rc = la.lib().la_prefill_noalloc(ptr(q), ptr(k), ptr(v), ptr(al), None, ptr(out), ptr(S_out), None,
                                         p.B, p.H, p.N, p.d, p.dv, ctypes.byref(cfg))
        assert rc == la.LA_OK, la.la_status_string(rc)
        la.la_prefill_check()
        assert H.rel_max(out.float().cpu().numpy(), o_ref.float().cpu().numpy()) <= H.TOL_O["bf16"]
        assert H.rel_fro(S_out.cpu().numpy(), S_ref.cpu().numpy()) <= H.TOL_STATE


@pytest.mark.gpu
def test_noalloc_runs_workspace_free_paths_as_la_prefill():
    """fp32 inputs need no workspace: the no-allocation call runs them as
    la_prefill does, bit for bit."""
    import torch
    p = inputs.make_kernelized(1, 2, 300, 64, 64, dtype="f32", mode="decay", seed=33)
    q, k, v = H.device_inputs(p)
    gamma = H.dev(p.gamma, torch)
    o_ref, S_ref, z_ref = la.la_prefill(q, k, v, mode="decay", gamma=gamma, eps=p.eps)
    out, S_out, z_out = torch.empty_like(v), torch.empty_like(S_ref), torch.empty_like(z_ref)
    s = torch.cuda.current_stream()
    cfg = LaConfig(la.LA_F32, la.MODES["decay"], p.eps, ctypes.c_void_p(s.cuda_stream), None, None, None, 0)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = la.lib().la_prefill_noalloc(ptr(q), ptr(k), ptr(v), ptr(gamma), None, ptr(out), ptr(S_out), ptr(z_out),
                                     p.B, p.H, p.N, p.d, p.dv, ctypes.byref(cfg))
    assert rc == la.LA_OK, la.la_status_string(rc)
    la.la_prefill_check()
    assert torch.equal(out, o_ref) and torch.equal(S_out, S_ref) and torch.equal(z_out, z_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("name,mode,over", [("plain_bf16", "plain", {}),
                                            ("decay_bf16", "decay", {"B": 1, "N": 5000})])
def test_noalloc_matches_la_prefill_twice(name, mode, over):
    import torch
    p = inputs.make_workload(name, **over)
    q, k, v = H.device_inputs(p)
    gamma = H.dev(p.gamma, torch) if mode == "decay" else None
    o_ref, S_ref, z_ref = la.la_prefill(q, k, v, mode=mode, gamma=gamma, eps=p.eps)
    torch.cuda.synchronize()
    o_ref = o_ref.float().cpu().numpy()
    S_ref, z_ref = S_ref.cpu().numpy(), z_ref.cpu().numpy()
    for _ in range(2):
        out = torch.full_like(q[..., : v.shape[-1]], float("nan"))
        S_out = torch.full((p.B, p.H, p.d, p.dv), float("nan"), device="cuda")
        z_out = torch.full((p.B, p.H, p.d), float("nan"), device="cuda")
        rc = _raw_noalloc(q, k, v, gamma, out, S_out, z_out, mode, p.eps)
        assert rc == la.LA_OK, la.la_status_string(rc)
        la.la_prefill_check()
        o = out.float().cpu().numpy()
        assert H.rel_max(o, o_ref) <= H.TOL_O["bf16"]
        assert H.rel_fro(S_out.cpu().numpy(), S_ref) <= H.TOL_STATE
        assert H.rel_fro(z_out.cpu().numpy(), z_ref) <= H.TOL_STATE


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    """B*H*(d*dv + d)*4 bytes above 16 MiB cannot fit even one segment per
    chain: rejected before anything is launched (no GPU needed).  bf16 gated
    delta, whose workspace grows with N, has no fixed-size form."""
    cfg = LaConfig(la.LA_BF16, la.MODES["plain"], 1e-6, None, None, None, None, 0)
    fake = ctypes.c_void_p(0x10000)
    B, Hh, N, d, dv = 8, 32, 4096, 128, 128   # 256 chains x 66 KB > 16 MiB
    rc = la.lib().la_prefill_noalloc(fake, fake, fake, None, None, fake, fake, fake, B, Hh, N, d, dv,
                                     ctypes.byref(cfg))
    assert rc == la.LA_ERR_WORKSPACE
    cfgd = LaConfig(la.LA_BF16, la.MODES["gated_delta"], 1e-6, None, None, None, None, 0)
    rc = la.lib().la_prefill_noalloc(fake, fake, fake, fake, fake, fake, fake, None, 1, 1, 64, 64, 64,
                                     ctypes.byref(cfgd))
    assert rc == la.LA_ERR_UNSUPPORTED
