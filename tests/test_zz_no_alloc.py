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
    chain: rejected before anything is launched (no GPU needed)."""
    cfg = LaConfig(la.LA_BF16, la.MODES["plain"], 1e-6, None, None, None, None, 0)
    fake = ctypes.c_void_p(0x10000)
    B, Hh, N, d, dv = 8, 32, 4096, 128, 128   # 256 chains x 66 KB > 16 MiB
    rc = la.lib().la_prefill_noalloc(fake, fake, fake, None, None, fake, fake, fake, B, Hh, N, d, dv,
                                     ctypes.byref(cfg))
    assert rc == la.LA_ERR_WORKSPACE
    cfg32 = LaConfig(la.LA_F32, la.MODES["plain"], 1e-6, None, None, None, None, 0)
    rc = la.lib().la_prefill_noalloc(fake, fake, fake, None, None, fake, fake, fake, 1, 1, 64, 64, 64,
                                     ctypes.byref(cfg32))
    assert rc == la.LA_ERR_UNSUPPORTED
