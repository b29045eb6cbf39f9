"""Run-to-run determinism of the tensor-core prefills: the same inputs give the
same bits on every call.  Every reduction in these kernels has a fixed order
(tensor-core K-steps, segment summaries combined in segment order), so a
difference between two calls can only come from a race between the warps of
a CTA or between kernels: a check that catches ordering bugs the tolerance of
a parity test can hide.  Workloads with many segments per chain, several
CTAs per SM and ragged chunk tails, each called five times; the first call
also runs against a workspace filled with garbage."""
import numpy as np
import pytest

from causal_kernelized_linear_la_b200 import inputs

pytestmark = pytest.mark.gpu


def _bf16(x, torch):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


CASES = [
    ("plain", 2, 8, 3000, 64, 64),
    ("decay", 1, 8, 5000, 128, 128),
    ("plain", 1, 4, 1111, 64, 128),
    ("gated_delta", 1, 4, 9000, 128, 128),
    ("gla", 1, 4, 2500, 128, 128),
]


@pytest.mark.parametrize("mode,B,H,N,d,dv", CASES)
def test_prefill_is_deterministic(mode, B, H, N, d, dv):
    import torch
    import causal_kernelized_linear_la_b200 as la
    if mode == "gated_delta":
        p = inputs.make_gated_delta(B, H, N, d, dv, dtype="bf16", seed=2000 + N)
    elif mode == "gla":
        p = inputs.make_gla(B, H, N, d, dv, dtype="bf16", seed=2000 + N)
    else:
        p = inputs.make_kernelized(B, H, N, d, dv, dtype="bf16", mode=mode, seed=2000 + N)
    q, k, v = _bf16(p.q_bits, torch), _bf16(p.k_bits, torch), _bf16(p.v_bits, torch)
    kw = {"mode": mode}
    if mode == "decay":
        kw["gamma"] = torch.from_numpy(p.gamma).cuda()
    if mode in ("gated_delta", "gla"):
        kw["alpha"] = torch.from_numpy(p.alpha).cuda()
    if mode == "gated_delta":
        kw["g"] = torch.from_numpy(p.g).cuda()
    nbytes = la.la_prefill_workspace_bytes(B, H, N, d, dv, "bf16", mode)
    ws = torch.full((max(nbytes, 16),), 0x7F, device="cuda", dtype=torch.uint8)   # garbage floats
    runs = []
    for r in range(5):
        o, S, z = la.la_prefill(q, k, v, workspace=ws, **kw)
        runs.append((o.clone(), S.clone(), None if z is None else z.clone()))
    torch.cuda.synchronize()
    la.la_prefill_check()
    o0, S0, z0 = runs[0]
    assert torch.isfinite(o0.float()).all() and torch.isfinite(S0).all()
    for r, (o, S, z) in enumerate(runs[1:], 1):
        assert torch.equal(o, o0), f"{mode}: o of call {r} differs from call 0"
        assert torch.equal(S, S0), f"{mode}: S of call {r} differs from call 0"
        if z is not None:
            assert torch.equal(z, z0), f"{mode}: z of call {r} differs from call 0"
