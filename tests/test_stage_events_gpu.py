"""The per-kernel timing hook (la_set_stage_events) on a GPU: each kernel of
a call records its event, the events complete in launch order, and turning
the hook off stops the recording.  Results of the call are unaffected."""
import numpy as np
import pytest
import torch

import causal_kernelized_linear_la_b200 as la
from causal_kernelized_linear_la_b200 import inputs

pytestmark = pytest.mark.gpu


def _dev(p):
    b = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return b(p.q_bits), b(p.k_bits), b(p.v_bits)


@pytest.mark.parametrize("name,nk", [("plain_bf16", 3), ("gdelta_bf16", 2), ("gla_bf16", 3)])
def test_stage_events_follow_the_kernels(name, nk):
    p = inputs.make_workload(name, B=1, H=2, N=512)
    q, k, v = _dev(p)
    kw = {}
    if p.mode == "gated_delta":
        kw = dict(alpha=torch.from_numpy(p.alpha).cuda(), g=torch.from_numpy(p.g).cuda())
    elif p.mode == "gla":
        kw = dict(alpha=torch.from_numpy(p.alpha).cuda())
    ref = la.la_prefill(q, k, v, mode=p.mode, **kw)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)]
    for e in [start] + marks:
        e.record(s)
    torch.cuda.synchronize()
    sentinel = marks[-1]                       # one more event than the call has kernels
    probe = torch.cuda.Event(enable_timing=True)
    try:
        la.la_set_stage_events(marks)
        start.record(s)
        got = la.la_prefill(q, k, v, mode=p.mode, **kw)
        probe.record(s)
        torch.cuda.synchronize()
    finally:
        la.la_set_stage_events(None)
    t = [start.elapsed_time(m) for m in marks[:nk]]
    assert all(x > 0 for x in t) and t == sorted(t)
    assert t[-1] <= start.elapsed_time(probe) + 1e-3
    # the sentinel was recorded before the call, not by it
    assert sentinel.elapsed_time(start) > 0
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
