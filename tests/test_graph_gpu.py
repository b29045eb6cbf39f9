"""The library's launches inside a CUDA graph: a prefill or a run of decode
steps captured once and replayed gives the same bits as the same calls run
eagerly, and a replay after new inputs are copied into the captured buffers
computes on the new inputs (the graph holds pointers, not values).  Every
kernel of a call, with its programmatic-dependent-launch edges, is captured;
the workspace is a buffer the caller owns, so the graph allocates nothing."""
import numpy as np
import pytest

from causal_kernelized_linear_la_b200 import inputs

pytestmark = pytest.mark.gpu


def _bf16(x, torch):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def _args(p, torch):
    q, k, v = _bf16(p.q_bits, torch), _bf16(p.k_bits, torch), _bf16(p.v_bits, torch)
    kw = {"mode": p.mode}
    if p.mode == "decay":
        kw["gamma"] = torch.from_numpy(p.gamma).cuda()
    if p.mode in ("gated_delta", "gla"):
        kw["alpha"] = torch.from_numpy(p.alpha).cuda()
    if p.mode == "gated_delta":
        kw["g"] = torch.from_numpy(p.g).cuda()
    return q, k, v, kw


@pytest.mark.parametrize("name", ["plain_bf16", "decay_bf16", "gdelta_bf16", "gla_bf16"])
def test_prefill_replays_in_a_cuda_graph(name):
    import torch
    import causal_kernelized_linear_la_b200 as la
    p = inputs.make_workload(name, B=1, H=4, N=1000)
    q, k, v, kw = _args(p, torch)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    ref = la.la_prefill(q, k, v, **kw)
    torch.cuda.synchronize()
    out = torch.empty_like(ref[0])
    S = torch.empty_like(ref[1])
    z = None if ref[2] is None else torch.empty_like(ref[2])
    ws = torch.empty(max(la.la_prefill_workspace_bytes(B, H, N, d, dv, "bf16", p.mode), 16), device="cuda",
                     dtype=torch.uint8)
    call = lambda: la.la_prefill(q, k, v, out=out, S_out=S, z_out=z, workspace=ws, **kw)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()                                    # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    out.zero_()
    S.zero_()
    graph.replay()
    torch.cuda.synchronize()
    la.la_prefill_check()
    assert torch.equal(out, ref[0]) and torch.equal(S, ref[1])
    if z is not None:
        assert torch.equal(z, ref[2])
    # new inputs in the captured buffers: the replay computes on them
    p2 = inputs.make_workload(name, B=1, H=4, N=1000, seed=4242)
    q2, k2, v2, kw2 = _args(p2, torch)
    ref2 = la.la_prefill(q2, k2, v2, **kw2)
    q.copy_(q2)
    k.copy_(k2)
    v.copy_(v2)
    for key in ("gamma", "alpha", "g"):
        if key in kw:
            kw[key].copy_(kw2[key])
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref2[0]) and torch.equal(S, ref2[1])


def test_decode_steps_replay_in_a_cuda_graph():
    import torch
    import causal_kernelized_linear_la_b200 as la
    nseq, H, d, steps = 8, 4, 128, 16
    g = torch.Generator(device="cpu").manual_seed(4343)
    S0 = (torch.randn((nseq, H, d, d), generator=g) * 0.1).cuda()
    z0 = (torch.randn((nseq, H, d), generator=g).abs() + 1).cuda()
    toks = [tuple((torch.randn((nseq, H, d), generator=g) / d ** 0.5).to(torch.bfloat16).cuda() for _ in range(3))
            for _ in range(steps)]
    # eager reference
    S, z = S0.clone(), z0.clone()
    ref = [la.la_decode_step(q, k, v, S, z).clone() for q, k, v in toks]
    torch.cuda.synchronize()
    # captured: the same steps, in place on the same state buffers
    S, z = S0.clone(), z0.clone()
    outs = [torch.empty_like(r) for r in ref]
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        Sw, zw = S0.clone(), z0.clone()
        la.la_decode_step(*toks[0], Sw, zw, out=torch.empty_like(ref[0]))   # warm-up
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(graph):
        for (q, k, v), o in zip(toks, outs):
            la.la_decode_step(q, k, v, S, z, out=o)
    S.copy_(S0)
    z.copy_(z0)
    graph.replay()
    torch.cuda.synchronize()
    for i, (o, r) in enumerate(zip(outs, ref)):
        assert torch.equal(o, r), f"step {i}"
