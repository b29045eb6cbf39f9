"""Short causal convolution with conv cache ("What Is Linear Attention?" §5.4)
on the GPU through the C ABI, against the float64 oracle: element by element
at small sizes spanning several token tiles with ragged tails, every filter
width 1..8, both head sizes and dtypes, with and without a cache; bit-exact
continuation through the cache; the degenerate sizes."""
import numpy as np
import pytest
import torch

import causal_kernelized_linear_la_b200 as la
import oracle

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}   # max|dy| / max|y|, as for prefill outputs


def _inputs(B, H, N, d, w, dtype, seed, cache=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, N, d), dtype=np.float32)
    c = rng.standard_normal((B, H, max(w - 1, 0), d), dtype=np.float32) if cache else None
    wt = (rng.standard_normal((H, d, w), dtype=np.float32) / np.sqrt(w)).astype(np.float32)
    xt = torch.from_numpy(x).to(dtype)
    ct = None if c is None else torch.from_numpy(c).to(dtype)
    # the oracle consumes exactly the rounded inputs the GPU sees
    x64 = xt.float().numpy().astype(np.float64)
    c64 = None if ct is None else ct.float().numpy().astype(np.float64)
    return xt, ct, torch.from_numpy(wt), x64, c64, wt.astype(np.float64)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("w", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("N,cache", [(1, True), (7, False), (300, True), (1000, False)])
def test_conv_matches_oracle(dtype, d, w, N, cache):
    xt, ct, wt, x64, c64, w64 = _inputs(2, 3, N, d, w, dtype, seed=N * 10 + w, cache=cache)
    y, c_out = la.la_causal_conv(xt.cuda(), wt.cuda(), None if ct is None or w == 1 else ct.cuda())
    torch.cuda.synchronize()
    y_ref, c_ref = oracle.causal_conv(x64, w64, c64 if w > 1 else None)
    yg = y.float().cpu().numpy()
    err = np.abs(yg - y_ref).max() / max(np.abs(y_ref).max(), 1e-30)
    assert err <= TOL[dtype], err
    if w > 1:
        # the cache is a copy of inputs: bit-exact
        assert np.array_equal(c_out.float().cpu().numpy(), c_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_conv_cache_continuation_is_bit_exact(dtype):
    xt, ct, wt, *_ = _inputs(2, 2, 777, 128, 4, dtype, seed=3)
    x, c0, w = xt.cuda(), ct.cuda(), wt.cuda()
    y_all, c_all = la.la_causal_conv(x, w, c0)
    ya, ca = la.la_causal_conv(x[:, :, :300].contiguous(), w, c0)
    yb, cb = la.la_causal_conv(x[:, :, 300:301].contiguous(), w, ca)
    yc, cc = la.la_causal_conv(x[:, :, 301:].contiguous(), w, cb)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([ya, yb, yc], dim=2), y_all)
    assert torch.equal(cc, c_all)


def test_conv_degenerate_sizes():
    xt, ct, wt, x64, c64, w64 = _inputs(1, 2, 2, 64, 5, torch.bfloat16, seed=4)
    c0 = ct.cuda()
    # N = 0 moves the cache only
    empty = torch.empty((1, 2, 0, 64), device="cuda", dtype=torch.bfloat16)
    _, c_out = la.la_causal_conv(empty, wt.cuda(), c0)
    torch.cuda.synchronize()
    assert torch.equal(c_out, c0)
    # N < w - 1 keeps the older cache rows, shifted
    _, c_out = la.la_causal_conv(xt.cuda(), wt.cuda(), c0)
    torch.cuda.synchronize()
    _, c_ref = oracle.causal_conv(x64, w64, c64)
    assert np.array_equal(c_out.float().cpu().numpy(), c_ref)
    # B*H = 0 launches nothing and succeeds
    z = torch.empty((0, 2, 5, 64), device="cuda", dtype=torch.bfloat16)
    la.la_causal_conv(z, wt.cuda(), None, cache_out=torch.empty((0, 2, 4, 64), device="cuda", dtype=torch.bfloat16))


def test_conv_rejects_bad_arguments():
    x = torch.zeros((1, 1, 8, 64), device="cuda", dtype=torch.bfloat16)
    w = torch.zeros((1, 64, 4), device="cuda", dtype=torch.float32)
    c = torch.zeros((1, 1, 3, 64), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(la.LaError):                     # cache_out overlapping cache
        la.la_causal_conv(x, w, c, cache_out=c)
    with pytest.raises(la.LaError):                     # w > 8
        la.la_causal_conv(x, torch.zeros((1, 64, 9), device="cuda"), None)
    with pytest.raises(la.LaError):                     # head size
        la.la_causal_conv(torch.zeros((1, 1, 8, 32), device="cuda", dtype=torch.bfloat16),
                          torch.zeros((1, 32, 4), device="cuda"), None)
