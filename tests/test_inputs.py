"""Checks of the seeded input generators (no method arithmetic here)."""
import numpy as np
import torch

from causal_kernelized_linear_la_b200 import inputs


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 65504.0, 3e38], np.float32)]).astype(np.float32)
    bits, vals = inputs.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16)
    np.testing.assert_array_equal(bits, ref.view(torch.int16).numpy().view(np.uint16))
    np.testing.assert_array_equal(vals, ref.float().numpy())


def test_decay_gammas():
    g = inputs.decay_gammas(16)
    assert g.dtype == np.float32
    assert g[0] == np.float32(1 - 2 ** -5) and g[15] == np.float32(1 - 2 ** -8)
    assert np.all(np.diff(g) > 0)


def test_workloads_are_seeded_and_rounded():
    a = inputs.make_workload("plain_bf16", N=64)
    b = inputs.make_workload("plain_bf16", N=64)
    np.testing.assert_array_equal(a.q_bits, b.q_bits)
    assert a.q.dtype == np.float32 and a.q_bits.dtype == np.uint16
    assert abs(a.q.std() - 1 / 8) < 0.01
    f = inputs.make_workload("plain_f32")
    assert f.q_bits is None and f.q.shape == (1, 1, 256, 64)


def test_gated_delta_inputs():
    p = inputs.make_workload("gdelta_bf16", H=4, N=512)
    n = np.linalg.norm(p.k.astype(np.float64), axis=-1)
    assert np.all(np.abs(n - 1) < 1e-2)  # unit before bf16 rounding
    assert np.all((p.g > 0) & (p.g < 1)) and np.all((p.alpha > 0) & (p.alpha < 1))
    assert p.alpha.dtype == np.float32 and p.alpha.shape == (1, 4, 512)


def test_decode_token_regenerates():
    t1 = inputs.make_decode_token(7, Bs=4, H=2)
    t2 = inputs.make_decode_token(7, Bs=4, H=2)
    t3 = inputs.make_decode_token(8, Bs=4, H=2)
    np.testing.assert_array_equal(t1.q_bits, t2.q_bits)
    assert not np.array_equal(t1.q_bits, t3.q_bits)
    st = inputs.make_decode_state(Bs=4, H=2)
    assert np.all(st.z >= 1.0) and abs(st.S.std() - 0.1) < 0.02
