"""GLA with a per-key-channel gate ("Efficient attention variants" §7.2) on the
GPU through the C ABI, against the float64 oracle: small cases element by
element (every head-size pair, both dtypes, ragged lengths, with and without
a start state), continuation from a state, closed gates (alpha -> 0, a reset
of one channel), and the bench workload at full size on sampled chains over
all their tokens."""
import numpy as np
import pytest

from causal_kernelized_linear_la_b200 import inputs
from tests.helpers import assert_close, run_library, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("N", [1, 5, 37, 300])
def test_gla_small(dtype, d, dv, N):
    p = inputs.make_gla(2, 2, N, d, dv, dtype=dtype, seed=900 + N + d + dv)
    chains = [(b, h) for b in range(2) for h in range(2)]
    assert_close(p, run_library(p), run_oracle(p), chains)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gla_from_a_start_state(dtype):
    p = inputs.make_gla(1, 3, 100, 128, 64, dtype=dtype, seed=31)
    S0 = np.random.default_rng(5).standard_normal((1, 3, 128, 64)).astype(np.float32)
    chains = [(0, h) for h in range(3)]
    assert_close(p, run_library(p, S0=S0), run_oracle(p, S0=S0), chains)


def test_gla_workload_full_size_sampled_chains():
    p = inputs.make_workload("gla_bf16")
    chains = [(0, 0), (0, 17), (0, 31)]
    assert_close(p, run_library(p), run_oracle(p, chains), chains)


def _closed_gates(p, positions):
    """Close the gate (alpha = 1e-40) of some (token, channel) pairs: the
    channel's state row is reset there."""
    for h, t, i in positions:
        p.alpha[0, h, t, i] = np.float32(1e-40)
    return p


def test_gla_closed_gates():
    p = inputs.make_gla(1, 3, 400, 128, 128, dtype="bf16", seed=41)
    # one closed gate in a chunk, two in one chunk of one channel, and gates
    # on chunk borders
    _closed_gates(p, [(0, 10, 5), (0, 200, 5), (1, 70, 0), (1, 100, 0), (2, 63, 127), (2, 64, 127), (2, 128, 3)])
    chains = [(0, h) for h in range(3)]
    assert_close(p, run_library(p), run_oracle(p), chains)


def test_gla_closed_gates_at_chunk_start():
    """A closed gate on a chunk's first token and a second one later in the
    chunk: the chunk's midpoint log decay falls below -80, where e^R is no
    longer a normal float and the gate factors take their own exponentials."""
    p = inputs.make_gla(1, 2, 300, 128, 128, dtype="bf16", seed=47)
    _closed_gates(p, [(0, 64, 9), (0, 90, 9), (1, 128, 2), (1, 129, 2), (1, 192, 100), (1, 250, 100)])
    chains = [(0, h) for h in range(2)]
    assert_close(p, run_library(p), run_oracle(p), chains)


def test_gla_chunk_out_of_range_is_reported():
    """Three closed gates of one channel inside one 64-token chunk exceed the
    chunk form's factor range: reported as unsupported by la_prefill_check
    (no fault, no hang)."""
    import torch
    import causal_kernelized_linear_la_b200 as la
    from tests import helpers as H
    p = inputs.make_gla(1, 1, 128, 64, 64, dtype="bf16", seed=43)
    _closed_gates(p, [(0, 3, 7), (0, 20, 7), (0, 40, 7)])
    q, k, v = H.device_inputs(p)
    la.la_prefill(q, k, v, mode="gla", alpha=H.dev(p.alpha, torch))
    with pytest.raises(la.LaError) as ei:
        la.la_prefill_check()
    assert ei.value.code == la.LA_ERR_UNSUPPORTED
    la.la_prefill_check()
