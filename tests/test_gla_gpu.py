"""GLA with a per-key-channel gate ("Efficient attention variants" §7.2) on the
GPU through the C ABI, against the float64 oracle: small cases element by
element (every head-size pair, both dtypes, ragged lengths, with and without
a start state), continuation from a state, and the bench workload at full
size on sampled chains over all their tokens."""
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
