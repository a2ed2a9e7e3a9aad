"""The backward with a cached reference plan against the float64 oracle.

The staircase vectors of the R-step adjoint are banded matrix-vector products with the one
reference plan P(R,R) ("Blockwise Differentiable Sinkhorn Attention" §2.2).  The default backward
recomputes the plan in every sweep; the cached schedule stores it once (bf16 band store, written
by the alpha_R sweep) and streams it in the staircase sweeps.  Both must match the oracle within
the bf16 tolerance; problems the cached form does not cover (half-width not a multiple of 128,
a dustbin) run the default and stay exact."""
import numpy as np
import pytest

import eot_inputs
from harness import TOL, compare, gpu_run, oracle_run

pytestmark = pytest.mark.gpu


def _ragged(B, L, seed):
    rng = np.random.default_rng(seed)
    m = np.zeros((B, L), np.uint8)
    for b in range(B):
        n = int(rng.integers(L // 2, L + 1))
        m[b, :n] = 1
        m[b, rng.choice(n, size=max(1, n // 40), replace=False)] = 0
    return m


CASES = {
    "d64_W256_R2_ragged": lambda: eot_inputs.dense_case(2, 2, 1024, 64, 256, 5, 2, "bf16", seed=61,
                                                        mask=_ragged(2, 1024, 61), name="c_d64_W256"),
    "d128_W512_R3": lambda: eot_inputs.dense_case(1, 2, 1536, 128, 512, 4, 3, "bf16", seed=62, name="c_d128_W512_R3"),
    "d128_W1024_R2_long_init": lambda: eot_inputs.dense_case(1, 2, 2048, 128, 1024, 4, 2, "bf16", seed=63,
                                                             std=128 ** -0.5, name="c_d128_W1024"),
    "d64_W0_R2": lambda: eot_inputs.dense_case(1, 2, 512, 64, 0, 3, 2, "bf16", seed=64, name="c_W0"),
    "not_covered_W100": lambda: eot_inputs.dense_case(1, 2, 512, 64, 100, 4, 2, "bf16", seed=65, name="c_W100"),
    "not_covered_dustbin": lambda: eot_inputs.dustbin_case(1, 2, 300, 64, 256, 4, 2, "bf16", seed=66, mass=0.1,
                                                           name="c_dustbin"),
}


@pytest.fixture
def cached():
    from entropic_ot_attention_b200 import _abi
    _abi.eot_set_backward_schedule(1)
    yield
    _abi.eot_set_backward_schedule(0)


@pytest.mark.parametrize("name", sorted(CASES))
def test_cached_plan_backward_parity(name, cached):
    case = CASES[name]()
    errs = compare(gpu_run(case), oracle_run(case))
    assert all(e <= TOL[case.dtype] for e in errs.values()), f"{name}: {errs}"


def test_cached_plan_workspace_and_agreement(cached):
    """The band store is part of the backward workspace only under the cached schedule, and the
    cached and recomputed staircases agree to rounding."""
    import torch
    from entropic_ot_attention_b200 import _abi, api
    case = CASES["d128_W512_R3"]()
    B, H, L, d = case.Q.shape
    p = api.make_problem(B, H, L, d, case.W, case.T, case.R, torch.bfloat16)
    with_cache = _abi.eot_workspace_bytes(p, True)
    a = gpu_run(case)
    _abi.eot_set_backward_schedule(0)
    without = _abi.eot_workspace_bytes(p, True)
    b = gpu_run(case)
    # the recompute schedule holds the split alpha_R sweep's partial sums instead: 4 (2 E + 1)
    # slots and their total, E = ceil(h / 128), one 256-byte-aligned [B H L] fp32 vector each
    vec = (B * H * L * 4 + 255) // 256 * 256
    E = (case.W // 2 + 127) // 128
    split = (4 * (2 * E + 1) + 1) * vec
    assert with_cache - without >= B * H * L * (case.W + 128) * 2 - split
    assert with_cache - without <= B * H * L * (case.W + 128) * 2 + 256
    errs = compare(a, b, keys=("dQ", "dK", "dV"))
    assert all(e <= 1.2e-2 for e in errs.values()), errs
