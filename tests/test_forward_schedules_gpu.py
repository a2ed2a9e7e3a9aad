"""Both forward schedules against the float64 oracle.

The one-exponential schedule forms the plan entries E = exp(S + u + v) of a 128-row strip once
per Sinkhorn iteration, takes their row sums in registers and the column sums (a/r)^T E on the
tensor core from E kept in shared memory ("Blockwise Differentiable Sinkhorn Attention" §2.1
steps, with §2.2's orbit identity applied forward).  It runs with one CTA per strip (windows of
up to 3 tiles at d = 128, 5 at d = 64) or a CTA pair sharing each strip (up to 9 tiles), in one
cooperative launch or one launch per iteration.  The half-step schedule forms the entries once
per half-step.  Every variant is compared with the oracle element by element (bf16 tolerance
2e-2 on O, u, v, dQ, dK, dV) on cases that cover each form, ragged masks, odd band widths, W = 0,
T = 1, R = 0 and R = 4."""
import numpy as np
import pytest

import eot_inputs
from harness import TOL, compare, gpu_run, oracle_run

pytestmark = pytest.mark.gpu

SCHEDULES = {"one_exp": 2, "one_exp_per_iteration": 3, "half_steps": 1}


def _ragged(B, L, seed, lo_frac=0.4):
    rng = np.random.default_rng(seed)
    m = np.zeros((B, L), np.uint8)
    for b in range(B):
        n = int(rng.integers(int(lo_frac * L), L + 1))
        m[b, :n] = 1
        m[b, rng.choice(n, size=max(1, n // 40), replace=False)] = 0
    return m


CASES = {
    # one CTA per strip: d = 64 windows of 3 and 5 tiles, d = 128 window of 3 with R = 4
    "d64_W256_ragged": lambda: eot_inputs.dense_case(2, 2, 1024, 64, 256, 8, 2, "bf16", seed=41,
                                                     mask=_ragged(2, 1024, 41), name="d64_W256"),
    "d64_W512": lambda: eot_inputs.dense_case(1, 2, 1280, 64, 512, 6, 2, "bf16", seed=42, name="d64_W512"),
    "d128_W128_R4_ragged": lambda: eot_inputs.dense_case(2, 2, 768, 128, 128, 6, 4, "bf16", seed=43,
                                                         mask=_ragged(2, 768, 43), name="d128_W128_R4"),
    # CTA pairs: odd and even tile counts per strip, the long workload's shape at a short length
    "d64_W1024_pair": lambda: eot_inputs.dense_case(1, 2, 1536, 64, 1024, 5, 2, "bf16", seed=44, name="d64_W1024"),
    "d128_W512_pair_ragged": lambda: eot_inputs.dense_case(1, 2, 1408, 128, 512, 5, 2, "bf16", seed=45,
                                                           mask=_ragged(1, 1408, 45), name="d128_W512"),
    "d128_W1024_pair_long_init": lambda: eot_inputs.dense_case(1, 2, 2048, 128, 1024, 4, 2, "bf16", seed=46,
                                                               std=128 ** -0.5, name="d128_W1024"),
    # edge cases of the band and the schedule
    "d128_W0": lambda: eot_inputs.dense_case(1, 2, 256, 128, 0, 3, 2, "bf16", seed=47, name="d128_W0"),
    "d64_oddW_T1_R0": lambda: eot_inputs.dense_case(1, 2, 384, 64, 77, 1, 0, "bf16", seed=48, name="d64_T1_R0"),
    "d64_masked_unit": lambda: eot_inputs.dense_case(2, 1, 512, 64, 100, 4, 2, "bf16", seed=49,
                                                     mask=np.stack([np.ones(512, np.uint8), np.zeros(512, np.uint8)]),
                                                     name="d64_masked_unit"),
}


@pytest.fixture
def schedule():
    from entropic_ot_attention_b200 import _abi
    yield lambda s: _abi.eot_set_forward_schedule(SCHEDULES[s])
    _abi.eot_set_forward_schedule(_abi.SCHEDULE_AUTO)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("sched", sorted(SCHEDULES))
def test_forward_schedule_parity(name, sched, schedule):
    case = CASES[name]()
    schedule(sched)
    errs = compare(gpu_run(case), oracle_run(case))
    tol = TOL[case.dtype]
    assert all(e <= tol for e in errs.values()), f"{name} [{sched}]: {errs}"


def test_one_exp_schedule_is_deterministic_and_counts_its_exponentials(schedule):
    """Two runs give identical bits (no atomics in the column sums); the library reports one
    exponential pass per iteration plus the first row half-step."""
    import torch
    from entropic_ot_attention_b200 import _abi, api
    case = CASES["d128_W512_pair_ragged"]()
    schedule("one_exp")
    a = gpu_run(case)
    b = gpu_run(case)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    B, H, L, d = case.Q.shape
    p = api.make_problem(B, H, L, d, case.W, case.T, case.R, torch.bfloat16)
    assert _abi.eot_solve_exp_passes(p) == case.T + case.R + 1
    schedule("half_steps")
    assert _abi.eot_solve_exp_passes(p) == 2 * (case.T + case.R)
    _abi.eot_set_forward_schedule(_abi.SCHEDULE_AUTO)
    assert _abi.eot_solve_exp_passes(p) == 2 * (case.T + case.R)
    schedule("one_exp")
    dust = api.make_problem(1, 1, 256, 64, 32, 2, 2, torch.bfloat16, None, 200, 0.1)
    assert _abi.eot_solve_exp_passes(dust) == 2 * 4


def test_schedules_agree(schedule):
    """The two schedules compute the same iterates: their outputs differ by rounding only."""
    case = CASES["d64_W1024_pair"]()
    schedule("one_exp")
    a = gpu_run(case)
    schedule("half_steps")
    b = gpu_run(case)
    errs = compare(a, b)
    # potentials: fp32 on both sides (the column sums of one see bf16 plan entries); outputs: bf16,
    # so one rounding step of the largest entry (2^-8) can separate them
    assert errs["u"] <= 2e-3 and errs["v"] <= 2e-3, errs
    assert all(errs[k] <= 1.2e-2 for k in ("O", "dQ", "dK", "dV")), errs
