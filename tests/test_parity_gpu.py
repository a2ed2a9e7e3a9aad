"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on identical
seeded inputs.  Tolerance (relative max error over active entries, per tensor): 1e-4 for
fp32 inputs, 2e-2 for bf16 inputs, on O, u, v, dQ, dK, dV.

Small cases use the dense oracle over every unit and span several 128-row tiles with ragged
masks; the named workloads run in full on the GPU and are compared on sampled units with
the banded C oracle (whole units: the iteration couples every position of a unit)."""
import numpy as np
import pytest

import eot_inputs
from harness import TOL, compare, gpu_run, oracle_run

pytestmark = pytest.mark.gpu

IMPLS = ["auto", "simt"]


def _ragged_mask(B, L, seed, lo_frac=0.3):
    rng = np.random.default_rng(seed)
    m = np.zeros((B, L), np.uint8)
    for b in range(B):
        n = int(rng.integers(int(lo_frac * L), L + 1))
        m[b, :n] = 1
        holes = rng.choice(n, size=max(1, n // 50), replace=False)
        m[b, holes] = 0
    return m


def _check(case, impl="auto", units=None, banded=False):
    g = gpu_run(case, impl)
    o = oracle_run(case, units=units, use_banded=banded)
    H = case.Q.shape[1]
    errs = compare(g, o, units=units, H=H)
    tol = TOL[case.dtype]
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, f"{case.name} [{impl}]: {errs}"
    return errs


SMALL = {
    "fp32_tiny_L256": lambda: eot_inputs.workload("tiny"),
    "fp32_masked_L384": lambda: eot_inputs.dense_case(2, 2, 384, 32, 48, 12, 2, "fp32", seed=3,
                                                      mask=_ragged_mask(2, 384, 3), name="fp32_masked"),
    "bf16_d64_ragged_L640": lambda: eot_inputs.dense_case(2, 2, 640, 64, 200, 8, 2, "bf16", seed=4,
                                                          mask=_ragged_mask(2, 640, 4), name="bf16_d64_ragged"),
    "bf16_d128_fullband_L384": lambda: eot_inputs.dense_case(1, 2, 384, 128, 1000, 5, 2, "bf16", seed=5,
                                                             name="bf16_d128_full"),
    "bf16_d64_W0": lambda: eot_inputs.dense_case(1, 2, 256, 64, 0, 4, 2, "bf16", seed=6, name="bf16_W0"),
    "bf16_d64_R0": lambda: eot_inputs.dense_case(1, 2, 384, 64, 96, 6, 0, "bf16", seed=7, name="bf16_R0"),
    "bf16_d64_R1_T0": lambda: eot_inputs.dense_case(1, 2, 256, 64, 64, 0, 1, "bf16", seed=8, name="bf16_R1_T0"),
    "bf16_d128_R4": lambda: eot_inputs.dense_case(2, 1, 512, 128, 130, 6, 4, "bf16", seed=9,
                                                  mask=_ragged_mask(2, 512, 9), name="bf16_R4"),
    "bf16_d64_oddW": lambda: eot_inputs.dense_case(1, 2, 384, 64, 77, 5, 2, "bf16", seed=10, name="bf16_oddW"),
    "bf16_dustbin_L300": lambda: eot_inputs.dustbin_case(2, 2, 300, 64, 64, 6, 2, "bf16", seed=11, mass=0.1,
                                                         mask=_ragged_mask(2, 300, 11), name="bf16_dustbin"),
    "fp32_dustbin_L200": lambda: eot_inputs.dustbin_case(1, 2, 200, 32, 40, 8, 2, "fp32", seed=12, mass=0.2,
                                                         name="fp32_dustbin"),
    "bf16_d128_dustbin": lambda: eot_inputs.dustbin_case(1, 2, 250, 128, 90, 5, 2, "bf16", seed=13, mass=0.1,
                                                         name="bf16_d128_dustbin"),
    # d = 128 with W >= 512: the fused half-steps take the column bias from the score product,
    # so masked columns and the dustbin run through its -2^100 operand rows
    "bf16_d128_W512_ragged_L896": lambda: eot_inputs.dense_case(2, 2, 896, 128, 512, 5, 2, "bf16", seed=22,
                                                                mask=_ragged_mask(2, 896, 22),
                                                                name="bf16_d128_W512_ragged"),
    "bf16_d128_W600_dustbin": lambda: eot_inputs.dustbin_case(1, 2, 700, 128, 600, 4, 2, "bf16", seed=23, mass=0.1,
                                                              mask=_ragged_mask(1, 700, 23),
                                                              name="bf16_d128_W600_dustbin"),
}


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("impl", IMPLS)
def test_small_parity(name, impl):
    case = SMALL[name]()
    if impl == "tcgen05" and (case.dtype != "bf16"):
        pytest.skip("tensor-core kernels are bf16 only")
    _check(case, impl)


def test_dustbin_without_self_link():
    import torch
    from entropic_ot_attention_b200 import sinkhorn_fwd
    from oracle import eot_oracle as eo
    case = eot_inputs.dustbin_case(1, 2, 200, 64, 50, 5, 2, "bf16", seed=14, mass=0.1, name="noself")
    q, k, v = (torch.from_numpy(x).cuda().to(torch.bfloat16).contiguous() for x in (case.Q, case.K, case.V))
    O, ut, vt = sinkhorn_fwd(q, k, v, case.W, case.T, case.R, None, None, case.dustbin_index, 0.1,
                             dustbin_self=False)
    Oo, uo, vo, _ = eo.forward(case.Q.astype(np.float64), case.K.astype(np.float64), case.V.astype(np.float64),
                               case.W, case.T, case.R, dustbin=True, dustbin_index=case.dustbin_index,
                               dustbin_mass=0.1, dustbin_self=False)
    from harness import rel_err
    assert rel_err(O.float().cpu().numpy(), Oo) <= 2e-2
    assert rel_err(ut.cpu().numpy(), uo) <= 2e-2


def test_backward_from_oracle_tail():
    """Feed the GPU backward the oracle's tail potentials: isolates the adjoint kernels."""
    case = eot_inputs.dense_case(2, 2, 512, 64, 150, 7, 2, "bf16", seed=15, mask=_ragged_mask(2, 512, 15),
                                 name="bwd_from_oracle")
    o = oracle_run(case)
    g = gpu_run(case, "auto", u_tail=o["u"], v_tail=o["v"])
    errs = compare(g, o, keys=("dQ", "dK", "dV"))
    assert all(e <= 2e-2 for e in errs.values()), errs


def test_fully_masked_row_and_empty_problem():
    import torch
    from entropic_ot_attention_b200 import sinkhorn_bwd, sinkhorn_fwd
    mask = np.ones((2, 256), np.uint8)
    mask[1] = 0
    case = eot_inputs.dense_case(2, 1, 256, 64, 32, 3, 2, "bf16", seed=16, mask=mask, name="masked_row")
    _check(case)
    q = torch.zeros(0, 2, 256, 64, device="cuda", dtype=torch.bfloat16)
    O, ut, vt = sinkhorn_fwd(q, q, q, 32, 3, 2)
    dQ, dK, dV = sinkhorn_bwd(q, q, q, ut, vt, q, 32)
    assert O.shape == q.shape and dQ.shape == q.shape


def test_simt_and_tensor_core_agree():
    """Both kernel families on the same bf16 problem agree closely (same fp32 potentials)."""
    case = eot_inputs.dense_case(1, 2, 512, 64, 128, 6, 2, "bf16", seed=17, name="impl_agree")
    a = gpu_run(case, "simt")
    b = gpu_run(case, "auto")
    errs = compare(b, a)
    assert all(e <= 2e-2 for e in errs.values()), errs


def test_device_status_reports_nonfinite():
    """A NaN input makes the potentials non-finite; the kernels flag it in the status word
    (no trap) and eot_last_device_status reports EOT_ERR_NONFINITE, then clears it."""
    import torch
    from entropic_ot_attention_b200 import _abi, api
    B, H, L, d = 1, 1, 256, 64
    q = torch.randn(B, H, L, d, device="cuda").to(torch.bfloat16)
    k = torch.randn_like(q)
    v = torch.randn_like(q)
    q[0, 0, 5, 3] = float("nan")
    p = api.make_problem(B, H, L, d, 32, 2, 2, torch.bfloat16)
    ws = api.workspace(p, False, q.device)
    O, ut, vt = torch.empty_like(q), torch.empty(B, H, 3, L, device="cuda"), torch.empty(B, H, 3, L, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    _abi.eot_sinkhorn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), None, O.data_ptr(), ut.data_ptr(),
                          vt.data_ptr(), ws.data_ptr(), ws.numel(), s)
    assert _abi.eot_last_device_status(ws.data_ptr(), s) == _abi.EOT_ERR_NONFINITE
    assert _abi.eot_last_device_status(ws.data_ptr(), s) == _abi.EOT_OK
    q[0, 0, 5, 3] = 0.5
    _abi.eot_sinkhorn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), None, O.data_ptr(), ut.data_ptr(),
                          vt.data_ptr(), ws.data_ptr(), ws.numel(), s)
    assert _abi.eot_last_device_status(ws.data_ptr(), s) == _abi.EOT_OK


# ----------------------------------------------------------------------------------------
# Named workloads at full size (sampled units vs the banded oracle)
# ----------------------------------------------------------------------------------------
WORKLOAD_UNITS = {
    "medium": [0, 13, 31],
    "dustbin": [0, 11],
    "protein_r2": [0, 37, 126],
    "protein_r4": [5, 64],
    "long": [2],
}


@pytest.mark.parametrize("name", ["tiny", "medium", "dustbin", "protein_r2", "protein_r4", "long"])
def test_workload_parity(name):
    case = eot_inputs.workload(name)
    units = None if name == "tiny" else WORKLOAD_UNITS[name]
    _check(case, "auto", units=units, banded=name != "tiny")


def test_kernel_family_selection():
    """bf16 with d in {64, 128} runs on the tensor-core kernels unless the band's tile list
    would not fit in shared memory; then AUTO picks the CUDA-core kernels and an explicit
    tensor-core request is refused before anything runs."""
    import torch
    from entropic_ot_attention_b200 import _abi, api
    p = api.make_problem(1, 4, 131072, 128, 1024, 10, 2, torch.bfloat16, 0.0, None, 0.0)
    assert _abi.eot_resolved_impl(p) == 2
    wide = api.make_problem(1, 1, 1 << 20, 128, 500000, 1, 1, torch.bfloat16, 0.0, None, 0.0)
    assert _abi.eot_resolved_impl(wide) == 1
    wide_tc = api.make_problem(1, 1, 1 << 20, 128, 500000, 1, 1, torch.bfloat16, 0.0, None, 0.0, impl="tcgen05")
    assert _abi.eot_validate(wide_tc) == 2   # EOT_ERR_UNSUPPORTED


@pytest.mark.parametrize("plan", [{"heads_per_chunk": 1}, {"rows_per_chunk": 1}, {"rows_per_chunk": 2}, {}],
                         ids=["heads1", "rows1", "rows2_ragged", "auto"])
def test_host_step_matches_device_calls(plan):
    """HostStep (chunks of heads of one row, or of whole rows, on three streams, host buffers)
    gives bit-identical results to one device-resident forward + backward over the whole batch:
    the units are independent.  rows_per_chunk=2 over B=3 leaves a smaller last chunk."""
    import torch
    from entropic_ot_attention_b200 import HostStep, sinkhorn_bwd, sinkhorn_fwd
    case = eot_inputs.dense_case(3, 2, 384, 64, 96, 4, 2, "bf16", seed=21, mask=_ragged_mask(3, 384, 21),
                                 name="host_step")
    dt = torch.bfloat16
    q, k, v, dO = (torch.from_numpy(x).to(dt) for x in (case.Q, case.K, case.V, case.dO))
    mask = torch.from_numpy(case.mask)
    O, ut, vt = sinkhorn_fwd(q.cuda(), k.cuda(), v.cuda(), case.W, case.T, case.R, mask=mask.cuda(), scale=case.scale)
    dQ, dK, dV = sinkhorn_bwd(q.cuda(), k.cuda(), v.cuda(), ut, vt, dO.cuda(), case.W, mask=mask.cuda(),
                              scale=case.scale)
    B, H, L, d = q.shape
    hs = HostStep(B, H, L, d, case.W, case.T, case.R, dt, case.scale, mask=mask, **plan)
    host = [t.pin_memory() for t in (q, k, v, dO)]
    outs = [torch.empty_like(q).pin_memory() for _ in range(4)]
    for _ in range(2):   # slots reused across steps
        hs.run(*host, *outs)
    assert hs.device_status() == 0
    for got, want in zip(outs, (O, dQ, dK, dV)):
        assert torch.equal(got, want.cpu())
