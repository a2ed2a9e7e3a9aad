"""The forward entry point that allocates nothing (eot_sinkhorn_fwd_static).

Some callers cannot call cudaMalloc where they run attention: a plug-in inside a host that
owns all device memory and gives it no allocator, or a serving loop that forbids
cudaMalloc/cudaFree after start-up because those calls can synchronise the device.  For them
the library keeps its forward scratch in a fixed device array of its own.  This test calls
that entry point through the C ABI and checks it against eot_sinkhorn_fwd (which uses a
caller-supplied workspace) on two calls in a row, within the parity tolerance of the tests.
The file name makes pytest collect it last."""
import numpy as np
import pytest

import eot_inputs
from harness import TOL, pot_err, rel_err

pytestmark = pytest.mark.gpu


def _run(case, use_static, calls=1):
    import torch
    from entropic_ot_attention_b200 import _abi, api
    dev = torch.device("cuda:0")
    tdt = torch.float32 if case.dtype == "fp32" else torch.bfloat16
    q, k, v = (torch.from_numpy(x).to(dev).to(tdt).contiguous() for x in (case.Q, case.K, case.V))
    mask = None if case.mask is None else torch.from_numpy(case.mask).to(dev)
    B, H, L, d = q.shape
    dbi = case.dustbin_index if case.dustbin else None
    p = api.make_problem(B, H, L, d, case.W, case.T, case.R, tdt, case.scale, dbi, case.dustbin_mass)
    s = torch.cuda.current_stream().cuda_stream
    m = None if mask is None else mask.data_ptr()
    outs = []
    for _ in range(calls):
        O = torch.full_like(q, float("nan"))
        ut = torch.full((B, H, case.R + 1, L), float("nan"), device=dev)
        vt = torch.full_like(ut, float("nan"))
        if use_static:
            st = _abi.eot_sinkhorn_fwd_static(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), m, O.data_ptr(),
                                              ut.data_ptr(), vt.data_ptr(), s)
            assert st == _abi.EOT_OK, _abi.eot_status_string(st)
        else:
            ws = api.workspace(p, False, dev)
            _abi.eot_sinkhorn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), m, O.data_ptr(), ut.data_ptr(),
                                  vt.data_ptr(), ws.data_ptr(), ws.numel(), s)
        torch.cuda.synchronize()
        outs.append(tuple(t.float().cpu().numpy().astype(np.float64) for t in (O, ut, vt)))
    return outs


@pytest.mark.parametrize("case_fn", [
    lambda: eot_inputs.dense_case(2, 2, 640, 64, 200, 8, 2, "bf16", seed=21,
                                  mask=(np.arange(640)[None, :] < np.array([[600], [333]])).astype(np.uint8),
                                  name="static_bf16"),
    lambda: eot_inputs.dustbin_case(1, 2, 300, 128, 96, 6, 2, "bf16", seed=22, mass=0.1, name="static_dustbin"),
    lambda: eot_inputs.dense_case(1, 1, 256, 32, 32, 10, 2, "fp32", seed=23, name="static_fp32"),
])
def test_static_scratch_forward_matches_workspace_forward(case_fn):
    case = case_fn()
    ref = _run(case, use_static=False)[0]
    tol = TOL[case.dtype]
    for O, ut, vt in _run(case, use_static=True, calls=2):
        assert np.all(np.isfinite(O)) and np.all(np.isfinite(ut)) and np.all(np.isfinite(vt))
        assert rel_err(O, ref[0]) <= tol
        assert pot_err(ut, ref[1]) <= tol
        assert pot_err(vt, ref[2]) <= tol


def test_static_scratch_rejects_oversized_problem():
    import torch
    from entropic_ot_attention_b200 import _abi, api
    # forward scratch of B=8, H=16, L=8192 is ~21 MB > 16 MiB; nothing is launched
    p = api.make_problem(8, 16, 8192, 64, 64, 2, 2, torch.bfloat16)
    assert _abi.eot_workspace_bytes(p, False) > _abi.EOT_STATIC_SCRATCH_BYTES
    fake = 1 << 20
    st = _abi.eot_sinkhorn_fwd_static(p, fake, fake, fake, None, fake, fake, fake, 0)
    assert st == _abi.EOT_ERR_WORKSPACE_TOO_SMALL
