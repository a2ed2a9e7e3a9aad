"""Repeated forward + backward calls at full workload size keep the device status clean.

Every wait inside the kernels is bounded; one that runs out sets the timeout bit and the call's
results are wrong, so a wait that cannot complete under some timing (a barrier phase that only
a later step of the waiting thread itself would complete) shows up here as a status other than
EOT_OK on one of many calls.  The dustbin workload runs the row sweep without products (alpha_R
on the sweep kernel); the protein-like batch has many inactive row tiles."""
import pytest

import eot_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,calls", [("dustbin", 60), ("protein_r2", 20)])
def test_repeated_calls_keep_status_ok(name, calls):
    import torch
    from entropic_ot_attention_b200 import _abi, api
    case = eot_inputs.workload(name)
    dev = torch.device("cuda:0")
    q, k, v, dO = (torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous() for x in (case.Q, case.K, case.V, case.dO))
    B, H, L, d = q.shape
    mask = None if case.mask is None else torch.from_numpy(case.mask).to(dev)
    dbi = case.dustbin_index if case.dustbin else None
    p = api.make_problem(B, H, L, d, case.W, case.T, case.R, torch.bfloat16, case.scale, dbi, case.dustbin_mass)
    wf, wb = api.workspace(p, False, dev), api.workspace(p, True, dev)
    O = torch.empty_like(q)
    ut = torch.empty(B, H, case.R + 1, L, device=dev)
    vt = torch.empty_like(ut)
    dQ, dK, dV = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    s = torch.cuda.current_stream().cuda_stream
    m = None if mask is None else mask.data_ptr()
    for i in range(calls):
        _abi.eot_sinkhorn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), m, O.data_ptr(), ut.data_ptr(),
                              vt.data_ptr(), wf.data_ptr(), wf.numel(), s)
        _abi.eot_sinkhorn_bwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), m, ut.data_ptr(), vt.data_ptr(),
                              dO.data_ptr(), dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(), wb.data_ptr(), wb.numel(), s)
        sf = _abi.eot_last_device_status(wf.data_ptr(), s)
        sb = _abi.eot_last_device_status(wb.data_ptr(), s)
        assert sf == 0 and sb == 0, (i, _abi.eot_status_string(sf), _abi.eot_status_string(sb))
