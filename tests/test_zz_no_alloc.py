"""The forward entry point that allocates nothing (eot_sinkhorn_fwd_static).

Some callers cannot call cudaMalloc where they run attention: a plug-in inside a host that
owns all device memory and gives it no allocator, or a serving loop that forbids
cudaMalloc/cudaFree after start-up because those calls can synchronise the device.  For them
the library keeps its forward scratch in a fixed device array of its own.  These tests call
that entry point through the C ABI and check it against eot_sinkhorn_fwd (which uses a
caller-supplied workspace) bit for bit, on two calls in a row and across calls whose scratch
layouts differ, against the float64 oracle within the parity tolerance, that its status word
is readable, and that a call after the first allocates no device memory.  The file name makes
pytest collect it last."""
import numpy as np
import pytest

import eot_inputs
from harness import TOL, oracle_run, pot_err, rel_err

pytestmark = pytest.mark.gpu


def _dense():
    return eot_inputs.dense_case(2, 2, 640, 64, 200, 8, 2, "bf16", seed=21,
                                 mask=(np.arange(640)[None, :] < np.array([[600], [333]])).astype(np.uint8),
                                 name="static_bf16")


def _dustbin():
    return eot_inputs.dustbin_case(1, 2, 300, 128, 96, 6, 2, "bf16", seed=22, mass=0.1, name="static_dustbin")


def _fp32():
    return eot_inputs.dense_case(1, 1, 256, 32, 32, 10, 2, "fp32", seed=23, name="static_fp32")


class _Call:
    """Device inputs and outputs of one forward problem, allocated up front."""

    def __init__(self, case):
        import torch
        from entropic_ot_attention_b200 import api
        self.dev = torch.device("cuda:0")
        tdt = torch.float32 if case.dtype == "fp32" else torch.bfloat16
        self.q, self.k, self.v = (torch.from_numpy(x).to(self.dev).to(tdt).contiguous()
                                  for x in (case.Q, case.K, case.V))
        self.mask = None if case.mask is None else torch.from_numpy(case.mask).to(self.dev)
        B, H, L, d = self.q.shape
        dbi = case.dustbin_index if case.dustbin else None
        self.p = api.make_problem(B, H, L, d, case.W, case.T, case.R, tdt, case.scale, dbi, case.dustbin_mass)
        self.O = torch.empty_like(self.q)
        self.ut = torch.empty((B, H, case.R + 1, L), device=self.dev)
        self.vt = torch.empty_like(self.ut)
        self.ws = api.workspace(self.p, False, self.dev)

    def _ptrs(self):
        m = None if self.mask is None else self.mask.data_ptr()
        return (self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), m, self.O.data_ptr(),
                self.ut.data_ptr(), self.vt.data_ptr())

    def poison(self):
        for t in (self.O, self.ut, self.vt):
            t.fill_(float("nan"))

    def static(self):
        import torch
        from entropic_ot_attention_b200 import _abi
        s = torch.cuda.current_stream().cuda_stream
        st = _abi.eot_sinkhorn_fwd_static(self.p, *self._ptrs(), s)
        assert st == _abi.EOT_OK, _abi.eot_status_string(st)

    def with_workspace(self):
        import torch
        from entropic_ot_attention_b200 import _abi
        s = torch.cuda.current_stream().cuda_stream
        _abi.eot_sinkhorn_fwd(self.p, *self._ptrs(), self.ws.data_ptr(), self.ws.numel(), s)

    def result(self):
        import torch
        torch.cuda.synchronize()
        return tuple(t.float().cpu().numpy() for t in (self.O, self.ut, self.vt))


def _static_status():
    import torch
    from entropic_ot_attention_b200 import _abi
    return _abi.eot_static_last_device_status(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("case_fn", [_dense, _dustbin, _fp32])
def test_static_scratch_forward_matches_workspace_forward(case_fn):
    from entropic_ot_attention_b200 import _abi
    case = case_fn()
    c = _Call(case)
    c.poison()
    c.with_workspace()
    ref = c.result()
    orc = oracle_run(case)
    tol = TOL[case.dtype]
    for _ in range(2):
        c.poison()
        c.static()
        got = c.result()
        assert _static_status() == _abi.EOT_OK
        for g, r in zip(got, ref):
            assert np.array_equal(g, r)
        assert rel_err(got[0], orc["O"]) <= tol
        assert pot_err(got[1], orc["u"]) <= tol
        assert pot_err(got[2], orc["v"]) <= tol


def test_static_scratch_across_layouts():
    """The array keeps the last call's contents: a dustbin problem, then a plain problem with
    another T (different workspace regions and grid-barrier counters), then the dustbin problem
    again must each equal eot_sinkhorn_fwd bit for bit."""
    from entropic_ot_attention_b200 import _abi
    plain = eot_inputs.dense_case(1, 3, 512, 64, 160, 3, 1, "bf16", seed=24, name="static_plain_T3")
    for case in (_dustbin(), plain, _dustbin()):
        c = _Call(case)
        c.poison()
        c.with_workspace()
        ref = c.result()
        c.poison()
        c.static()
        got = c.result()
        assert _static_status() == _abi.EOT_OK
        for g, r in zip(got, ref):
            assert np.array_equal(g, r)


def test_static_scratch_call_allocates_no_device_memory():
    """After a first call (which loads the kernels), a further call leaves the device's free
    memory unchanged."""
    import torch
    c = _Call(_dense())
    c.static()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    c.static()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0


def test_static_scratch_rejects_oversized_problem():
    import torch
    from entropic_ot_attention_b200 import _abi, api
    # forward scratch of B=8, H=16, L=16384 is ~42 MB, more than the static array; nothing is launched
    p = api.make_problem(8, 16, 16384, 64, 64, 2, 2, torch.bfloat16)
    assert _abi.eot_workspace_bytes(p, False) > _abi.EOT_STATIC_SCRATCH_BYTES
    fake = 1 << 20
    st = _abi.eot_sinkhorn_fwd_static(p, fake, fake, fake, None, fake, fake, fake, 0)
    assert st == _abi.EOT_ERR_WORKSPACE_TOO_SMALL
