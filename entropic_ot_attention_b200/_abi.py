"""ctypes binding of libeot's C ABI (include/eot.h): argument marshalling only.

Every function here has the name of the C entry point it wraps and forwards plain
pointers and sizes; all computation happens in the library's CUDA kernels.  Importing this
module fails loudly when libeot.so is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libeot.so")

EOT_OK = 0
EOT_ERR_INVALID_ARGUMENT = 1
EOT_ERR_UNSUPPORTED = 2
EOT_ERR_WORKSPACE_TOO_SMALL = 3
EOT_ERR_CUDA = 4
EOT_ERR_NONFINITE = 5
EOT_ERR_TIMEOUT = 6

EOT_FP32 = 0
EOT_BF16 = 1
EOT_IMPL_AUTO = 0
EOT_IMPL_SIMT = 1
EOT_IMPL_TCGEN05 = 2


class eot_problem(ctypes.Structure):
    """Mirror of ``eot_problem`` in include/eot.h (field order and types must match)."""

    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("L", ctypes.c_int32), ("d", ctypes.c_int32),
        ("W", ctypes.c_int32), ("T", ctypes.c_int32), ("R", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("scale", ctypes.c_float), ("dustbin", ctypes.c_int32), ("dustbin_index", ctypes.c_int32),
        ("dustbin_mass", ctypes.c_float), ("dustbin_self", ctypes.c_int32), ("impl", ctypes.c_int32),
    ]


class EotError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {eot_status_string(status)} (status {status})")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libeot.so not found at {LIB_PATH}; build it with "
                      "`python entropic_ot_attention_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.POINTER(eot_problem)
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t

lib.eot_abi_version.restype = ctypes.c_int
lib.eot_validate.argtypes = [_P]
lib.eot_validate.restype = ctypes.c_int
lib.eot_resolved_impl.argtypes = [_P]
lib.eot_resolved_impl.restype = ctypes.c_int
lib.eot_workspace_bytes.argtypes = [_P, ctypes.c_int]
lib.eot_workspace_bytes.restype = _sz
lib.eot_status_string.argtypes = [ctypes.c_int]
lib.eot_status_string.restype = ctypes.c_char_p
lib.eot_sinkhorn_fwd.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.eot_sinkhorn_fwd.restype = ctypes.c_int
lib.eot_sinkhorn_bwd.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.eot_sinkhorn_bwd.restype = ctypes.c_int
lib.eot_band_half_step.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.eot_band_half_step.restype = ctypes.c_int
lib.eot_band_half_step_dustbin.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _sz,
                                           _vp]
lib.eot_band_half_step_dustbin.restype = ctypes.c_int
lib.eot_band_output.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.eot_band_output.restype = ctypes.c_int
lib.eot_last_device_status.argtypes = [_vp, _vp]
lib.eot_last_device_status.restype = ctypes.c_int
lib.eot_device_status_bits.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]
lib.eot_device_status_bits.restype = ctypes.c_int
lib.eot_sq_norms.argtypes = [_vp, _vp, _sz, ctypes.c_int, _vp, _vp]
lib.eot_sq_norms.restype = ctypes.c_int
lib.eot_contraction_offsets.argtypes = [_P]
lib.eot_contraction_offsets.restype = ctypes.c_int
lib.eot_contraction.argtypes = [_P, _vp, _vp, _vp, _vp, _vp]
lib.eot_contraction.restype = ctypes.c_int

lib.eot_sinkhorn_fwd_static.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.eot_sinkhorn_fwd_static.restype = ctypes.c_int
lib.eot_static_last_device_status.argtypes = [_vp]
lib.eot_static_last_device_status.restype = ctypes.c_int
lib.eot_static_scratch_bytes.restype = _sz
EOT_STATIC_SCRATCH_BYTES = int(lib.eot_static_scratch_bytes())
lib.eot_wait_selftest.argtypes = [ctypes.c_int, ctypes.c_uint64, _vp, _vp]
lib.eot_wait_selftest.restype = ctypes.c_int
EOT_SELFTEST_MBARRIER = 0
EOT_SELFTEST_GRID = 1
EOT_SELFTEST_CONTROL = 2
lib.eot_kernel_launches.restype = ctypes.c_longlong
lib.eot_solve_exp_passes.argtypes = [_P]
lib.eot_solve_exp_passes.restype = ctypes.c_int
lib.eot_set_backward_schedule.argtypes = [ctypes.c_int]
lib.eot_set_backward_schedule.restype = ctypes.c_int
lib.eot_set_forward_schedule.argtypes = [ctypes.c_int]
lib.eot_set_forward_schedule.restype = ctypes.c_int
SCHEDULE_AUTO, SCHEDULE_HALF_STEPS, SCHEDULE_ONE_EXP, SCHEDULE_ONE_EXP_PER_ITERATION = 0, 1, 2, 3
lib.eot_profile_begin.restype = None
lib.eot_profile_end.argtypes = [_vp]
lib.eot_profile_end.restype = ctypes.c_int
lib.eot_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
lib.eot_profile_read.restype = ctypes.c_int

# Every symbol declared in include/eot.h (checked by the CPU tests).
EXPORTED = ("eot_workspace_bytes", "eot_validate", "eot_sinkhorn_fwd", "eot_sinkhorn_bwd",
            "eot_last_device_status", "eot_device_status_bits", "eot_status_string",
            "eot_abi_version", "eot_resolved_impl", "eot_kernel_launches", "eot_profile_begin",
            "eot_profile_end", "eot_profile_read", "eot_sinkhorn_fwd_static", "eot_solve_exp_passes",
            "eot_static_last_device_status", "eot_static_scratch_bytes", "eot_wait_selftest",
            "eot_set_forward_schedule", "eot_set_backward_schedule")

PROF_KINDS = {"fwd_sweep": 0, "fwd_output": 1, "bwd_sweep": 2, "aux": 3, "bwd_staircase": 4}


def eot_kernel_launches() -> int:
    return int(lib.eot_kernel_launches())


def eot_solve_exp_passes(p: eot_problem) -> int:
    return int(lib.eot_solve_exp_passes(ctypes.byref(p)))


def eot_set_backward_schedule(schedule: int) -> None:
    _check(lib.eot_set_backward_schedule(int(schedule)), "eot_set_backward_schedule")


def eot_set_forward_schedule(schedule: int) -> None:
    _check(lib.eot_set_forward_schedule(int(schedule)), "eot_set_forward_schedule")


def eot_profile_begin() -> None:
    lib.eot_profile_begin()


def eot_profile_end(stream: int) -> None:
    _check(lib.eot_profile_end(stream), "eot_profile_end")


def eot_profile_read(kind: int):
    ms = ctypes.c_double(0.0)
    n = ctypes.c_longlong(0)
    _check(lib.eot_profile_read(int(kind), ctypes.byref(ms), ctypes.byref(n)), "eot_profile_read")
    return float(ms.value), int(n.value)


def eot_status_string(status: int) -> str:
    return lib.eot_status_string(int(status)).decode()


def eot_abi_version() -> int:
    return lib.eot_abi_version()


def eot_validate(p: eot_problem) -> int:
    return lib.eot_validate(ctypes.byref(p))


def eot_resolved_impl(p: eot_problem) -> int:
    return lib.eot_resolved_impl(ctypes.byref(p))


def eot_workspace_bytes(p: eot_problem, for_backward: bool) -> int:
    return int(lib.eot_workspace_bytes(ctypes.byref(p), int(bool(for_backward))))


def _check(status: int, what: str) -> None:
    if status != EOT_OK:
        raise EotError(status, what)


def eot_sinkhorn_fwd(p: eot_problem, Q: int, K: int, V: int, mask: int | None, O: int, u_tail: int,
                     v_tail: int, workspace: int, workspace_bytes: int, stream: int) -> None:
    """Forward; all tensor arguments are raw device addresses (ints), mask may be None."""
    _check(lib.eot_sinkhorn_fwd(ctypes.byref(p), Q, K, V, mask, O, u_tail, v_tail, workspace,
                                workspace_bytes, stream), "eot_sinkhorn_fwd")


def eot_sinkhorn_bwd(p: eot_problem, Q: int, K: int, V: int, mask: int | None, u_tail: int, v_tail: int,
                     dO: int, dQ: int, dK: int, dV: int, workspace: int, workspace_bytes: int,
                     stream: int) -> None:
    """Backward; raw device addresses as in eot_sinkhorn_fwd."""
    _check(lib.eot_sinkhorn_bwd(ctypes.byref(p), Q, K, V, mask, u_tail, v_tail, dO, dQ, dK, dV, workspace,
                                workspace_bytes, stream), "eot_sinkhorn_bwd")


def eot_band_half_step(p: eot_problem, X: int, Y: int, log_marg: int, pot_in: int, pot_out: int,
                       workspace: int, workspace_bytes: int, stream: int) -> None:
    """One band half-step; raw device addresses as in eot_sinkhorn_fwd."""
    _check(lib.eot_band_half_step(ctypes.byref(p), X, Y, log_marg, pot_in, pot_out, workspace, workspace_bytes,
                                  stream), "eot_band_half_step")


def eot_band_half_step_dustbin(p: eot_problem, X: int, Y: int, log_marg: int, pot_in: int, pot_out: int,
                               own_lo: int, own_hi: int, dust_part: int, workspace: int, workspace_bytes: int,
                               stream: int) -> None:
    """One band half-step of a part of a sequence with a dustbin; raw device addresses."""
    _check(lib.eot_band_half_step_dustbin(ctypes.byref(p), X, Y, log_marg, pot_in, pot_out, int(own_lo), int(own_hi),
                                          dust_part, workspace, workspace_bytes, stream), "eot_band_half_step_dustbin")


def eot_band_output(p: eot_problem, Q: int, K: int, V: int, log_marg: int, u: int, v: int, O: int, workspace: int,
                    workspace_bytes: int, stream: int) -> None:
    """The output of given potentials; raw device addresses."""
    _check(lib.eot_band_output(ctypes.byref(p), Q, K, V, log_marg, u, v, O, workspace, workspace_bytes, stream),
           "eot_band_output")


def eot_sinkhorn_fwd_static(p: eot_problem, Q: int, K: int, V: int, mask: int | None, O: int, u_tail: int,
                            v_tail: int, stream: int) -> int:
    """Forward with the library's static scratch (no workspace); returns the raw status."""
    return lib.eot_sinkhorn_fwd_static(ctypes.byref(p), Q, K, V, mask, O, u_tail, v_tail, stream)


def eot_static_last_device_status(stream: int) -> int:
    """Status of the last eot_sinkhorn_fwd_static call(s) in this context (syncs ``stream``)."""
    return lib.eot_static_last_device_status(stream)


def eot_wait_selftest(which: int, limit_ns: int, scratch: int, stream: int) -> None:
    """Launch the bounded-wait self-test (raw device address of a 256-byte scratch buffer)."""
    _check(lib.eot_wait_selftest(int(which), int(limit_ns), scratch, stream), "eot_wait_selftest")


def eot_last_device_status(workspace: int, stream: int) -> int:
    return lib.eot_last_device_status(workspace, stream)


def eot_device_status_bits(workspace: int, stream: int) -> int:
    bits = ctypes.c_uint32(0)
    _check(lib.eot_device_status_bits(workspace, stream, ctypes.byref(bits)), "eot_device_status_bits")
    return int(bits.value)


def eot_sq_norms(a: int, b: int, n: int, dtype: int, out: int, stream: int) -> None:
    """out[0] = sum (a - b)^2, out[1] = sum a^2 over n elements (raw device addresses; out is a
    device array of two float64), enqueued on ``stream``."""
    _check(lib.eot_sq_norms(a, b, n, dtype, out, stream), "eot_sq_norms")


def eot_contraction_offsets(p: eot_problem) -> int:
    return int(lib.eot_contraction_offsets(ctypes.byref(p)))


def eot_contraction(p: eot_problem, Q: int, K: int, mask: int | None, kappa: int, stream: int) -> None:
    """Per-tile Birkhoff-Hopf ratios into kappa (raw device addresses; mask may be None)."""
    _check(lib.eot_contraction(ctypes.byref(p), Q, K, mask, kappa, stream), "eot_contraction")
