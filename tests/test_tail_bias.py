"""Bias of the stop-gradient tail against full backpropagation through every Sinkhorn step.

BDSA §2.4 (first certificate) and §4.1 ("bias decrease"): with a locally contractive
refinement map the gap between the full gradient and the tail surrogate's shrinks
geometrically in the tail depth R; measured against full BPTT it falls sharply from R = 0 to
R = 1 and R = 2.

CPU: the full-gradient oracle (``oracle.bptt``, torch autodiff) is pinned against the
hand-written tail adjoint of ``oracle.eot_oracle`` (independent code) for every base / tail
split of a fixed step count, and against central differences of the forward.  GPU: the kernels'
tail gradients for R = 0, 1, 2, 4 give the same bias curve as the oracle's.
"""
import math

import numpy as np
import pytest

import eot_inputs
from oracle import bptt
from oracle import eot_oracle as eo


def _unit(L, d, seed, mask=None, dustbin=False, mass=0.0):
    rng = np.random.default_rng(seed)
    q, k, v, dO = (rng.standard_normal((L, d)) for _ in range(4))
    kw = dict(mask_row=mask, dustbin=dustbin, dustbin_index=L - 2 if dustbin else -1, dustbin_mass=mass)
    return q, k, v, dO, kw


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


@pytest.mark.parametrize("masked,dustbin", [(False, False), (True, False), (True, True)])
@pytest.mark.parametrize("T", [0, 2, 5, 7])
def test_stopped_autodiff_equals_hand_written_tail_adjoint(T, masked, dustbin):
    """With the potentials after T of N = 7 steps held constant, autodiff gives the tail
    adjoint of depth N - T (R = 0: plan gradient only; T = 0: nothing is stopped, so the full
    gradient equals the tail adjoint of depth N)."""
    L, d, W, N = 24, 4, 6, 7
    mask = None
    if masked:
        mask = np.ones(L, np.uint8)
        mask[[3, 11, 12]] = 0
    q, k, v, dO, kw = _unit(L, d, 5 + T, mask, dustbin, 0.15 if dustbin else 0.0)
    f = eo.forward_unit(q, k, v, W, T, N - T, **kw)
    b = eo.backward_unit(q, k, v, dO, f)
    g = bptt.gradient_unit(q, k, v, dO, W, N, stop_after=T, **kw)
    for got, want in zip(g, (b.dQ, b.dK, b.dV)):
        assert _rel(got, want) <= 1e-12
    if T == 0:
        full = bptt.gradient_unit(q, k, v, dO, W, N, stop_after=None, **kw)
        for got, want in zip(full, (b.dQ, b.dK, b.dV)):
            assert _rel(got, want) <= 1e-12


@pytest.mark.parametrize("dustbin", [False, True])
def test_full_gradient_matches_central_differences(dustbin):
    """The full gradient is the derivative of the forward itself (all N steps move with the
    inputs): central differences of eot_oracle's forward."""
    L, d, W, N = 10, 3, 4, 5
    mask = np.ones(L, np.uint8)
    mask[4] = 0
    q, k, v, dO, kw = _unit(L, d, 41, mask, dustbin, 0.2 if dustbin else 0.0)
    scale = 1.0 / math.sqrt(d)
    g = bptt.gradient_unit(q, k, v, dO, W, N, None, scale, **kw)

    def phi(qq, kk, vv):
        # the forward does not depend on the base / tail split: all N steps as base
        return float(np.sum(dO * eo.forward_unit(qq, kk, vv, W, N, 0, scale, **kw).O))

    h = 1e-6
    for which, X, grad in ((0, q, g[0]), (1, k, g[1]), (2, v, g[2])):
        fd = np.zeros_like(X)
        for idx in np.ndindex(*X.shape):
            args_p, args_m = [q, k, v], [q, k, v]
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args_p[which], args_m[which] = Xp, Xm
            fd[idx] = (phi(*args_p) - phi(*args_m)) / (2 * h)
        assert _rel(grad, fd) <= 1e-6, which


def test_bias_decays_with_tail_depth():
    """bias(R) = ||g_full - g_tail(R)|| / ||g_full|| falls with R on a banded, masked unit and
    vanishes when the tail covers every step; the drop from R = 0 to R = 2 is large."""
    L, d, W, N = 96, 16, 24, 12
    mask = np.ones(L, np.uint8)
    mask[[10, 50, 51, 90]] = 0
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    dO = rng.standard_normal((L, d))
    curve = bptt.bias_curve(q, k, v, dO, W, N, Rs=(0, 1, 2, 4, N), mask_row=mask)
    assert curve[0] > curve[1] > curve[2] > curve[4] > 0.0
    assert curve[N] <= 1e-12
    assert curve[2] < 0.1 * curve[0]


@pytest.mark.gpu
def test_tail_bias_curve_matches_oracle():
    """The kernels' tail gradients (fp32, CUDA-core path) for R = 0, 1, 2, 4 at a fixed total
    step count N = T + R reproduce the oracle's bias curve against full backpropagation."""
    from harness import gpu_run
    B, H, L, d, W, N = 1, 2, 256, 32, 32, 12
    rows = []
    for R in (0, 1, 2, 4):
        case = eot_inputs.dense_case(B, H, L, d, W, N - R, R, "fp32", seed=77, name=f"bias_R{R}")
        g = gpu_run(case)
        for h in range(H):
            q, k, v, dO = (x[0, h].astype(np.float64) for x in (case.Q, case.K, case.V, case.dO))
            if R == 0:
                rows.append({})
            curve = rows[h]
            if "full" not in curve:
                curve.update(bptt.bias_curve(q, k, v, dO, W, N, Rs=(0, 1, 2, 4)))
            full = curve["full"]
            gpu_tail = np.concatenate([g[n][0, h].ravel() for n in ("dQ", "dK", "dV")])
            gpu_bias = float(np.linalg.norm(full - gpu_tail) / np.linalg.norm(full))
            print(f"head {h} R={R}: oracle bias {curve[R]:.4e}  GPU bias {gpu_bias:.4e}")
            assert abs(gpu_bias - curve[R]) <= 2e-4 + 1e-2 * curve[R]
    for curve in rows:
        assert curve[0] > curve[1] > curve[2] > curve[4]
