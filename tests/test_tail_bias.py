"""Bias of the stop-gradient tail against full backpropagation through every Sinkhorn step.

BDSA §2.4 (first certificate) and §4.1 ("bias decrease"): with a locally contractive
refinement map the gap between the full gradient and the tail surrogate's shrinks
geometrically in the tail depth R; measured against full BPTT it falls sharply from R = 0 to
R = 1 and R = 2.

CPU: the full-gradient oracle (``oracle.bptt``, torch autodiff) is pinned against the
hand-written tail adjoint of ``oracle.eot_oracle`` (independent code) for every base / tail
split of a fixed step count, and against central differences of the forward.  GPU: the kernels'
tail gradients for R = 0, 1, 2, 4 give the same bias curve as the oracle's.

BDSA §2.4 (third certificate): the a-posteriori certificate (``entropic_ot_attention_b200.
certificate``) is checked against the true residual on the CPU and, on the GPU, computed by
the library and compared with the same quantities from oracle gradients.
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


# ----------------------------------------------------------------------------------------
# A-posteriori certificate (BDSA §2.4, third certificate; §4.1)
# ----------------------------------------------------------------------------------------
def test_geometric_estimate_closed_forms():
    from entropic_ot_attention_b200.certificate import geometric_estimate
    assert geometric_estimate(0.3, 0.5, 0) == 0.0
    assert geometric_estimate(0.3, None, 1) == 0.3
    assert geometric_estimate(0.3, 0.5, 3) == pytest.approx(0.3 + 0.15 + 0.075)
    assert geometric_estimate(0.3, 1.0, 3) == math.inf
    assert geometric_estimate(0.3, None, 2) == math.inf


def _oracle_tails(q, k, v, dO, W, N, **kw):
    """Stacked (dq, dk, dv) of every tail depth 0..N from the oracle (depth N: nothing stopped)."""
    return {R: np.concatenate([g.ravel() for g in bptt.gradient_unit(q, k, v, dO, W, N, N - R, **kw)])
            for R in range(N + 1)}


def _oracle_certificates(tails, N):
    """eta_R, rho_R and the certificate eta_hat_R from oracle tail gradients, with the same
    reading as the library's (the formula under test is the library's geometric_estimate)."""
    from entropic_ot_attention_b200.certificate import geometric_estimate
    eta = {R: np.linalg.norm(tails[R + 1] - tails[R]) / np.linalg.norm(tails[R]) for R in range(N)}
    out = {}
    for R in range(N):
        rho = eta[R + 1] / eta[R] if R + 1 < N else None
        out[R] = (eta[R], rho, geometric_estimate(eta[R], rho, N - R))
    return out


def test_certificate_tracks_the_true_residual():
    """On a banded, masked unit the certificate stays within a factor 2 of the true residual
    |g(N) - g(R)| / |g(N)| from full backpropagation (the pages: it reconstructs the residual),
    or declines (+inf) where the increments stop shrinking: the first steps from v = 0 move the
    gradient more than the geometric model allows, so with two increments left it has none."""
    L, d, W, N = 96, 16, 24, 12
    mask = np.ones(L, np.uint8)
    mask[[10, 50, 51, 90]] = 0
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((L, d)) for _ in range(3))
    dO = rng.standard_normal((L, d))
    tails = _oracle_tails(q, k, v, dO, W, N, mask_row=mask)
    certs = _oracle_certificates(tails, N)
    for R in range(N):
        true = np.linalg.norm(tails[N] - tails[R]) / np.linalg.norm(tails[N])
        est = certs[R][2]
        if R <= N - 3:
            assert math.isfinite(est), R
        assert est == math.inf or 0.5 * true <= est <= 2.0 * true, (R, true, est)


@pytest.mark.gpu
def test_bias_certificate_matches_oracle():
    """The library's certificate (tail gradients and norms on the GPU, fp32) equals the oracle's
    at every depth, its exact residual equals full backpropagation's, and choose_tail_depth
    picks the oracle's depth for tolerances away from the certificate values."""
    import torch
    from entropic_ot_attention_b200 import bias_certificate, choose_tail_depth
    B, H, L, d, W, N = 1, 2, 256, 32, 32, 8
    case = eot_inputs.dense_case(B, H, L, d, W, 0, N, "fp32", seed=78, name="certificate")
    dev = torch.device("cuda:0")
    q, k, v, dO = (torch.from_numpy(x).to(dev).contiguous() for x in (case.Q, case.K, case.V, case.dO))
    per_head = [_oracle_tails(*(x[0, h].astype(np.float64) for x in (case.Q, case.K, case.V, case.dO)), W, N)
                for h in range(H)]
    tails = {R: np.concatenate([t[R] for t in per_head]) for R in range(N + 1)}   # both units, as the GPU
    certs = _oracle_certificates(tails, N)
    for R in range(N - 1):
        c = bias_certificate(q, k, v, dO, W, N, R, exact=True)
        eta, rho, est = certs[R]
        true = np.linalg.norm(tails[N] - tails[R]) / np.linalg.norm(tails[N])
        print(f"R={R}: eta {c['eta']:.4e} (oracle {eta:.4e})  rho {c['rho']:.4f}  "
              f"estimate {c['estimate']:.4e} (oracle {est:.4e})  exact {c['exact']:.4e} (oracle {true:.4e})")
        # eta is a difference of two nearly equal fp32 gradients (1e-3 of their size at the
        # deeper tails), so a gradient error of ~1e-6 becomes ~1e-3 of eta
        assert c["eta"] == pytest.approx(eta, rel=1e-2, abs=1e-6)
        assert c["estimate"] == pytest.approx(est, rel=1e-2, abs=1e-6)
        assert c["exact"] == pytest.approx(true, rel=5e-3, abs=1e-6)
    ests = [certs[R][2] for R in range(N - 1)]
    for tau in (0.1, 0.03, 0.008, 0.003):
        if any(abs(e - tau) <= 0.05 * tau for e in ests):
            continue   # too close to a certificate value to compare the choice
        want = next((R for R, e in enumerate(ests) if e <= tau), None)
        got, _ = choose_tail_depth(q, k, v, dO, W, N, tau=tau, R_max=N - 2)
        assert got == want, (tau, got, want)


def test_choose_tail_depth_control_flow(monkeypatch):
    """The depth search on the host, with the library calls replaced by a synthetic gradient
    sequence whose increments shrink by 1/2 per step (g(N) - g(R) known in closed form): each
    depth is computed once, the first depth whose certificate is <= tau is returned, and the
    certificate equals the geometric sum exactly when the increments are geometric."""
    import numpy as np
    from entropic_ot_attention_b200 import certificate as cm
    N = 8
    base = np.ones(4)
    step = np.array([1.0, -2.0, 0.5, 3.0])

    def g(R):   # g(R) = base + sum_{j < R} step * 0.5^(N - 1 - j): increments grow toward the full gradient
        return base + sum(step * 0.5 ** (N - 1 - j) for j in range(R))

    calls = []

    def fake_tail(q, k, v, dO, W, N_, R, **kw):
        calls.append(R)
        return (g(R),)

    def fake_norms(ga, gb, stream=None):
        a, b = ga[0], gb[0]
        return float(np.sum((a - b) ** 2)), float(np.sum(a ** 2))

    monkeypatch.setattr(cm, "tail_gradients", fake_tail)
    monkeypatch.setattr(cm, "_norms", fake_norms)
    R, certs = cm.choose_tail_depth(None, None, None, None, 0, N, tau=1e-9)
    assert R is None and len(calls) == len(set(calls))          # every depth computed once
    # increments double with R here (rho = 2): no certificate except with one step left
    assert all(c["estimate"] == math.inf for c in certs[:-1])
    c = cm.bias_certificate(None, None, None, None, 0, N, N - 1)
    assert c["estimate"] == pytest.approx(np.linalg.norm(g(N) - g(N - 1)) / np.linalg.norm(g(N - 1)))

    # reversed: increments halve with R (rho = 1/2), the certificate is the exact geometric sum
    def g2(R):
        return base + sum(step * 0.5 ** j for j in range(R))

    monkeypatch.setattr(cm, "tail_gradients", lambda q, k, v, dO, W, N_, R, **kw: (g2(R),))
    R2 = 3
    c = cm.bias_certificate(None, None, None, None, 0, N, R2)
    eta = np.linalg.norm(g2(R2 + 1) - g2(R2)) / np.linalg.norm(g2(R2))
    eta1 = np.linalg.norm(g2(R2 + 2) - g2(R2 + 1)) / np.linalg.norm(g2(R2 + 1))
    assert c["eta"] == pytest.approx(eta) and c["rho"] == pytest.approx(eta1 / eta)
    assert c["estimate"] == pytest.approx(eta * (1 - (eta1 / eta) ** (N - R2)) / (1 - eta1 / eta))
    tau = c["estimate"] * 1.01
    R, certs = cm.choose_tail_depth(None, None, None, None, 0, N, tau=tau)
    assert R is not None and R <= R2 and certs[-1]["estimate"] <= tau
    assert all(cc["estimate"] > tau for cc in certs[:-1])
