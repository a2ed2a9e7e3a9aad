"""Pins for the float64 oracle, each checked against something other than the oracle itself.

Sources ("BDSA" = Blockwise Differentiable Sinkhorn Attention, technical summary,
gist.science 2605.08123):
* scaling-orbit identity P(a,b) = P(R,R) exp(u(a)-u(R)) exp(v(b)-v(R))      BDSA §2.2
* balanced Sinkhorn: column marginals are exact after each v-update, row marginals
  converge                                                                   BDSA §2.1
* exact tail adjoint == finite differences of the stopped-base surrogate     BDSA §2.2, §4.1
* exact tail adjoint == reverse-mode autodiff of the tail (independent torch code)
* dustbin with zero mass == the plain problem on the real tokens              BDSA §2.3
plus closed forms (W = 0, 2x2 converged plan), symmetries, and the banded C twin.
"""
import math

import numpy as np
import pytest

from oracle import eot_oracle as eo
from oracle import banded as eb


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _unit(L=12, d=3, W=4, seed=0, mask=None, dustbin=False, mass=0.0):
    rng = np.random.default_rng(seed)
    q, k, v, dO = (_rand(rng, L, d) for _ in range(4))
    D = -1
    if dustbin:
        D = L - 2          # one filler after the dustbin
    return q, k, v, dO, dict(mask_row=mask, dustbin=dustbin, dustbin_index=D, dustbin_mass=mass)


def _rel(a, b):
    den = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / den)


# ----------------------------------------------------------------------------------------
# BDSA §2.2: scaling-orbit identity (exact algebra)
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("R", [1, 2, 3])
@pytest.mark.parametrize("dustbin", [False, True])
def test_orbit_identity(R, dustbin):
    mask = np.array([1, 1, 0, 1, 1, 1, 1, 0, 1, 1, 1, 1], np.uint8)
    q, k, v, dO, kw = _unit(mask=mask, dustbin=dustbin, mass=0.2 if dustbin else 0.0)
    f = eo.forward_unit(q, k, v, W=4, T=5, R=R, **kw)
    for ai in range(R + 1):
        for bi in range(R + 1):
            direct = eo.plan(f.S, f.u_tail[ai], f.v_tail[bi])
            orbit = eo.orbit_plan(f.S, f.u_tail, f.v_tail, ai, bi)
            assert _rel(orbit, direct) <= 1e-12
    dS = eo.tail_adjoint_dS(f.S, f.st, f.u_tail, f.v_tail, v, dO)[0]
    dS_orbit = eo.tail_adjoint_dS_orbit(f.S, f.st, f.u_tail, f.v_tail, v, dO)
    assert _rel(dS_orbit, dS) <= 1e-12


# ----------------------------------------------------------------------------------------
# BDSA §2.1: balanced Sinkhorn marginals
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("dustbin", [False, True])
def test_column_marginals_exact_after_each_v_update(dustbin):
    mask = np.array([1, 0, 1, 1, 1, 1, 1, 1, 0, 1, 1, 1, 1, 1, 1, 1], np.uint8)
    q, k, v, dO, kw = _unit(L=16, d=4, W=6, seed=3, mask=mask, dustbin=dustbin, mass=0.1 if dustbin else 0.0)
    st = eo.unit_structure(16, 6, mask, kw["dustbin"], kw["dustbin_index"], kw["dustbin_mass"])
    S = eo.scores(q, k, 0.5, st.support)
    u = np.zeros(16)
    vv = np.zeros(16)
    b = np.where(st.active, np.exp(st.log_a), 0.0)
    for _ in range(7):
        u = eo.row_step(S, st.log_a, vv, st.active)
        vv = eo.col_step(S, st.log_a, u, st.active)
        P = eo.plan(S, u, vv)
        assert np.max(np.abs(P.sum(axis=0) - b)) <= 1e-15
    assert abs(b.sum() - 1.0) <= 1e-15


@pytest.mark.parametrize("dustbin", [False, True])
def test_converged_row_marginals(dustbin):
    """Run the base to convergence: row sums then equal a to 1e-9 (column sums are exact)."""
    L = 20
    mask = np.ones(L, np.uint8)
    mask[[3, 11]] = 0
    q, k, v, dO, kw = _unit(L=L, d=4, W=8, seed=5, mask=mask, dustbin=dustbin, mass=0.15 if dustbin else 0.0)
    st = eo.unit_structure(L, 8, mask, kw["dustbin"], kw["dustbin_index"], kw["dustbin_mass"])
    S = eo.scores(q, k, 0.5, st.support)
    a = np.where(st.active, np.exp(st.log_a), 0.0)
    u = np.zeros(L)
    vv = np.zeros(L)
    err = 1.0
    for it in range(100000):
        u = eo.row_step(S, st.log_a, vv, st.active)
        vv = eo.col_step(S, st.log_a, u, st.active)
        err = np.max(np.abs(eo.plan(S, u, vv).sum(axis=1) - a))
        if err < 1e-12:
            break
    assert err <= 1e-9
    P = eo.plan(S, u, vv)
    assert np.max(np.abs(P.sum(axis=0) - a)) <= 1e-12


def test_two_by_two_converged_plan_closed_form():
    """2x2, full support, a = b = (1/2, 1/2): the Sinkhorn fixed point is
    P = [[p, 1/2 - p], [1/2 - p, p]] with p / (1/2 - p) = sqrt(exp(s11 + s22 - s12 - s21)),
    because diag-scaling preserves the cross ratio P11 P22 / (P12 P21) = K11 K22 / (K12 K21)."""
    q = np.array([[0.3, -1.1], [0.7, 0.4]])
    k = np.array([[1.2, 0.5], [-0.6, 0.9]])
    s = q @ k.T
    kappa = math.exp(s[0, 0] + s[1, 1] - s[0, 1] - s[1, 0])
    p = math.sqrt(kappa) / (2.0 * (1.0 + math.sqrt(kappa)))
    f = eo.forward_unit(q, k, np.eye(2), W=2, T=200, R=2, scale=1.0)
    P = eo.plan(f.S, f.u_tail[2], f.v_tail[2])
    expect = np.array([[p, 0.5 - p], [0.5 - p, p]])
    assert np.max(np.abs(P - expect)) <= 1e-14
    # O = diag(1/a) P V with V = I gives 2 P
    assert np.max(np.abs(f.O - 2.0 * expect)) <= 1e-13


# ----------------------------------------------------------------------------------------
# BDSA §2.2 / §4.1: exact adjoint of the stopped-base surrogate
# ----------------------------------------------------------------------------------------
def _phi_fixed_base(q, k, v, dO, st, v0, R, scale):
    S = eo.scores(q, k, scale, st.support)
    us, vs = eo.tail_solve(S, st, v0, R)
    uR = us[R] if R > 0 else None
    if R == 0:
        raise ValueError
    O = eo.output(S, st, uR, vs[R], v)
    return float(np.sum(dO * O))


@pytest.mark.parametrize("R,dustbin,masked", [(1, False, False), (2, False, False), (2, False, True),
                                              (3, False, False), (2, True, True)])
def test_adjoint_matches_central_differences(R, dustbin, masked):
    L, d, W = 12, 3, 4
    mask = None
    if masked:
        mask = np.ones(L, np.uint8)
        mask[[2, 7]] = 0
    q, k, v, dO, kw = _unit(L=L, d=d, W=W, seed=11 + R, mask=mask, dustbin=dustbin,
                            mass=0.2 if dustbin else 0.0)
    scale = 1.0 / math.sqrt(d)
    f = eo.forward_unit(q, k, v, W, T=3, R=R, scale=scale, **kw)
    g = eo.backward_unit(q, k, v, dO, f, scale)
    v0 = f.v_tail[0]
    st = f.st
    hstep = 1e-6
    for name, X, grad in (("q", q, g.dQ), ("k", k, g.dK), ("v", v, g.dV)):
        fd = np.zeros_like(X)
        for idx in np.ndindex(*X.shape):
            Xp = X.copy()
            Xm = X.copy()
            Xp[idx] += hstep
            Xm[idx] -= hstep
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name] = Xp
            args_m[name] = Xm
            fp = _phi_fixed_base(args_p["q"], args_p["k"], args_p["v"], dO, st, v0, R, scale)
            fm = _phi_fixed_base(args_m["q"], args_m["k"], args_m["v"], dO, st, v0, R, scale)
            fd[idx] = (fp - fm) / (2 * hstep)
        assert _rel(grad, fd) <= 1e-6, name


def _torch_tail(q, k, v, active, log_a, support, v0, R, scale):
    """The tail written independently in torch (active sub-problem only), for autodiff."""
    import torch
    idx = torch.nonzero(active).flatten()
    qa, ka, va = q[idx], k[idx], v[idx]
    sup = support[idx][:, idx]
    la = log_a[idx]
    S = scale * qa @ ka.T
    S = S.masked_fill(~sup, float("-inf"))
    vv = v0[idx]
    u = None
    for _ in range(R):
        u = la - torch.logsumexp(S + vv[None, :], dim=1)
        vv = la - torch.logsumexp(S + u[:, None], dim=0)
    P = torch.exp(S + u[:, None] + vv[None, :])
    Oa = (P @ va) / torch.exp(la)[:, None]
    O = torch.zeros(q.shape[0], v.shape[1], dtype=q.dtype)
    O = O.index_put((idx,), Oa)
    return O


@pytest.mark.parametrize("R,dustbin", [(1, False), (2, False), (4, False), (2, True)])
def test_adjoint_matches_torch_autograd(R, dustbin):
    import torch
    L, d, W = 24, 5, 6
    mask = np.ones(L, np.uint8)
    mask[[4, 5, 17]] = 0
    q, k, v, dO, kw = _unit(L=L, d=d, W=W, seed=23, mask=mask, dustbin=dustbin, mass=0.1 if dustbin else 0.0)
    scale = 0.7
    f = eo.forward_unit(q, k, v, W, T=4, R=R, scale=scale, **kw)
    g = eo.backward_unit(q, k, v, dO, f, scale)
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    O = _torch_tail(tq, tk, tv, torch.tensor(f.st.active), torch.tensor(f.st.log_a),
                    torch.tensor(f.st.support), torch.tensor(f.v_tail[0]), R, scale)
    assert _rel(O.detach().numpy(), f.O) <= 1e-13
    (O * torch.tensor(dO)).sum().backward()
    assert _rel(g.dQ, tq.grad.numpy()) <= 1e-10
    assert _rel(g.dK, tk.grad.numpy()) <= 1e-10
    assert _rel(g.dV, tv.grad.numpy()) <= 1e-10


@pytest.mark.parametrize("R", [1, 2, 4])
def test_dS_row_sums_vanish(R):
    """Adding c_i to row i of S shifts u(k)_i by -c_i at every tail step (v0 is fixed and the
    row update absorbs it), leaves every v(k) and P unchanged, so sum_j dS_ij = 0."""
    mask = np.ones(16, np.uint8)
    mask[6] = 0
    q, k, v, dO, kw = _unit(L=16, d=4, W=6, seed=7, mask=mask)
    f = eo.forward_unit(q, k, v, 6, T=2, R=R, **kw)
    g = eo.backward_unit(q, k, v, dO, f)
    scale_ref = np.max(np.abs(g.dS))
    assert np.max(np.abs(g.dS.sum(axis=1))) <= 1e-12 * max(scale_ref, 1.0) * 16


def test_R0_adjoint_is_plain_plan_gradient():
    """R = 0: nothing is differentiated through an LSE, so dS = P * dP exactly."""
    q, k, v, dO, kw = _unit(L=10, d=3, W=4, seed=9)
    f = eo.forward_unit(q, k, v, 4, T=6, R=0, **kw)
    g = eo.backward_unit(q, k, v, dO, f)
    P = eo.plan(f.S, f.u_tail[0], f.v_tail[0])
    a = np.exp(f.st.log_a)
    dP = (dO @ v.T) / a[:, None]
    assert _rel(g.dS, P * dP) <= 1e-14


# ----------------------------------------------------------------------------------------
# Closed forms and symmetries
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("R", [1, 2])
def test_W0_closed_form(R):
    """W = 0: the support is the diagonal, so after any v-update P_ii = b_i = a_i:
    O = V, dV = dO, and dS = 0 (the LSE terms cancel G exactly), so dQ = dK = 0."""
    mask = np.ones(9, np.uint8)
    mask[4] = 0
    q, k, v, dO, kw = _unit(L=9, d=3, W=0, seed=2, mask=mask)
    dO[4] = 0.0
    f = eo.forward_unit(q, k, v, 0, T=3, R=R, **kw)
    g = eo.backward_unit(q, k, v, dO, f)
    act = f.st.active
    assert np.max(np.abs(f.O[act] - v[act])) <= 1e-13
    assert np.all(f.O[~act] == 0)
    assert np.max(np.abs(g.dV[act] - dO[act])) <= 1e-13
    assert np.max(np.abs(g.dQ)) <= 1e-13 and np.max(np.abs(g.dK)) <= 1e-13


def test_reversal_symmetry():
    """The band is symmetric and the updates are index-free: reversing the token order
    reverses every output."""
    mask = np.ones(14, np.uint8)
    mask[[1, 9]] = 0
    q, k, v, dO, kw = _unit(L=14, d=4, W=5, seed=4, mask=mask)
    f = eo.forward_unit(q, k, v, 5, T=4, R=2, **kw)
    g = eo.backward_unit(q, k, v, dO, f)
    r = slice(None, None, -1)
    fr = eo.forward_unit(q[r], k[r], v[r], 5, T=4, R=2, mask_row=mask[r])
    gr = eo.backward_unit(q[r], k[r], v[r], dO[r], fr)
    assert _rel(fr.O[r], f.O) <= 1e-12
    assert _rel(fr.u_tail[:, r], f.u_tail) <= 1e-12
    assert _rel(fr.v_tail[:, r], f.v_tail) <= 1e-12
    for x, y in ((gr.dQ, g.dQ), (gr.dK, g.dK), (gr.dV, g.dV)):
        assert _rel(x[r], y) <= 1e-11


def test_row_shift_invariance():
    """An extra feature (q_i,extra = c_i / scale, k_j,extra = 1) adds c_i to row i of S:
    u shifts by -c_i at every step, v and O are unchanged."""
    L, d = 12, 3
    q, k, v, dO, kw = _unit(L=L, d=d, W=4, seed=8)
    scale = 0.6
    c = np.linspace(-1.0, 2.0, L)
    q2 = np.concatenate([q, (c / scale)[:, None]], axis=1)
    k2 = np.concatenate([k, np.ones((L, 1))], axis=1)
    f = eo.forward_unit(q, k, v, 4, T=5, R=2, scale=scale)
    f2 = eo.forward_unit(q2, k2, v, 4, T=5, R=2, scale=scale)
    assert _rel(f2.O, f.O) <= 1e-12
    assert np.max(np.abs(f2.u_tail - (f.u_tail - c[None, :]))) <= 1e-12
    assert np.max(np.abs(f2.v_tail - f.v_tail)) <= 1e-12


def test_dustbin_zero_mass_is_plain_problem():
    """BDSA §2.3 reading: with mass 0 the dustbin has a zero marginal, i.e. it is inactive,
    and the extended problem equals the plain one on the real tokens."""
    L_real, L = 13, 16
    rng = np.random.default_rng(12)
    q, k, v, dO = (rng.standard_normal((L, 3)) for _ in range(4))
    f = eo.forward_unit(q, k, v, 4, T=4, R=2, dustbin=True, dustbin_index=L_real, dustbin_mass=0.0)
    fp = eo.forward_unit(q[:L_real], k[:L_real], v[:L_real], 4, T=4, R=2)
    assert _rel(f.O[:L_real], fp.O) <= 1e-13
    assert np.all(f.O[L_real:] == 0)
    g = eo.backward_unit(q, k, v, dO, f)
    gp = eo.backward_unit(q[:L_real], k[:L_real], v[:L_real], dO[:L_real], fp)
    assert _rel(g.dQ[:L_real], gp.dQ) <= 1e-12
    assert _rel(g.dK[:L_real], gp.dK) <= 1e-12


def test_dustbin_marginals():
    """Dustbin marginal = mass; real tokens share 1 - mass uniformly (BDSA §2.3 reading)."""
    st = eo.unit_structure(10, 4, np.array([1, 1, 0, 1, 1, 1, 1, 1, 1, 1], np.uint8), True, 7, 0.1)
    a = np.exp(st.log_a)
    assert abs(a[7] - 0.1) <= 1e-16
    real = [0, 1, 3, 4, 5, 6]
    assert np.allclose(a[real], 0.9 / 6, rtol=0, atol=1e-16)
    assert not st.active[2] and not st.active[8] and not st.active[9]
    assert st.support[0, 7] and st.support[7, 0] and st.support[7, 7]
    assert not st.support[7, 8] and not st.support[0, 5]


def test_fully_masked_unit_gives_zeros():
    q, k, v, dO, kw = _unit(L=8, d=3, W=4, seed=1, mask=np.zeros(8, np.uint8))
    f = eo.forward_unit(q, k, v, 4, T=3, R=2, **kw)
    g = eo.backward_unit(q, k, v, dO, f)
    for x in (f.O, f.u_tail, f.v_tail, g.dQ, g.dK, g.dV):
        assert np.all(x == 0)


# ----------------------------------------------------------------------------------------
# Banded C twin == dense oracle
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("L,d,W,T,R,masked,dustbin", [
    (40, 4, 10, 5, 2, False, False),
    (40, 4, 10, 5, 2, True, False),
    (37, 3, 80, 3, 1, True, False),       # W >= L: full support
    (30, 5, 0, 2, 2, False, False),       # W = 0: diagonal
    (33, 4, 7, 0, 3, True, False),        # T = 0, odd W
    (48, 4, 12, 4, 4, True, True),        # dustbin + mask, R = 4
    (48, 4, 12, 4, 0, False, True),       # R = 0
])
def test_banded_matches_dense(L, d, W, T, R, masked, dustbin):
    B, H = 2, 2
    rng = np.random.default_rng(L * 7 + W)
    Q, K, V, dO = (rng.standard_normal((B, H, L, d)) for _ in range(4))
    mask = None
    if masked:
        mask = (rng.random((B, L)) > 0.2).astype(np.uint8)
    kw = dict(mask=mask, dustbin=dustbin, dustbin_index=L - 3 if dustbin else -1,
              dustbin_mass=0.1 if dustbin else 0.0)
    O, ut, vt, recs = eo.forward(Q, K, V, W, T, R, **kw)
    dQ, dK, dV = eo.backward(Q, K, V, dO, recs)
    Ob, utb, vtb = eb.forward(Q, K, V, W, T, R, **kw)
    dQb, dKb, dVb = eb.backward(Q, K, V, dO, utb, vtb, W, **kw)
    assert _rel(Ob, O) <= 1e-12
    assert np.max(np.abs(utb - ut)) <= 1e-11
    assert np.max(np.abs(vtb - vt)) <= 1e-11
    for x, y in ((dQb, dQ), (dKb, dK), (dVb, dV)):
        if np.max(np.abs(y)) == 0.0:          # W = 0: dQ = dK = 0 exactly (closed form)
            assert np.max(np.abs(x)) <= 1e-13
        else:
            assert _rel(x, y) <= 1e-11


# ----------------------------------------------------------------------------------------
# The pins bite: a planted mistake in the oracle fails them
# ----------------------------------------------------------------------------------------
def test_planted_mistakes_are_caught(monkeypatch):
    L, d, W, R = 12, 3, 4, 2
    q, k, v, dO, kw = _unit(L=L, d=d, W=W, seed=31)
    scale = 1.0 / math.sqrt(d)
    f = eo.forward_unit(q, k, v, W, T=3, R=R, scale=scale)

    def fd_err():
        g = eo.backward_unit(q, k, v, dO, f, scale)
        fd = np.zeros_like(q)
        for idx in np.ndindex(*q.shape):
            qp, qm = q.copy(), q.copy()
            qp[idx] += 1e-6
            qm[idx] -= 1e-6
            fd[idx] = (_phi_fixed_base(qp, k, v, dO, f.st, f.v_tail[0], R, scale)
                       - _phi_fixed_base(qm, k, v, dO, f.st, f.v_tail[0], R, scale)) / 2e-6
        return _rel(g.dQ, fd)

    assert fd_err() <= 1e-6
    orig = eo.tail_adjoint_dS

    def dropped_last_factor(S, st, u_tail, v_tail, V, dO_):
        dS, al, be = orig(S, st, u_tail, v_tail, V, dO_)
        a = np.exp(st.log_a)
        # put back the P(1,0) term, i.e. drop it from dS
        dS = dS + eo.plan(S, u_tail[1], v_tail[0]) * (al[1] / a)[:, None]
        return dS, al, be

    monkeypatch.setattr(eo, "tail_adjoint_dS", dropped_last_factor)
    assert fd_err() > 1e-3

    def wrong_sign(S, st, u_tail, v_tail, V, dO_):
        dS, al, be = orig(S, st, u_tail, v_tail, V, dO_)
        a = np.exp(st.log_a)
        dS = dS + 2.0 * eo.plan(S, u_tail[2], v_tail[2]) * (be[2] / a)[None, :]
        return dS, al, be

    monkeypatch.setattr(eo, "tail_adjoint_dS", wrong_sign)
    assert fd_err() > 1e-3
