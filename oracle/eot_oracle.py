"""Float64 CPU oracle for blockwise, fixed-support, balanced log-domain Sinkhorn attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The product path (``entropic_ot_attention_b200``) never imports, links or executes
anything under ``oracle/``; the two share no code.

Sources.  "BDSA" below is the technical summary "Blockwise Differentiable Sinkhorn
Attention" (gist.science, paper 2605.08123; the same text exists in Korean, Japanese and
Italian).  Section numbers are that page's:

* BDSA §2.1 Forward: fixed active support Omega of band width W, entropic temperature
  absorbed into the score matrix S, a stopped (stop-gradient) balanced Sinkhorn base of
  T steps giving (u0, v0), then an R-step differentiable refinement tail.
* BDSA §2.2 R=2 staircase: the exact tail adjoint needs the plan factors
  P(2,2), P(2,1), P(1,1), P(1,0), and every P(a,b) equals
  P(2,2) * exp(u(a) - u(2)) * exp(v(b) - v(2)) (the scaling-orbit identity).
* BDSA §2.3 Dustbin bridge: a learned dustbin token plus inactive fillers are appended
  to Q/K/V and the same balanced solver runs on the extended state space.

The pages state the method in words; the concrete equations below are the plainest
reading of them:

* score      S_ij = scale * <q_i, k_j>, scale = 1/sqrt(d) by default (temperature absorbed)
* support    Omega = {(i, j) : i, j active, |i - j| <= W // 2}; with a dustbin D also
             (i, D), (D, j) for every active real i, j, and (D, D)
* marginals  uniform over the active real tokens; with a dustbin a_D = b_D = mass and
             the real tokens share 1 - mass
* one step   u_i = log a_i - LSE_{j:(i,j) in Omega}(S_ij + v_j), then
             v_j = log b_j - LSE_{i:(i,j) in Omega}(S_ij + u_i)
* base       v = 0, then T steps; (u0, v0) is the state after them (u0 = v0 = 0 if T = 0)
* tail       R more steps from v0, giving u(k), v(k) for k = 1..R
* output     P = exp(S + u(R) + v(R)) on Omega, O = diag(1/a) P V

Everything is dense L x L float64 with -inf outside Omega: slow and obviously checkable.
Arrays for one (batch, head) unit are [L, d]; the batched helpers loop over units.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------------------
# Problem structure: active set, marginals, support (BDSA §2.1, §2.3)
# ----------------------------------------------------------------------------------------
@dataclass
class UnitStructure:
    """Active flags, log-marginals and the dense support of one unit (one sequence)."""

    active: np.ndarray      # bool [L]
    log_a: np.ndarray       # float64 [L]; -inf where inactive (a == b: balanced, same mask)
    support: np.ndarray     # bool [L, L]
    dustbin_index: int      # -1 when there is no (active) dustbin


def unit_structure(L: int, W: int, mask_row=None, dustbin: bool = False,
                   dustbin_index: int = -1, dustbin_mass: float = 0.0,
                   dustbin_self: bool = True) -> UnitStructure:
    """Build the active set, uniform marginals and support for one sequence.

    BDSA §2.1: a fixed support of band width W; the band is taken as |i - j| <= W // 2
    on token positions, restricted to active tokens.  Marginals are uniform over the
    active tokens (balanced OT, a == b).
    BDSA §2.3: the dustbin token is appended after the real tokens and is linked to every
    active real token in both directions (plus itself when ``dustbin_self``); fillers after
    it are inactive (zero marginal, no support).  Mass 0 makes the dustbin inactive.
    """
    if W < 0:
        raise ValueError("W must be >= 0")
    h = W // 2
    real = np.ones(L, dtype=bool) if mask_row is None else np.asarray(mask_row).astype(bool).copy()
    D = -1
    if dustbin:
        if not (0 <= dustbin_index < L):
            raise ValueError("dustbin_index out of range")
        real[dustbin_index:] = False          # the dustbin itself and the fillers after it
        D = dustbin_index
    n_real = int(real.sum())
    active = real.copy()
    log_a = np.full(L, NEG_INF)
    use_dustbin = dustbin and n_real > 0 and dustbin_mass > 0.0
    if n_real > 0:
        real_mass = (1.0 - dustbin_mass) if use_dustbin else 1.0
        log_a[real] = math.log(real_mass / n_real)
    if use_dustbin:
        active[D] = True
        log_a[D] = math.log(dustbin_mass)
    else:
        D = -1
    idx = np.arange(L)
    band = np.abs(idx[:, None] - idx[None, :]) <= h
    support = band & real[:, None] & real[None, :]
    if D >= 0:
        support[real, D] = True
        support[D, real] = True
        if dustbin_self:
            support[D, D] = True
    return UnitStructure(active=active, log_a=log_a, support=support, dustbin_index=D)


def scores(q: np.ndarray, k: np.ndarray, scale: float, support: np.ndarray) -> np.ndarray:
    """S_ij = scale * <q_i, k_j> on the support, -inf elsewhere (BDSA §2.1: epsilon absorbed)."""
    S = scale * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)
    return np.where(support, S, NEG_INF)


def lse(x: np.ndarray, axis: int) -> np.ndarray:
    """Textbook log-sum-exp with the max shift; an all -inf slice gives -inf."""
    m = np.max(x, axis=axis, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    with np.errstate(divide="ignore"):
        s = np.log(np.sum(np.exp(x - m_safe), axis=axis, keepdims=True)) + m_safe
    return np.squeeze(s, axis=axis)


# ----------------------------------------------------------------------------------------
# One balanced Sinkhorn step (BDSA §2.1)
# ----------------------------------------------------------------------------------------
def row_step(S: np.ndarray, log_a: np.ndarray, v: np.ndarray, active: np.ndarray) -> np.ndarray:
    """u_i = log a_i - LSE_j (S_ij + v_j); inactive rows get 0."""
    with np.errstate(invalid="ignore"):
        u = log_a - lse(S + v[None, :], axis=1)
    return np.where(active, u, 0.0)


def col_step(S: np.ndarray, log_b: np.ndarray, u: np.ndarray, active: np.ndarray) -> np.ndarray:
    """v_j = log b_j - LSE_i (S_ij + u_i); inactive columns get 0."""
    with np.errstate(invalid="ignore"):
        v = log_b - lse(S + u[:, None], axis=0)
    return np.where(active, v, 0.0)


def plan(S: np.ndarray, u: np.ndarray, v: np.ndarray) -> np.ndarray:
    """P = exp(S + u 1^T + 1 v^T) on the support (0 elsewhere, since S = -inf there)."""
    return np.exp(S + u[:, None] + v[None, :])


# ----------------------------------------------------------------------------------------
# Forward: stopped base + R-step tail + output (BDSA §2.1)
# ----------------------------------------------------------------------------------------
@dataclass
class UnitForward:
    O: np.ndarray           # [L, dv]
    u_tail: np.ndarray      # [R+1, L]: u_tail[0] = base u (u(T)), u_tail[k] = u(k)
    v_tail: np.ndarray      # [R+1, L]: v_tail[0] = stopped base v (v0), v_tail[k] = v(k)
    S: np.ndarray
    st: UnitStructure


def base_solve(S: np.ndarray, st: UnitStructure, T: int):
    """T stopped balanced steps from v = 0 (BDSA §2.1, stopped base).  Returns (u0, v0)."""
    L = S.shape[0]
    u = np.zeros(L)
    v = np.zeros(L)
    for _ in range(T):
        u = row_step(S, st.log_a, v, st.active)
        v = col_step(S, st.log_a, u, st.active)
    return u, v


def tail_solve(S: np.ndarray, st: UnitStructure, v0: np.ndarray, R: int):
    """R differentiable steps from the stopped v0 (BDSA §2.1, refinement tail).

    Returns lists us, vs with us[k] = u(k), vs[k] = v(k) for k = 1..R (index 0 unused)."""
    us = [None]
    vs = [v0]
    v = v0
    for _ in range(R):
        u = row_step(S, st.log_a, v, st.active)
        v = col_step(S, st.log_a, u, st.active)
        us.append(u)
        vs.append(v)
    return us, vs


def output(S: np.ndarray, st: UnitStructure, u: np.ndarray, v: np.ndarray, V: np.ndarray) -> np.ndarray:
    """O = diag(1/a) P V with P = exp(S + u + v); inactive rows are 0."""
    P = plan(S, u, v)
    a = np.exp(st.log_a)
    O = np.zeros((S.shape[0], V.shape[1]))
    act = st.active
    O[act] = (P[act] @ np.asarray(V, np.float64)) / a[act, None]
    return O


def forward_unit(q, k, v, W: int, T: int, R: int, scale: float | None = None, mask_row=None,
                 dustbin: bool = False, dustbin_index: int = -1, dustbin_mass: float = 0.0,
                 dustbin_self: bool = True) -> UnitForward:
    """Full forward for one unit: base (stopped), tail, output."""
    q = np.asarray(q, np.float64)
    L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    st = unit_structure(L, W, mask_row, dustbin, dustbin_index, dustbin_mass, dustbin_self)
    S = scores(q, k, scale, st.support)
    u0, v0 = base_solve(S, st, T)
    us, vs = tail_solve(S, st, v0, R)
    uR = us[R] if R > 0 else u0
    vR = vs[R]
    O = output(S, st, uR, vR, v)
    u_tail = np.stack([u0] + us[1:]) if R > 0 else u0[None, :]
    v_tail = np.stack(vs)
    return UnitForward(O=O, u_tail=u_tail, v_tail=v_tail, S=S, st=st)


# ----------------------------------------------------------------------------------------
# Exact tail adjoint (BDSA §2.2), hand-written
# ----------------------------------------------------------------------------------------
@dataclass
class UnitBackward:
    dQ: np.ndarray
    dK: np.ndarray
    dV: np.ndarray
    dS: np.ndarray
    alpha: list             # alpha[k] = adjoint of u(k), k = 1..R (index 0 unused)
    beta: list              # beta[k]  = adjoint of v(k), k = 1..R (index 0 unused)


def tail_adjoint_dS(S: np.ndarray, st: UnitStructure, u_tail: np.ndarray, v_tail: np.ndarray,
                    V: np.ndarray, dO: np.ndarray):
    """Adjoint of Phi = <dO, O> w.r.t. S through the R-step tail, base held fixed.

    Derivative facts (from the step equations of BDSA §2.1):
      dv(k)_j / dS_ij = dv(k)_j / du(k)_i   = -P(k,k)_ij   / b_j
      du(k)_i / dS_ij = du(k)_i / dv(k-1)_j = -P(k,k-1)_ij / a_i
    Chain, output first:
      dP_ij  = <dO_i, V_j> / a_i,   G = P(R,R) * dP
      beta_R = colsum G,            alpha_R = rowsum G - P(R,R) (beta_R / b)
      k = R-1 .. 1:  beta_k  = -P(k+1,k)^T (alpha_{k+1} / a)
                     alpha_k = -P(k,k) (beta_k / b)
      dS = G - sum_k [ P(k,k) * 1 (beta_k/b)^T + P(k,k-1) * (alpha_k/a) 1^T ]
    For R = 2 the factors are P(2,2), P(2,1), P(1,1), P(1,0): BDSA §2.2's staircase.
    The factors are built directly from the stored potentials here; the orbit form is
    checked separately (``orbit_plan``, ``tail_adjoint_dS_orbit``).
    """
    R = u_tail.shape[0] - 1
    a = np.exp(st.log_a)
    b = a
    act = st.active
    inv_a = np.where(act, 1.0 / np.where(act, a, 1.0), 0.0)
    inv_b = inv_a
    V = np.asarray(V, np.float64)
    dO = np.asarray(dO, np.float64)

    def P(ai, bi):
        return plan(S, u_tail[ai], v_tail[bi])

    PRR = P(R, R)
    dP = (dO @ V.T) * inv_a[:, None]
    G = PRR * dP
    if R == 0:
        return G, [None], [None]
    alpha = [None] * (R + 1)
    beta = [None] * (R + 1)
    beta[R] = G.sum(axis=0)
    alpha[R] = G.sum(axis=1) - PRR @ (beta[R] * inv_b)
    for kk in range(R - 1, 0, -1):
        beta[kk] = -(P(kk + 1, kk).T @ (alpha[kk + 1] * inv_a))
        alpha[kk] = -(P(kk, kk) @ (beta[kk] * inv_b))
    dS = G.copy()
    for kk in range(1, R + 1):
        dS -= P(kk, kk) * (beta[kk] * inv_b)[None, :]
        dS -= P(kk, kk - 1) * (alpha[kk] * inv_a)[:, None]
    return dS, alpha, beta


def orbit_plan(S, u_tail, v_tail, ai: int, bi: int) -> np.ndarray:
    """P(a,b) rebuilt from the single reference P(R,R) (BDSA §2.2 scaling-orbit identity)."""
    R = u_tail.shape[0] - 1
    PRR = plan(S, u_tail[R], v_tail[R])
    return PRR * np.exp(u_tail[ai] - u_tail[R])[:, None] * np.exp(v_tail[bi] - v_tail[R])[None, :]


def tail_adjoint_dS_orbit(S, st, u_tail, v_tail, V, dO):
    """Same dS as ``tail_adjoint_dS`` but in the single-reference-tile form (BDSA §2.2).

    dS = P(R,R) * (dP - sum_m x_m y_m^T), with, for k = 1..R,
      x = exp(u(k)-u(R)),               y = exp(v(k)-v(R)) * beta_k / b
      x = exp(u(k)-u(R)) * alpha_k / a, y = exp(v(k-1)-v(R)).
    alpha, beta are taken from ``tail_adjoint_dS`` (the vectors, not the factors)."""
    R = u_tail.shape[0] - 1
    _, alpha, beta = tail_adjoint_dS(S, st, u_tail, v_tail, V, dO)
    act = st.active
    a = np.exp(st.log_a)
    inv_a = np.where(act, 1.0 / np.where(act, a, 1.0), 0.0)
    PRR = plan(S, u_tail[R], v_tail[R])
    dP = (np.asarray(dO, np.float64) @ np.asarray(V, np.float64).T) * inv_a[:, None]
    M = dP.copy()
    for kk in range(1, R + 1):
        x1 = np.exp(u_tail[kk] - u_tail[R])
        y1 = np.exp(v_tail[kk] - v_tail[R]) * beta[kk] * inv_a
        x2 = np.exp(u_tail[kk] - u_tail[R]) * alpha[kk] * inv_a
        y2 = np.exp(v_tail[kk - 1] - v_tail[R])
        M -= np.outer(x1, y1) + np.outer(x2, y2)
    return PRR * M


def backward_unit(q, k, v, dO, fwd: UnitForward, scale: float | None = None) -> UnitBackward:
    """dQ = scale dS K, dK = scale dS^T Q, dV = P(R,R)^T (dO / a)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    V = np.asarray(v, np.float64)
    dO = np.asarray(dO, np.float64)
    L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    st = fwd.st
    R = fwd.u_tail.shape[0] - 1
    dS, alpha, beta = tail_adjoint_dS(fwd.S, st, fwd.u_tail, fwd.v_tail, V, dO)
    act = st.active
    a = np.exp(st.log_a)
    inv_a = np.where(act, 1.0 / np.where(act, a, 1.0), 0.0)
    PRR = plan(fwd.S, fwd.u_tail[R], fwd.v_tail[R])
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    dV = PRR.T @ (dO * inv_a[:, None])
    return UnitBackward(dQ=dQ, dK=dK, dV=dV, dS=dS, alpha=alpha, beta=beta)


# ----------------------------------------------------------------------------------------
# Batched helpers over [B, H, L, d]
# ----------------------------------------------------------------------------------------
def forward(Q, K, V, W, T, R, scale=None, mask=None, dustbin=False, dustbin_index=-1,
            dustbin_mass=0.0, dustbin_self=True, units=None):
    """Loop ``forward_unit`` over (b, h).  Returns O [B,H,L,d], u_tail/v_tail [B,H,R+1,L]
    and the per-unit records.  ``units`` restricts the work to a list of (b, h)."""
    B, H, L, d = Q.shape
    O = np.zeros((B, H, L, V.shape[-1]))
    ut = np.zeros((B, H, R + 1, L))
    vt = np.zeros((B, H, R + 1, L))
    recs = {}
    todo = units if units is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in todo:
        m = None if mask is None else mask[b]
        f = forward_unit(Q[b, h], K[b, h], V[b, h], W, T, R, scale, m, dustbin, dustbin_index,
                         dustbin_mass, dustbin_self)
        O[b, h], ut[b, h], vt[b, h] = f.O, f.u_tail, f.v_tail
        recs[(b, h)] = f
    return O, ut, vt, recs


def backward(Q, K, V, dO, recs, scale=None):
    """Loop ``backward_unit`` over the units present in ``recs``."""
    dQ = np.zeros(Q.shape)
    dK = np.zeros(K.shape)
    dV = np.zeros(V.shape)
    for (b, h), f in recs.items():
        g = backward_unit(Q[b, h], K[b, h], V[b, h], dO[b, h], f, scale)
        dQ[b, h], dK[b, h], dV[b, h] = g.dQ, g.dK, g.dV
    return dQ, dK, dV
