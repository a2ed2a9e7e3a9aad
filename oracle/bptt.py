"""Gradients through every Sinkhorn step (no stopped base), to measure the bias of the
stop-gradient tail.

TEST INFRASTRUCTURE ONLY, under the same rules as ``eot_oracle``: only ``tests/`` may import
it; the product path never does.

Sources ("BDSA" is the technical summary "Blockwise Differentiable Sinkhorn Attention",
gist.science 2605.08123, section numbers of that page):

* BDSA §2.4, first certificate (local surrogate bias bound): when the refinement map is
  locally contractive, the gap between the full gradient through the base solve and the
  gradient of the stop-gradient surrogate shrinks geometrically with the tail depth R.
* BDSA §4.1, bias decrease: against full backpropagation through time the gradient mismatch
  falls sharply from R = 0 to R = 1 and R = 2, and R = 2 is practically as close as R = 4.

Reading (the pages give no formula): the forward is ``eot_oracle``'s, N = T + R balanced
steps from v = 0 and the output from the last potentials.  The full gradient differentiates
through all N steps; the tail gradient of depth R holds the potentials after the first T = N - R
steps constant.  For a fixed N the forward is the same function for every split, so
bias(R) = ||grad_full - grad_tail(R)|| / ||grad_full|| compares two gradients of one loss,
<O, dO>.  Reverse-mode autodiff in torch (float64, CPU) over the dense masked problem; the
support, marginals and active set come from ``eot_oracle.unit_structure``.
"""
from __future__ import annotations

import math

import numpy as np

from .eot_oracle import unit_structure


def gradient_unit(q, k, v, dO, W: int, N: int, stop_after: int | None = None, scale: float | None = None,
                  mask_row=None, dustbin: bool = False, dustbin_index: int = -1, dustbin_mass: float = 0.0,
                  dustbin_self: bool = True):
    """d<O, dO>/d(q, k, v) for one unit after N balanced steps from v = 0.

    ``stop_after=None``: through all N steps (full backpropagation).  ``stop_after=T``
    (0 <= T <= N): the potentials after T steps are constants (the stopped base); the result
    is then the tail gradient of depth N - T.  Returns (dq, dk, dv) as float64 arrays."""
    import torch

    q = np.asarray(q, np.float64)
    L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if stop_after is not None and not 0 <= stop_after <= N:
        raise ValueError("stop_after must be in [0, N]")
    st = unit_structure(L, W, mask_row, dustbin, dustbin_index, dustbin_mass, dustbin_self)
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(np.asarray(k, np.float64), requires_grad=True)
    tv = torch.tensor(np.asarray(v, np.float64), requires_grad=True)
    idx = torch.from_numpy(np.nonzero(st.active)[0])
    if idx.numel() == 0:
        z = np.zeros_like(q)
        return z, np.zeros_like(np.asarray(k, np.float64)), np.zeros_like(np.asarray(v, np.float64))
    # the active sub-problem: every active row and column holds at least one support entry
    sup = torch.from_numpy(st.support[np.ix_(st.active, st.active)])
    la = torch.from_numpy(st.log_a[st.active])
    S = scale * (tq[idx] @ tk[idx].T)
    S = torch.where(sup, S, torch.tensor(-math.inf, dtype=torch.float64))
    u = torch.zeros(idx.numel(), dtype=torch.float64)
    vv = torch.zeros(idx.numel(), dtype=torch.float64)
    for step in range(N):
        if step == stop_after:
            vv = vv.detach()
        u = la - torch.logsumexp(S + vv[None, :], dim=1)
        vv = la - torch.logsumexp(S + u[:, None], dim=0)
    if stop_after == N:
        u, vv = u.detach(), vv.detach()
    P = torch.exp(S + u[:, None] + vv[None, :])
    Oa = (P @ tv[idx]) / torch.exp(la)[:, None]
    loss = (Oa * torch.from_numpy(np.asarray(dO, np.float64)[st.active])).sum()
    loss.backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def bias_curve(q, k, v, dO, W: int, N: int, Rs=(0, 1, 2, 4), **kw):
    """{R: ||g_full - g_tail(R)|| / ||g_full||} over the stacked (dq, dk, dv) of one unit,
    plus the full gradient itself under the key "full"."""
    full = np.concatenate([g.ravel() for g in gradient_unit(q, k, v, dO, W, N, None, **kw)])
    out = {"full": full}
    for R in Rs:
        tail = np.concatenate([g.ravel() for g in gradient_unit(q, k, v, dO, W, N, N - R, **kw)])
        out[R] = float(np.linalg.norm(full - tail) / np.linalg.norm(full))
    return out
