"""A-posteriori bias certificate of the stop-gradient tail, and the tail depth chosen from it.

"Blockwise Differentiable Sinkhorn Attention" §2.4 (third certificate): measure the gradient
residual eta_R, certify that leaving the base solve's gradient out costs less than a
tolerance tau, and pick the tail depth R with it.  §4.1 reports the certificate reconstructing
the full-gradient residual and picking R = 2 at tau = 1e-5 on its synthetic problems.

Reading (the pages give no formula).  Fix the number of balanced steps N = T + R: the forward
is then the same function whatever the split.  Let g(j) be the tail gradient of depth j, i.e.
(dQ, dK, dV) from eot_sinkhorn_bwd after eot_sinkhorn_fwd with T = N - j.  g(N) differentiates
through every step, so the residual of depth R telescopes,

    g(N) - g(R) = sum_{j=R}^{N-1} delta_j,      delta_j = g(j + 1) - g(j).

The certificate measures eta_R = |delta_R| / |g(R)| and the ratio rho = eta_{R+1} / eta_R of
the next increment (three backward passes: depths R, R + 1, R + 2) and sums the remaining
N - R increments as a geometric series with that ratio:

    eta_hat_R = eta_R (1 - rho^(N - R)) / (1 - rho)       (+inf, no certificate, if rho >= 1).

With one increment left (R = N - 1) eta_hat = eta; with none (R = N) it is 0.  Where the
library's largest tail depth reaches N the exact residual |g(N) - g(R)| / |g(N)| can be measured
too.  Every norm is computed by the library (eot_sq_norms, float64 accumulation) from the
library's gradients; this module orders the calls and combines float64 scalars.

Precision: eta is a difference of two nearly equal gradients.  With float32 tensors the
gradients' own error (~1e-6 relative) is far below the increments; bfloat16 gradients are
rounded to ~4e-3 relative, which swamps the increments of all but the first depths, so run the
certificate on float32 copies of the inputs.
"""
from __future__ import annotations

import math

import torch

from . import _abi
from .api import sinkhorn_bwd, sinkhorn_fwd

MAX_TAIL_DEPTH = 8   # eot_problem.R is at most 8 (include/eot.h)

_DT = {torch.float32: _abi.EOT_FP32, torch.bfloat16: _abi.EOT_BF16}


def geometric_estimate(eta: float, rho: float | None, remaining: int) -> float:
    """eta (1 - rho^remaining) / (1 - rho): the sum of ``remaining`` increments whose norms
    start at eta and shrink by rho per step; eta itself for one increment, 0 for none, +inf
    when rho >= 1 (the increments do not shrink: no certificate)."""
    if remaining <= 0:
        return 0.0
    if remaining == 1:
        return eta
    if rho is None or not rho < 1.0:
        return math.inf
    return eta * (1.0 - rho ** remaining) / (1.0 - rho)


def tail_gradients(q, k, v, dO, W: int, N: int, R: int, **kw):
    """(dQ, dK, dV) of the depth-R tail after N = T + R balanced steps (T = N - R stopped).
    ``kw``: mask, scale, dustbin_index, dustbin_mass, dustbin_self, impl, stream, as in
    sinkhorn_fwd / sinkhorn_bwd."""
    if "ws" in kw:
        raise TypeError("the certificate sizes its own workspaces")
    if not 0 <= R <= N:
        raise ValueError("need 0 <= R <= N")
    if R > MAX_TAIL_DEPTH:
        raise ValueError(f"tail depth {R} above the library's {MAX_TAIL_DEPTH}")
    O, ut, vt = sinkhorn_fwd(q, k, v, W, N - R, R, **kw)
    return sinkhorn_bwd(q, k, v, ut, vt, dO, W, **kw)


class _Depths:
    """Tail gradients by depth for one problem, each computed once."""

    def __init__(self, q, k, v, dO, W, N, kw):
        self.args = (q, k, v, dO, W, N)
        self.kw = kw
        self.g = {}

    def __call__(self, R: int):
        if R not in self.g:
            q, k, v, dO, W, N = self.args
            self.g[R] = tail_gradients(q, k, v, dO, W, N, R, **self.kw)
        return self.g[R]


def _norms(ga, gb, stream=None):
    """(|ga - gb|^2, |ga|^2) over the three gradient tensors, by the library's kernel."""
    dev = ga[0].device
    out = torch.empty((len(ga), 2), dtype=torch.float64, device=dev)
    st = int((torch.cuda.current_stream(dev) if stream is None else stream).cuda_stream)
    for i, (a, b) in enumerate(zip(ga, gb)):
        if a.dtype not in _DT or b.dtype != a.dtype or a.shape != b.shape:
            raise TypeError("gradients must be float32 or bfloat16 tensors of one shape")
        _abi.eot_sq_norms(a.data_ptr(), b.data_ptr(), a.numel(), _DT[a.dtype], out[i].data_ptr(), st)
    torch.cuda.synchronize(dev)
    rows = out.cpu().tolist()
    return sum(r[0] for r in rows), sum(r[1] for r in rows)


def _eta(depths: _Depths, R: int, stream=None) -> float:
    d2, a2 = _norms(depths(R), depths(R + 1), stream)
    return math.sqrt(d2 / a2) if a2 > 0 else 0.0


def bias_certificate(q, k, v, dO, W: int, N: int, R: int, exact: bool = False, _depths=None, **kw) -> dict:
    """Certificate of the depth-R tail after N balanced steps (tensors as in sinkhorn_fwd).

    Returns {"R", "eta", "rho", "estimate", "exact"}: eta = |g(R+1) - g(R)| / |g(R)|, rho the
    ratio of the next increment's eta to this one (None when fewer than two increments remain),
    estimate = eta_hat_R, and with ``exact=True`` (needs N <= MAX_TAIL_DEPTH) the measured
    residual |g(N) - g(R)| / |g(N)|, else None."""
    if not 0 <= R <= N:
        raise ValueError("need 0 <= R <= N")
    depths = _depths if _depths is not None else _Depths(q, k, v, dO, W, N, kw)
    stream = kw.get("stream")
    remaining = N - R
    eta = rho = None
    if remaining >= 1:
        if R + 1 > MAX_TAIL_DEPTH:
            raise ValueError(f"the certificate of depth {R} needs a tail of depth {R + 1}")
        eta = _eta(depths, R, stream)
    if remaining >= 2 and R + 2 <= MAX_TAIL_DEPTH:
        eta1 = _eta(depths, R + 1, stream)
        rho = eta1 / eta if eta > 0 else 0.0
    estimate = geometric_estimate(eta if eta is not None else 0.0, rho, remaining)
    residual = None
    if exact:
        if N > MAX_TAIL_DEPTH:
            raise ValueError(f"the exact residual needs a tail of depth N = {N}")
        d2, a2 = _norms(depths(N), depths(R), stream)
        residual = math.sqrt(d2 / a2) if a2 > 0 else 0.0
    return {"R": R, "eta": eta, "rho": rho, "estimate": estimate, "exact": residual}


def choose_tail_depth(q, k, v, dO, W: int, N: int, tau: float = 1e-5, R_max: int | None = None, **kw):
    """The smallest tail depth R <= R_max whose certificate eta_hat_R is at most tau, with the
    certificates computed on the way; (None, certificates) when no depth qualifies.  R_max
    defaults to the deepest tail the certificate can use, min(N, MAX_TAIL_DEPTH - 1)."""
    R_max = min(N, MAX_TAIL_DEPTH - 1) if R_max is None else R_max
    depths = _Depths(q, k, v, dO, W, N, kw)
    certs = []
    for R in range(0, R_max + 1):
        c = bias_certificate(q, k, v, dO, W, N, R, _depths=depths, **kw)
        certs.append(c)
        if c["estimate"] <= tau:
            return R, certs
    return None, certs


def contraction_certificate(q, k, W: int, mask=None, scale=None, dustbin_index=None, stream=None):
    """Projective contraction certificate of the band's strictly positive blocks
    ("Blockwise Differentiable Sinkhorn Attention" §2.4, second certificate): for every pair of
    128-position tiles (I, I + o) that lies wholly inside the band, the Birkhoff-Hopf ratio
    tanh(Delta / 4) < 1 of exp(S) on the block's active real tokens (eot_contraction).

    Returns a float32 tensor [B, H, ceil(L / 128), 2 m + 1] (offset o at index o + m, -1 where
    the pair is out of range or has no active token), empty in its last dimension when the
    band is narrower than a tile."""
    from .api import _check_inputs, _stream, make_problem
    _check_inputs(q, k, k, mask)
    B, H, L, d = q.shape
    p = make_problem(B, H, L, d, W, 0, 0, q.dtype, scale, dustbin_index, 0.1 if dustbin_index is not None else 0.0)
    n = _abi.eot_contraction_offsets(p)
    if n < 0:
        raise ValueError(f"problem rejected: {_abi.eot_status_string(_abi.eot_validate(p))}")
    kappa = torch.empty((B, H, (L + 127) // 128, n), dtype=torch.float32, device=q.device)
    if n > 0 and kappa.numel() > 0:
        m = None if mask is None else mask.view(torch.uint8).data_ptr()
        _abi.eot_contraction(p, q.data_ptr(), k.data_ptr(), m, kappa.data_ptr(), _stream(stream))
    return kappa
