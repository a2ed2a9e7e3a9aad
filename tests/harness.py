"""Shared test helpers: run a seeded case through the C ABI on the GPU and through the
float64 oracle, and compare them element by element over active entries."""
from __future__ import annotations

import numpy as np

import eot_inputs
from oracle import banded as eb
from oracle import eot_oracle as eo

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def rel_err(x, ref, active_rows=None):
    """||x - ref||_inf / ||ref||_inf over active entries (inactive entries must match too).

    A reference that is identically zero (e.g. v and dQ, dK for W = 0, where the closed form
    gives exact zeros) has no relative error; the absolute error is returned instead."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(x - ref))) if ref.size else 0.0
    return err / den if den > 0.0 else err


def oracle_run(case: eot_inputs.Case, units=None, use_banded=False):
    """Oracle forward + backward.  ``units``: list of flattened b*H+h to compute (others 0)."""
    Q = case.Q.astype(np.float64)
    K = case.K.astype(np.float64)
    V = case.V.astype(np.float64)
    dO = case.dO.astype(np.float64)
    kw = case.oracle_kwargs()
    B, H = Q.shape[:2]
    if use_banded:
        O, ut, vt = eb.forward(Q, K, V, units=units, **kw)
        kwb = {k: v for k, v in kw.items() if k not in ("T", "R")}
        dQ, dK, dV = eb.backward(Q, K, V, dO, ut, vt, units=units, **kwb)
    else:
        us = None if units is None else [(u // H, u % H) for u in units]
        O, ut, vt, recs = eo.forward(Q, K, V, units=us, **kw)
        dQ, dK, dV = eo.backward(Q, K, V, dO, recs, scale=case.scale)
    return dict(O=O, u=ut, v=vt, dQ=dQ, dK=dK, dV=dV)


def gpu_run(case: eot_inputs.Case, impl="auto", u_tail=None, v_tail=None):
    """Forward + backward through the C ABI on cuda:0.  Optionally feed the backward a given
    (oracle) tail instead of the GPU forward's."""
    import torch
    from entropic_ot_attention_b200 import sinkhorn_bwd, sinkhorn_fwd
    dev = torch.device("cuda:0")
    tdt = torch.float32 if case.dtype == "fp32" else torch.bfloat16
    q, k, v, dO = (torch.from_numpy(x).to(dev).to(tdt).contiguous() for x in (case.Q, case.K, case.V, case.dO))
    mask = None if case.mask is None else torch.from_numpy(case.mask).to(dev)
    dbi = case.dustbin_index if case.dustbin else None
    O, ut, vt = sinkhorn_fwd(q, k, v, case.W, case.T, case.R, mask, case.scale, dbi, case.dustbin_mass, impl=impl)
    if u_tail is not None:
        ut = torch.from_numpy(np.ascontiguousarray(u_tail, np.float32)).to(dev)
        vt = torch.from_numpy(np.ascontiguousarray(v_tail, np.float32)).to(dev)
    dQ, dK, dV = sinkhorn_bwd(q, k, v, ut, vt, dO, case.W, mask, case.scale, dbi, case.dustbin_mass, impl=impl)
    torch.cuda.synchronize()
    f = lambda t: t.float().cpu().numpy().astype(np.float64)
    return dict(O=f(O), u=f(ut), v=f(vt), dQ=f(dQ), dK=f(dK), dV=f(dV))


def compare(gpu: dict, orc: dict, units=None, H=None, keys=("O", "u", "v", "dQ", "dK", "dV")):
    """Per-tensor relative max error, restricted to the computed units."""
    errs = {}
    for k in keys:
        g, o = gpu[k], orc[k]
        if units is not None:
            g = np.stack([g[u // H, u % H] for u in units])
            o = np.stack([o[u // H, u % H] for u in units])
        errs[k] = rel_err(g, o) if k not in ("u", "v") else pot_err(g, o)
    return errs


def pot_err(x, ref):
    """Error of log-domain potentials: ||x - ref||_inf / max(||ref||_inf, 1).  A potential is a
    log-scaling; an absolute error e changes the plan entries by a factor exp(e), so below a
    magnitude of 1 the absolute error is the meaningful measure (W = 0 gives v = 0 exactly)."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(float(np.max(np.abs(ref))), 1.0))
