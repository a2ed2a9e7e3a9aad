"""PyTorch-facing helpers over libeot.  Torch supplies device memory and streams only; every
step of the forward and backward passes runs in libeot's CUDA kernels.

Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
2605.08123): §2.1 stopped base + R-step tail of balanced log-domain Sinkhorn on a fixed band
support, O = diag(1/a) P V; §2.2 exact tail adjoint; §2.3 dustbin token and fillers.
"""
from __future__ import annotations

import math

import torch

from . import _abi

_DTYPES = {torch.float32: _abi.EOT_FP32, torch.bfloat16: _abi.EOT_BF16}
_IMPLS = {"auto": _abi.EOT_IMPL_AUTO, "simt": _abi.EOT_IMPL_SIMT, "tcgen05": _abi.EOT_IMPL_TCGEN05}
TILE = 128


def make_problem(B: int, H: int, L: int, d: int, W: int, T: int, R: int, dtype: torch.dtype,
                 scale: float | None = None, dustbin_index: int | None = None, dustbin_mass: float = 0.0,
                 dustbin_self: bool = True, impl: str = "auto") -> _abi.eot_problem:
    """Fill an ``eot_problem``.  ``dustbin_index=None`` means no dustbin."""
    if dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {dtype}; use float32 or bfloat16")
    p = _abi.eot_problem()
    p.B, p.H, p.L, p.d, p.W, p.T, p.R = B, H, L, d, W, T, R
    p.dtype = _DTYPES[dtype]
    p.scale = 0.0 if scale is None else float(scale)
    p.dustbin = 0 if dustbin_index is None else 1
    p.dustbin_index = -1 if dustbin_index is None else int(dustbin_index)
    p.dustbin_mass = float(dustbin_mass)
    p.dustbin_self = int(bool(dustbin_self))
    p.impl = _IMPLS[impl]
    return p


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _check_inputs(q, k, v, mask):
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if q.shape != k.shape or q.shape != v.shape or q.dim() != 4:
        raise ValueError("q, k, v must all be [B, H, L, d] with the same shape")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise ValueError("q, k, v must share one dtype")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    if mask is not None:
        if mask.dtype not in (torch.uint8, torch.bool) or mask.shape != (q.shape[0], q.shape[2]):
            raise ValueError("mask must be uint8/bool [B, L]")
        if not mask.is_cuda or not mask.is_contiguous():
            raise ValueError("mask must be a contiguous CUDA tensor")


def workspace(p: _abi.eot_problem, backward: bool, device) -> torch.Tensor:
    n = _abi.eot_workspace_bytes(p, backward)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def sinkhorn_fwd(q, k, v, W: int, T: int, R: int, mask=None, scale=None, dustbin_index=None,
                 dustbin_mass: float = 0.0, dustbin_self: bool = True, impl: str = "auto", stream=None,
                 ws: torch.Tensor | None = None):
    """Forward pass.  Returns O [B,H,L,d] (input dtype), u_tail, v_tail [B,H,R+1,L] (fp32)."""
    _check_inputs(q, k, v, mask)
    B, H, L, d = q.shape
    p = make_problem(B, H, L, d, W, T, R, q.dtype, scale, dustbin_index, dustbin_mass, dustbin_self, impl)
    O = torch.empty_like(q)
    ut = torch.empty((B, H, R + 1, L), dtype=torch.float32, device=q.device)
    vt = torch.empty_like(ut)
    if ws is None:
        ws = workspace(p, False, q.device)
    m = None if mask is None else mask.view(torch.uint8).data_ptr()
    _abi.eot_sinkhorn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), m, O.data_ptr(), ut.data_ptr(),
                          vt.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    return O, ut, vt


def band_half_step(x, y, log_marg, pot_in, W: int, scale=None, impl: str = "auto", stream=None,
                   ws: torch.Tensor | None = None, dustbin_index: int | None = None, own=None,
                   dustbin_self: bool = True):
    """One band half-step: out[b,h,i] = log_marg[b,i] - LSE_{|i-j| <= W/2, active j}
    (scale <x_i, y_j> + pot_in[b,h,j]), 0 at inactive positions.  x, y [B,H,L,d] (fp32 or bf16,
    L a multiple of 128), log_marg [B,L] fp32 (-inf = inactive), pot_in [B,H,L] fp32.  Returns
    out [B,H,L] fp32.  Row half-step: x = q, y = k, pot_in = v; column half-step: x = k, y = q,
    pot_in = u.

    With ``dustbin_index`` D (a part of a sequence with a dustbin, eot_band_half_step_dustbin):
    real rows also sum the dustbin term, and the result is (out, part) with part [B,H,2] the
    (max, sum) partial of the dustbin's dense row over the positions ``own`` = (lo, hi)
    (default: every real position), (D, D) excluded; out[..., D] is unspecified."""
    if x.shape != y.shape or x.dim() != 4 or x.dtype != y.dtype:
        raise ValueError("x and y must be [B,H,L,d] tensors of one dtype")
    B, H, L, d = x.shape
    if log_marg.shape != (B, L) or log_marg.dtype != torch.float32:
        raise ValueError("log_marg must be a float32 [B, L] tensor")
    if pot_in.shape != (B, H, L) or pot_in.dtype != torch.float32:
        raise ValueError("pot_in must be a float32 [B, H, L] tensor")
    for t in (x, y, log_marg, pot_in):
        if not t.is_contiguous() or t.device != x.device:
            raise ValueError("inputs must be contiguous and on one device")
    if dustbin_index is None:
        p = make_problem(B, H, L, d, W, 0, 0, x.dtype, scale, impl=impl)
    else:
        # (the mass only selects the dustbin's activity in the problem; the step reads log_marg)
        p = make_problem(B, H, L, d, W, 0, 0, x.dtype, scale, dustbin_index, 0.5, dustbin_self, impl)
    out = torch.empty((B, H, L), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(p, False, x.device)
    if dustbin_index is None:
        _abi.eot_band_half_step(p, x.data_ptr(), y.data_ptr(), log_marg.data_ptr(), pot_in.data_ptr(), out.data_ptr(),
                                ws.data_ptr(), ws.numel(), _stream(stream))
        return out
    part = torch.empty((B, H, 2), dtype=torch.float32, device=x.device)
    lo, hi = own if own is not None else (0, dustbin_index)
    _abi.eot_band_half_step_dustbin(p, x.data_ptr(), y.data_ptr(), log_marg.data_ptr(), pot_in.data_ptr(),
                                    out.data_ptr(), lo, hi, part.data_ptr(), ws.data_ptr(), ws.numel(),
                                    _stream(stream))
    return out, part


def band_output(q, k, v, log_marg, u, v_pot, W: int, scale=None, impl: str = "auto", stream=None,
                ws: torch.Tensor | None = None):
    """O = diag(1/a) P V of given potentials (no dustbin): P_ij = exp(scale <q_i, k_j> + u_i +
    v_pot_j) on the band, a_i = exp(log_marg_i).  q, k, v [B,H,L,d]; log_marg [B,L] fp32;
    u, v_pot [B,H,L] fp32.  Returns O [B,H,L,d] in q's dtype."""
    if not (q.shape == k.shape == v.shape) or q.dim() != 4 or not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must be [B,H,L,d] tensors of one dtype")
    B, H, L, d = q.shape
    if log_marg.shape != (B, L) or log_marg.dtype != torch.float32:
        raise ValueError("log_marg must be a float32 [B, L] tensor")
    for t in (u, v_pot):
        if t.shape != (B, H, L) or t.dtype != torch.float32:
            raise ValueError("u and v_pot must be float32 [B, H, L] tensors")
    for t in (q, k, v, log_marg, u, v_pot):
        if not t.is_contiguous() or t.device != q.device:
            raise ValueError("inputs must be contiguous and on one device")
    p = make_problem(B, H, L, d, W, 0, 0, q.dtype, scale, impl=impl)
    O = torch.empty_like(q)
    if ws is None:
        ws = workspace(p, False, q.device)
    _abi.eot_band_output(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), log_marg.data_ptr(), u.data_ptr(),
                         v_pot.data_ptr(), O.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    return O


def sinkhorn_bwd(q, k, v, u_tail, v_tail, dO, W: int, mask=None, scale=None, dustbin_index=None,
                 dustbin_mass: float = 0.0, dustbin_self: bool = True, impl: str = "auto", stream=None,
                 ws: torch.Tensor | None = None):
    """Exact tail adjoint.  Returns dQ, dK, dV [B,H,L,d] (input dtype)."""
    _check_inputs(q, k, v, mask)
    B, H, L, d = q.shape
    R = u_tail.shape[2] - 1
    if u_tail.shape != (B, H, R + 1, L) or v_tail.shape != u_tail.shape:
        raise ValueError("u_tail / v_tail must be [B, H, R+1, L]")
    if u_tail.dtype != torch.float32 or v_tail.dtype != torch.float32:
        raise ValueError("u_tail / v_tail must be float32")
    dO = dO.contiguous()
    if dO.shape != q.shape or dO.dtype != q.dtype:
        raise ValueError("dO must match q in shape and dtype")
    p = make_problem(B, H, L, d, W, 0, R, q.dtype, scale, dustbin_index, dustbin_mass, dustbin_self, impl)
    dQ = torch.empty_like(q)
    dK = torch.empty_like(q)
    dV = torch.empty_like(q)
    if ws is None:
        ws = workspace(p, True, q.device)
    m = None if mask is None else mask.view(torch.uint8).data_ptr()
    _abi.eot_sinkhorn_bwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), m, u_tail.contiguous().data_ptr(),
                          v_tail.contiguous().data_ptr(), dO.data_ptr(), dQ.data_ptr(), dK.data_ptr(),
                          dV.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    return dQ, dK, dV


class SinkhornAttentionFn(torch.autograd.Function):
    """Autograd node: forward = base + tail + output, backward = exact tail adjoint (§2.2)."""

    @staticmethod
    def forward(ctx, q, k, v, mask, W, T, R, scale, dustbin_index, dustbin_mass, dustbin_self, impl):
        O, ut, vt = sinkhorn_fwd(q, k, v, W, T, R, mask, scale, dustbin_index, dustbin_mass, dustbin_self, impl)
        ctx.save_for_backward(q, k, v, ut, vt, mask if mask is not None else torch.empty(0))
        ctx.has_mask = mask is not None
        ctx.cfg = (W, scale, dustbin_index, dustbin_mass, dustbin_self, impl)
        return O

    @staticmethod
    def backward(ctx, dO):
        q, k, v, ut, vt, mask = ctx.saved_tensors
        W, scale, dustbin_index, dustbin_mass, dustbin_self, impl = ctx.cfg
        dQ, dK, dV = sinkhorn_bwd(q, k, v, ut, vt, dO, W, mask if ctx.has_mask else None, scale, dustbin_index,
                                  dustbin_mass, dustbin_self, impl)
        return dQ, dK, dV, None, None, None, None, None, None, None, None, None


def sinkhorn_attention(q, k, v, W: int, T: int, R: int = 2, mask=None, dustbin=None, dustbin_mass: float = 0.1,
                       scale=None, dustbin_self: bool = True, impl: str = "auto"):
    """Band Sinkhorn attention over real tokens q, k, v [B, H, N, d].

    ``dustbin`` = (q_D, k_D, v_D), each [H, d] (learned per head), appends the dustbin
    token after the N real tokens (§2.3); the sequence is padded with inactive fillers to a
    multiple of 128.  Returns O [B, H, N, d]; gradients flow to q, k, v and the dustbin
    parameters (summed over the batch)."""
    B, H, N, d = q.shape
    extra = 1 if dustbin is not None else 0
    L = ((N + extra + TILE - 1) // TILE) * TILE
    pad = L - N - extra
    parts_q, parts_k, parts_v = [q], [k], [v]
    if dustbin is not None:
        qD, kD, vD = dustbin
        parts_q.append(qD.to(q.dtype)[None, :, None, :].expand(B, H, 1, d))
        parts_k.append(kD.to(q.dtype)[None, :, None, :].expand(B, H, 1, d))
        parts_v.append(vD.to(q.dtype)[None, :, None, :].expand(B, H, 1, d))
    if pad:
        z = q.new_zeros(B, H, pad, d)
        parts_q.append(z)
        parts_k.append(z)
        parts_v.append(z)
    qe = torch.cat(parts_q, dim=2).contiguous()
    ke = torch.cat(parts_k, dim=2).contiguous()
    ve = torch.cat(parts_v, dim=2).contiguous()
    me = torch.zeros(B, L, dtype=torch.uint8, device=q.device)
    me[:, :N] = 1 if mask is None else mask.to(torch.uint8)
    O = SinkhornAttentionFn.apply(qe, ke, ve, me, W, T, R, scale, N if dustbin is not None else None,
                                  dustbin_mass, dustbin_self, impl)
    return O[:, :, :N]


def resolved_impl(B, H, L, d, W, T, R, dtype, impl="auto") -> str:
    p = make_problem(B, H, L, d, W, T, R, dtype, impl=impl)
    r = _abi.eot_resolved_impl(p)
    return {1: "simt", 2: "tcgen05"}.get(r, "unsupported")


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
