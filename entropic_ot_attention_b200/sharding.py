"""Sequence sharding of one (batch, head) unit over ranks: contiguous row ranges, with the band
neighbours' potentials exchanged after every half-step.

"Blockwise Differentiable Sinkhorn Attention" §2.1 keeps the extra state of the solve at O(L)
potentials because the support is a fixed band: position i is coupled only with |i - j| <= h,
h = W // 2.  A rank that owns positions [r0, r1) therefore needs, for its row half-steps, the
scores of its rows against the columns [r0 - h, r1 + h) and the column potentials over that
range; for its column half-steps the same with rows and columns swapped.  The Q and K rows of
that halo are copied to the rank once; after every half-step each rank sends the potentials its
neighbours' halos cover (at most h values to each side) and receives theirs, point to point.
Shards are at least h positions long, so only the two adjacent ranks exchange.

With a dustbin (§2.3) the dustbin row and column are dense: their log-sum-exp is a sum over all
positions, formed per rank as a (max, sum) partial and merged with one all-reduce of the maxima
and one of the rescaled sums per half-step (``allreduce_lse``).

Every rank takes the same collective steps in the same order.  The per-rank half-step is a
callable, so the same driver runs a rank's part of the solve wherever its scores live.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Shard:
    """Positions [r0, r1) owned by ``rank``; [c0, c1) = [max(0, r0 - h), min(L, r1 + h)) is the
    range its band reaches (its rows' columns, and its columns' rows)."""

    rank: int
    r0: int
    r1: int
    c0: int
    c1: int

    @property
    def n(self) -> int:
        return self.r1 - self.r0

    @property
    def owned(self) -> slice:
        """The owned positions inside the halo range."""
        return slice(self.r0 - self.c0, self.r1 - self.c0)


def shard_plan(L: int, W: int, world: int, align: int = 128) -> list[Shard]:
    """Split L positions into ``world`` contiguous ranges of whole ``align``-position tiles (the
    first ranks take one tile more when the tiles do not divide evenly).  Raises ValueError when
    a range would be shorter than the band's half-width h = W // 2 (then a rank's halo would
    reach past its neighbour) or empty."""
    if world < 1 or L <= 0 or L % align != 0 or W < 0:
        raise ValueError("need world >= 1, L > 0 a multiple of align, W >= 0")
    h = W // 2
    tiles = L // align
    if tiles < world:
        raise ValueError(f"{tiles} tiles cannot be shared by {world} ranks")
    base, extra = divmod(tiles, world)
    out, r0 = [], 0
    for r in range(world):
        n = (base + (1 if r < extra else 0)) * align
        r1 = r0 + n
        if world > 1 and n < h:
            raise ValueError(f"rank {r} owns {n} positions, fewer than the band half-width {h}")
        out.append(Shard(r, r0, r1, max(0, r0 - h), min(L, r1 + h)))
        r0 = r1
    return out


def halo_exchange(x_owned: torch.Tensor, plan: list[Shard], rank: int, group=None) -> torch.Tensor:
    """Potentials over this rank's halo range [c0, c1): its own values in the middle, the left
    neighbour's last values and the right neighbour's first values on the sides.  Sends this
    rank's first and last values to the neighbours whose halos reach them (send / recv pairs
    batched into one exchange)."""
    sh = plan[rank]
    out = torch.zeros(sh.c1 - sh.c0, dtype=x_owned.dtype, device=x_owned.device)
    out[sh.owned] = x_owned
    ops, recv = [], []
    if rank > 0:
        left = plan[rank - 1]
        # the left neighbour's halo reaches [left.r1, left.c1) = the first values of this rank
        n_send = left.c1 - left.r1
        if n_send > 0:
            ops.append(dist.P2POp(dist.isend, x_owned[:n_send].contiguous(), rank - 1, group))
        n_recv = sh.r0 - sh.c0
        if n_recv > 0:
            buf = torch.empty(n_recv, dtype=x_owned.dtype, device=x_owned.device)
            ops.append(dist.P2POp(dist.irecv, buf, rank - 1, group))
            recv.append((slice(0, n_recv), buf))
    if rank < len(plan) - 1:
        right = plan[rank + 1]
        n_send = right.r0 - right.c0
        if n_send > 0:
            ops.append(dist.P2POp(dist.isend, x_owned[sh.n - n_send:].contiguous(), rank + 1, group))
        n_recv = sh.c1 - sh.r1
        if n_recv > 0:
            buf = torch.empty(n_recv, dtype=x_owned.dtype, device=x_owned.device)
            ops.append(dist.P2POp(dist.irecv, buf, rank + 1, group))
            recv.append((slice(sh.r1 - sh.c0, sh.c1 - sh.c0), buf))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    for sl, buf in recv:
        out[sl] = buf
    return out


def allreduce_lse(m: torch.Tensor, s: torch.Tensor, group=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Merge per-rank log-sum-exp partials: sum_r s_r exp(m_r - M) with M = max_r m_r (one
    all-reduce of the maxima, one of the rescaled sums).  Returns (M, total); an all -inf
    partial set gives (-inf, 0)."""
    M = m.clone()
    dist.all_reduce(M, op=dist.ReduceOp.MAX, group=group)
    finite = torch.isfinite(M)
    scaled = torch.where(finite & torch.isfinite(m), s * torch.exp(m - torch.where(finite, M, torch.zeros_like(M))),
                         torch.zeros_like(s))
    dist.all_reduce(scaled, op=dist.ReduceOp.SUM, group=group)
    return M, scaled


def device_half_steps(sh: Shard, q_halo: torch.Tensor, k_halo: torch.Tensor, log_marg_halo: torch.Tensor,
                      W: int, scale: float | None = None, impl: str = "auto"):
    """``(row_step, col_step)`` for ``sharded_solve`` that run each half-step of this rank's part
    as one ``eot_band_half_step`` call on the device holding ``q_halo``.

    q_halo, k_halo: [c1 - c0, d] rows of the halo range (float32 or bfloat16, on a CUDA device);
    log_marg_halo: [c1 - c0] the whole problem's log marginals over the halo range (-inf =
    inactive).  The range is padded to whole 128-position tiles with inactive positions, which no
    band sum reads.  The steps take and return potentials in the caller's dtype and device (the
    device computes in float32); positions of the halo outside [r0, r1) come out truncated and
    are not returned."""
    from .api import band_half_step, make_problem, workspace   # needs the built library

    n = sh.c1 - sh.c0
    if q_halo.shape != k_halo.shape or q_halo.shape[0] != n or log_marg_halo.shape != (n,):
        raise ValueError("q_halo, k_halo [c1 - c0, d] and log_marg_halo [c1 - c0] expected")
    Lp = (n + 127) // 128 * 128
    dev = q_halo.device

    def pad(x):
        out = torch.zeros((1, 1, Lp, x.shape[1]), dtype=x.dtype, device=dev)
        out[0, 0, :n] = x
        return out

    q, k = pad(q_halo), pad(k_halo)
    lm = torch.full((1, Lp), float("-inf"), dtype=torch.float32, device=dev)
    lm[0, :n] = log_marg_halo.to(device=dev, dtype=torch.float32)
    ws = workspace(make_problem(1, 1, Lp, q.shape[-1], W, 0, 0, q.dtype, scale, impl=impl), False, dev)

    def step(x, y, pot_halo):
        pin = torch.zeros((1, 1, Lp), dtype=torch.float32, device=dev)
        pin[0, 0, :n] = pot_halo.to(device=dev, dtype=torch.float32)
        out = band_half_step(x, y, lm, pin, W, scale, impl, ws=ws)
        return out[0, 0, sh.owned].to(device=pot_halo.device, dtype=pot_halo.dtype)

    return (lambda v_halo: step(q, k, v_halo)), (lambda u_halo: step(k, q, u_halo))


def device_output(sh: Shard, q_halo: torch.Tensor, k_halo: torch.Tensor, v_halo: torch.Tensor,
                  log_marg_halo: torch.Tensor, u_halo: torch.Tensor, vpot_halo: torch.Tensor, W: int,
                  scale: float | None = None, impl: str = "auto") -> torch.Tensor:
    """O = diag(1/a) P V of this rank's owned rows (one ``eot_band_output`` call on the halo range,
    padded to whole tiles with inactive positions), from the potentials over the halo (u and v
    after the last half-step, exchanged with ``halo_exchange``).  q_halo, k_halo, v_halo:
    [c1 - c0, d] on a CUDA device; returns [r1 - r0, d] in their dtype on that device."""
    from .api import band_output   # needs the built library

    n = sh.c1 - sh.c0
    Lp = (n + 127) // 128 * 128
    dev = q_halo.device

    def pad(x, dtype=None):
        shape = (1, 1, Lp) + tuple(x.shape[1:])
        out = torch.zeros(shape, dtype=dtype or x.dtype, device=dev)
        out[0, 0, :n] = x.to(device=dev, dtype=dtype or x.dtype)
        return out

    lm = torch.full((1, Lp), float("-inf"), dtype=torch.float32, device=dev)
    lm[0, :n] = log_marg_halo.to(device=dev, dtype=torch.float32)
    O = band_output(pad(q_halo), pad(k_halo), pad(v_halo), lm, pad(u_halo, torch.float32),
                    pad(vpot_halo, torch.float32), W, scale, impl)
    return O[0, 0, sh.owned]


def sharded_solve(plan: list[Shard], rank: int, T: int, R: int,
                  row_step: Callable[[torch.Tensor], torch.Tensor],
                  col_step: Callable[[torch.Tensor], torch.Tensor],
                  group=None, dtype=torch.float64, device=None) -> tuple[torch.Tensor, torch.Tensor]:
    """This rank's part of the T stopped + R tail iterations (§2.1).

    ``row_step(v_halo)`` returns the owned rows' u from the column potentials over [c0, c1);
    ``col_step(u_halo)`` returns the owned columns' v from the row potentials over [c0, c1).
    Returns (u_tail, v_tail), each [R + 1, r1 - r0], in the slot layout of eot_sinkhorn_fwd:
    slot 0 the stopped base (u after T steps, 0 when T = 0; v0), slot k tail step k."""
    sh = plan[rank]
    u_tail = torch.zeros(R + 1, sh.n, dtype=dtype, device=device)
    v_tail = torch.zeros(R + 1, sh.n, dtype=dtype, device=device)
    v_halo = torch.zeros(sh.c1 - sh.c0, dtype=dtype, device=device)
    for k in range(T + R):
        u = row_step(v_halo)
        v = col_step(halo_exchange(u, plan, rank, group))
        v_halo = halo_exchange(v, plan, rank, group)
        slot = 0 if k < T else k - T + 1
        u_tail[slot] = u
        v_tail[slot] = v
    return u_tail, v_tail


def _lse_add(M: torch.Tensor, S: torch.Tensor, x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Add one term x to a (max, sum) log-sum-exp pair (elementwise)."""
    M2 = torch.maximum(M, x)
    fin = torch.isfinite(M2)
    base = torch.where(fin, M2, torch.zeros_like(M2))
    S2 = torch.where(torch.isfinite(M), S * torch.exp(M - base), torch.zeros_like(S)) + \
        torch.where(torch.isfinite(x), torch.exp(x - base), torch.zeros_like(S))
    return M2, S2


def sharded_solve_dustbin(plan: list[Shard], rank: int, T: int, R: int,
                          row_step: Callable[[torch.Tensor, torch.Tensor], tuple],
                          col_step: Callable[[torch.Tensor, torch.Tensor], tuple],
                          log_mass: float, self_score: float | None,
                          group=None, dtype=torch.float64, device=None):
    """``sharded_solve`` for a sequence with a dustbin (§2.3): the dustbin D is linked to every
    active real position, so its potentials u_D, v_D are held by every rank and its dense row and
    column are merged from per-rank partials with ``allreduce_lse``.

    ``row_step(v_halo, v_D)`` returns (u of the owned rows, their sums including the dustbin term
    S_iD + v_D; m, s) with (m, s) the (max, sum) partial of S_Dc + v_c over the owned active
    columns c; ``col_step(u_halo, u_D)`` the same with rows and columns swapped.  ``log_mass`` is
    log b_D = log a_D; ``self_score`` is S_DD when (D, D) is in the support, else None.  Returns
    (u_tail, v_tail, uD_tail, vD_tail): the owned potentials [R + 1, r1 - r0] and the dustbin's
    [R + 1], slot layout of eot_sinkhorn_fwd."""
    sh = plan[rank]
    u_tail = torch.zeros(R + 1, sh.n, dtype=dtype, device=device)
    v_tail = torch.zeros(R + 1, sh.n, dtype=dtype, device=device)
    uD_tail = torch.zeros(R + 1, dtype=dtype, device=device)
    vD_tail = torch.zeros(R + 1, dtype=dtype, device=device)
    v_halo = torch.zeros(sh.c1 - sh.c0, dtype=dtype, device=device)
    vD = torch.zeros(1, dtype=dtype, device=device)

    def dense(m, s, other_D):
        M, S = allreduce_lse(m.reshape(1).to(dtype), s.reshape(1).to(dtype), group)
        if self_score is not None:
            M, S = _lse_add(M, S, self_score + other_D)
        lse = torch.where(S > 0, M + torch.log(torch.where(S > 0, S, torch.ones_like(S))),
                          torch.full_like(S, float("-inf")))
        return log_mass - lse

    for k in range(T + R):
        u, m, s_ = row_step(v_halo, vD)
        uD = dense(m, s_, vD)
        v, m, s_ = col_step(halo_exchange(u, plan, rank, group), uD)
        vD = dense(m, s_, uD)
        v_halo = halo_exchange(v, plan, rank, group)
        slot = 0 if k < T else k - T + 1
        u_tail[slot] = u
        v_tail[slot] = v
        uD_tail[slot] = uD[0]
        vD_tail[slot] = vD[0]
    return u_tail, v_tail, uD_tail, vD_tail


def device_half_steps_dustbin(sh: Shard, q_halo: torch.Tensor, k_halo: torch.Tensor, q_dust: torch.Tensor,
                              k_dust: torch.Tensor, log_marg_halo: torch.Tensor, log_mass: float, W: int,
                              scale: float | None = None, impl: str = "auto"):
    """``(row_step, col_step)`` for ``sharded_solve_dustbin`` on the device holding ``q_halo``:
    each step is one ``eot_band_half_step_dustbin`` call on the halo range padded to whole tiles,
    followed by a tile holding the dustbin (its q and k rows ``q_dust``, ``k_dust`` [d]) and
    inactive fillers; the dustbin's partial covers the owned positions only."""
    from .api import band_half_step, make_problem, workspace   # needs the built library

    n = sh.c1 - sh.c0
    if q_halo.shape != k_halo.shape or q_halo.shape[0] != n or log_marg_halo.shape != (n,):
        raise ValueError("q_halo, k_halo [c1 - c0, d] and log_marg_halo [c1 - c0] expected")
    D = (n + 127) // 128 * 128
    Lp = D + 128
    dev = q_halo.device

    def pad(x, xd):
        out = torch.zeros((1, 1, Lp, x.shape[1]), dtype=x.dtype, device=dev)
        out[0, 0, :n] = x
        out[0, 0, D] = xd.to(device=dev, dtype=x.dtype)
        return out

    q, k = pad(q_halo, q_dust), pad(k_halo, k_dust)
    lm = torch.full((1, Lp), float("-inf"), dtype=torch.float32, device=dev)
    lm[0, :n] = log_marg_halo.to(device=dev, dtype=torch.float32)
    lm[0, D] = float(log_mass)
    ws = workspace(make_problem(1, 1, Lp, q.shape[-1], W, 0, 0, q.dtype, scale, D, 0.5, True, impl), False, dev)
    own = (sh.owned.start, sh.owned.stop)

    def step(x, y, pot_halo, pot_D):
        pin = torch.zeros((1, 1, Lp), dtype=torch.float32, device=dev)
        pin[0, 0, :n] = pot_halo.to(device=dev, dtype=torch.float32)
        pin[0, 0, D] = pot_D.reshape(()).to(device=dev, dtype=torch.float32)
        out, part = band_half_step(x, y, lm, pin, W, scale, impl, ws=ws, dustbin_index=D, own=own)
        part = part[0, 0].to(device=pot_halo.device, dtype=pot_halo.dtype)
        return out[0, 0, sh.owned].to(device=pot_halo.device, dtype=pot_halo.dtype), part[0], part[1]

    return (lambda v_halo, v_D: step(q, k, v_halo, v_D)), (lambda u_halo, u_D: step(k, q, u_halo, u_D))
