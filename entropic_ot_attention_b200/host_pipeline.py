"""Forward + backward on inputs held in pinned host memory, with the host <-> device copies
overlapped with the kernels.

The (batch, head) units of a problem are independent (each has its own potentials and band),
so a step over B x H units can run as a sequence of smaller problems: chunks of whole batch
rows, or of heads of one batch row.  Three CUDA streams carry the chunks through copy-in, compute
(eot_sinkhorn_fwd then eot_sinkhorn_bwd through the C ABI) and copy-out; two device staging
slots alternate, so chunk c + 1's inputs arrive and chunk c - 1's results leave while chunk c
computes.  Within a chunk the forward starts once Q, K and V are in (dO, which only the backward
reads, arrives meanwhile) and O leaves while the backward runs.  Every step of the method still
runs in libeot's kernels; this module only moves data and orders the streams.
"""
from __future__ import annotations

import torch

from . import _abi
from .api import make_problem, workspace


def plan_chunks(B: int, H: int, heads_per_chunk: int | None = None, rows_per_chunk: int | None = None,
                target_chunks: int = 4) -> tuple[int | None, int]:
    """(rows_per_chunk, heads_per_chunk) of a step: rows_per_chunk is None when a chunk is
    heads_per_chunk heads of one batch row; else a chunk is that many whole rows (all H heads).
    With neither given: about ``target_chunks`` chunks, of whole rows when B >= target_chunks
    (a short problem's per-call latency is then paid once per chunk, not once per unit), else
    of the most heads of one row that still give that many chunks."""
    if heads_per_chunk is not None and rows_per_chunk is not None:
        raise ValueError("give heads_per_chunk or rows_per_chunk, not both")
    if heads_per_chunk is None and rows_per_chunk is None:
        if B >= target_chunks:
            rows_per_chunk = -(-B // target_chunks)
        else:
            heads_per_chunk = next((hc for hc in range(H, 0, -1)
                                    if H % hc == 0 and B * (H // hc) >= target_chunks), 1)
    if rows_per_chunk is not None:
        if not 1 <= rows_per_chunk <= B:
            raise ValueError("rows_per_chunk must be in [1, B]")
        return rows_per_chunk, H
    if heads_per_chunk < 1 or H % heads_per_chunk != 0:
        raise ValueError("heads_per_chunk must divide H")
    return None, heads_per_chunk


def chunk_list(B: int, H: int, rows: int | None, hc: int) -> list[tuple[int, int, int, int]]:
    """(b0, b1, h0, h1) of every chunk of a plan, in order; together they cover every unit once."""
    if rows is not None:
        return [(b0, min(B, b0 + rows), 0, H) for b0 in range(0, B, rows)]
    return [(b, b + 1, h0, h0 + hc) for b in range(B) for h0 in range(0, H, hc)]


class HostStep:
    """One forward + backward over host tensors q, k, v, dO [B, H, L, d] (pinned), writing
    O, dQ, dK, dV [B, H, L, d] (pinned) back to the host.

    A chunk is either ``rows_per_chunk`` whole batch rows (all heads) or ``heads_per_chunk``
    heads of one batch row; with neither given, ``plan_chunks`` picks about ``target_chunks``
    chunks.  The mask, if any, is a host or device uint8 [B, L] fixed at construction; the
    dustbin arguments are those of ``sinkhorn_fwd``."""

    def __init__(self, B: int, H: int, L: int, d: int, W: int, T: int, R: int, dtype: torch.dtype,
                 scale=None, mask=None, heads_per_chunk: int | None = None, rows_per_chunk: int | None = None,
                 device=None, impl: str = "auto", target_chunks: int = 4, dustbin_index: int | None = None,
                 dustbin_mass: float = 0.0, dustbin_self: bool = True):
        self.rows, self.hc = plan_chunks(B, H, heads_per_chunk, rows_per_chunk, target_chunks)
        self.B, self.H, self.L, self.d, self.R = B, H, L, d, R
        self.dev = torch.device("cuda") if device is None else torch.device(device)
        self._args = (L, d, W, T, R, dtype, scale, dustbin_index, dustbin_mass, dustbin_self)
        self._impl = impl
        self._problems = {}
        nb_max = 1 if self.rows is None else self.rows
        self.p = self.problem(nb_max, self.hc)   # the largest chunk: sizes the slots' buffers
        self.mask = None if mask is None else mask.to(self.dev, torch.uint8).contiguous()
        shape = (nb_max, self.hc, L, d)
        tshape = (nb_max, self.hc, R + 1, L)
        self.slots = []
        for _ in range(2):
            s = {name: torch.empty(shape, dtype=dtype, device=self.dev)
                 for name in ("q", "k", "v", "dO", "O", "dQ", "dK", "dV")}
            s["ut"] = torch.empty(tshape, dtype=torch.float32, device=self.dev)
            s["vt"] = torch.empty(tshape, dtype=torch.float32, device=self.dev)
            s["wsf"] = workspace(self.p, False, self.dev)
            s["wsb"] = workspace(self.p, True, self.dev)
            self.slots.append(s)
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(self.dev) for _ in range(3))
        self.ev_comp = [torch.cuda.Event() for _ in range(2)]
        self.ev_fwd = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.ev_in = [torch.cuda.Event() for _ in range(2)]       # Q, K, V of the slot are in
        self.ev_in_dO = [torch.cuda.Event() for _ in range(2)]
        self.c = 0   # running chunk counter (slot = counter % 2)

    def problem(self, nb: int, nh: int):
        """The problem of one chunk of nb batch rows x nh heads (validated once per shape)."""
        key = (nb, nh)
        if key not in self._problems:
            L, d, W, T, R, dtype, scale, dbi, dbm, dbs = self._args
            p = make_problem(nb, nh, L, d, W, T, R, dtype, scale, dbi, dbm, dbs, impl=self._impl)
            st = _abi.eot_validate(p)
            if st != 0:
                raise ValueError(f"problem rejected: {_abi.eot_status_string(st)}")
            self._problems[key] = p
        return self._problems[key]

    def chunks(self):
        """(b0, b1, h0, h1) of every chunk, in order."""
        return chunk_list(self.B, self.H, self.rows, self.hc)

    def run(self, hq, hk, hv, hdO, hO, hdQ, hdK, hdV):
        """Enqueue one step; returns at once (synchronise ``s_out`` or the device to wait)."""
        for b0, b1, h0, h1 in self.chunks():
            nb, nh = b1 - b0, h1 - h0
            p = self.problem(nb, nh)
            i = self.c % 2
            s = {name: t[:nb] for name, t in self.slots[i].items() if name not in ("wsf", "wsb")}
            ws = self.slots[i]
            first_use = self.c < 2
            # inputs of this slot are free once the compute two chunks back has finished
            with torch.cuda.stream(self.s_in):
                if not first_use:
                    self.s_in.wait_event(self.ev_comp[i])
                for name, src in (("q", hq), ("k", hk), ("v", hv)):
                    s[name].copy_(src[b0:b1, h0:h1], non_blocking=True)
                self.ev_in[i].record(self.s_in)
                s["dO"].copy_(hdO[b0:b1, h0:h1], non_blocking=True)
                self.ev_in_dO[i].record(self.s_in)
            # outputs of this slot are free once the copy-out two chunks back has finished
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(self.ev_in[i])
                if not first_use:
                    self.s_comp.wait_event(self.ev_out[i])
                sp = int(self.s_comp.cuda_stream)
                m = None if self.mask is None else self.mask[b0:b1].data_ptr()
                _abi.eot_sinkhorn_fwd(p, s["q"].data_ptr(), s["k"].data_ptr(), s["v"].data_ptr(), m,
                                      s["O"].data_ptr(), s["ut"].data_ptr(), s["vt"].data_ptr(),
                                      ws["wsf"].data_ptr(), ws["wsf"].numel(), sp)
                self.ev_fwd[i].record(self.s_comp)
                self.s_comp.wait_event(self.ev_in_dO[i])
                _abi.eot_sinkhorn_bwd(p, s["q"].data_ptr(), s["k"].data_ptr(), s["v"].data_ptr(), m,
                                      s["ut"].data_ptr(), s["vt"].data_ptr(), s["dO"].data_ptr(),
                                      s["dQ"].data_ptr(), s["dK"].data_ptr(), s["dV"].data_ptr(),
                                      ws["wsb"].data_ptr(), ws["wsb"].numel(), sp)
                self.ev_comp[i].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_fwd[i])
                hO[b0:b1, h0:h1].copy_(s["O"], non_blocking=True)
                self.s_out.wait_event(self.ev_comp[i])
                for name, dst in (("dQ", hdQ), ("dK", hdK), ("dV", hdV)):
                    dst[b0:b1, h0:h1].copy_(s[name], non_blocking=True)
                self.ev_out[i].record(self.s_out)
            self.c += 1

    def device_status(self) -> int:
        """Device status of the last chunk's calls (synchronises)."""
        torch.cuda.synchronize(self.dev)
        st = 0
        for s in self.slots:
            st = st or _abi.eot_last_device_status(s["wsf"].data_ptr(), 0) or \
                _abi.eot_last_device_status(s["wsb"].data_ptr(), 0)
        return st
