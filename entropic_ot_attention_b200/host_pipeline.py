"""Forward + backward on inputs held in pinned host memory, with the host <-> device copies
overlapped with the kernels.

The (batch, head) units of a problem are independent (each has its own potentials and band),
so a step over B x H units can run as a sequence of smaller problems, one chunk of heads of
one batch row at a time.  Three CUDA streams carry the chunks through copy-in, compute
(eot_sinkhorn_fwd then eot_sinkhorn_bwd through the C ABI) and copy-out; two device staging
slots alternate, so chunk c + 1's inputs arrive and chunk c - 1's results leave while chunk c
computes.  Every step of the method still runs in libeot's kernels; this module only moves
data and orders the streams.
"""
from __future__ import annotations

import torch

from . import _abi
from .api import make_problem, workspace


class HostStep:
    """One forward + backward over host tensors q, k, v, dO [B, H, L, d] (pinned), writing
    O, dQ, dK, dV [B, H, L, d] (pinned) back to the host.  ``heads_per_chunk`` heads of one
    batch row form a chunk.  The mask, if any, is a host or device uint8 [B, L] fixed at
    construction."""

    def __init__(self, B: int, H: int, L: int, d: int, W: int, T: int, R: int, dtype: torch.dtype,
                 scale=None, mask=None, heads_per_chunk: int = 1, device=None, impl: str = "auto"):
        if H % heads_per_chunk != 0:
            raise ValueError("heads_per_chunk must divide H")
        self.B, self.H, self.L, self.d, self.R = B, H, L, d, R
        self.hc = heads_per_chunk
        self.dev = torch.device("cuda") if device is None else torch.device(device)
        self.p = make_problem(1, heads_per_chunk, L, d, W, T, R, dtype, scale, impl=impl)
        st = _abi.eot_validate(self.p)
        if st != 0:
            raise ValueError(f"problem rejected: {_abi.eot_status_string(st)}")
        self.mask = None if mask is None else mask.to(self.dev, torch.uint8).contiguous()
        shape = (heads_per_chunk, L, d)
        tshape = (heads_per_chunk, R + 1, L)
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
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.c = 0   # running chunk counter (slot = counter % 2)

    def chunks(self):
        for b in range(self.B):
            for h0 in range(0, self.H, self.hc):
                yield b, h0, h0 + self.hc

    def run(self, hq, hk, hv, hdO, hO, hdQ, hdK, hdV):
        """Enqueue one step; returns at once (synchronise ``s_out`` or the device to wait)."""
        for b, h0, h1 in self.chunks():
            i = self.c % 2
            s = self.slots[i]
            first_use = self.c < 2
            # inputs of this slot are free once the compute two chunks back has finished
            with torch.cuda.stream(self.s_in):
                if not first_use:
                    self.s_in.wait_event(self.ev_comp[i])
                for name, src in (("q", hq), ("k", hk), ("v", hv), ("dO", hdO)):
                    s[name].copy_(src[b, h0:h1], non_blocking=True)
                self.ev_in[i].record(self.s_in)
            # outputs of this slot are free once the copy-out two chunks back has finished
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(self.ev_in[i])
                if not first_use:
                    self.s_comp.wait_event(self.ev_out[i])
                sp = int(self.s_comp.cuda_stream)
                m = None if self.mask is None else self.mask[b:b + 1].data_ptr()
                _abi.eot_sinkhorn_fwd(self.p, s["q"].data_ptr(), s["k"].data_ptr(), s["v"].data_ptr(), m,
                                      s["O"].data_ptr(), s["ut"].data_ptr(), s["vt"].data_ptr(),
                                      s["wsf"].data_ptr(), s["wsf"].numel(), sp)
                _abi.eot_sinkhorn_bwd(self.p, s["q"].data_ptr(), s["k"].data_ptr(), s["v"].data_ptr(), m,
                                      s["ut"].data_ptr(), s["vt"].data_ptr(), s["dO"].data_ptr(),
                                      s["dQ"].data_ptr(), s["dK"].data_ptr(), s["dV"].data_ptr(),
                                      s["wsb"].data_ptr(), s["wsb"].numel(), sp)
                self.ev_comp[i].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_comp[i])
                for name, dst in (("O", hO), ("dQ", hdQ), ("dK", hdK), ("dV", hdV)):
                    dst[b, h0:h1].copy_(s[name], non_blocking=True)
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
