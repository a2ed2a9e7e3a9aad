"""Host-side logic of bench.py: rank aggregation over a 2-rank gloo group on CPU, and the
support-size count used for the algorithmic work."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import eot_inputs
from oracle import eot_oracle as eo


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    mx = bench.max_over_ranks(1.5 + rank)
    sm = bench.sum_over_ranks(10.0 * (rank + 1))
    bench.barrier()
    out[rank] = (mx, sm)
    dist.destroy_process_group()


def test_rank_aggregation_gloo_two_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == (2.5, 30.0) and out[1] == (2.5, 30.0)


def test_aggregation_without_process_group_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.sum_over_ranks(7.0) == 7.0


@pytest.mark.parametrize("dustbin", [False, True])
def test_support_size_matches_oracle(dustbin):
    rng = np.random.default_rng(3)
    mask = (rng.random((2, 256)) > 0.3).astype(np.uint8)
    if dustbin:
        case = eot_inputs.dustbin_case(2, 3, 200, 8, 40, 2, 1, "fp32", mask=mask[:, :200])
    else:
        case = eot_inputs.dense_case(2, 3, 256, 8, 40, 2, 1, "fp32", mask=mask)
    n = 0
    B, H, L, _ = case.Q.shape
    for b in range(B):
        st = eo.unit_structure(L, case.W, None if case.mask is None else case.mask[b], case.dustbin,
                               case.dustbin_index, case.dustbin_mass)
        n += int(st.support.sum()) * H
    assert bench.band_support_size(case) == n


def test_long_workload_support_size_closed_form():
    """|Omega| per unit of a full band = L(W+1) - (W/2)(W/2+1)."""
    class C:
        pass
    c = C()
    c.Q = np.zeros((1, 4, 131072, 1), np.float32)
    c.W, c.mask, c.dustbin, c.dustbin_index, c.dustbin_mass = 1024, None, False, -1, 0.0
    assert bench.band_support_size(c) == 4 * (131072 * 1025 - 512 * 513)


@pytest.mark.parametrize("B,H,kw,n_want", [
    (1, 4, {}, 4),                       # long context: one head per chunk
    (4, 8, {}, 4),                       # whole rows
    (32, 4, {}, 4),                      # many short units: 8 rows per chunk
    (5, 2, {}, 3),                       # ragged last chunk of rows
    (2, 3, {}, 6),                       # too few rows: heads of one row
    (3, 2, {"rows_per_chunk": 2}, 2),
    (3, 2, {"heads_per_chunk": 2}, 3),
])
def test_host_step_chunk_plans(B, H, kw, n_want):
    """Every (batch, head) unit of a host-memory step lands in exactly one chunk, in order, and
    the automatic plan keeps many short units together instead of one call per unit."""
    from entropic_ot_attention_b200.host_pipeline import chunk_list, plan_chunks
    rows, hc = plan_chunks(B, H, **kw)
    chunks = chunk_list(B, H, rows, hc)
    assert len(chunks) == n_want
    seen = [(b, h) for b0, b1, h0, h1 in chunks for b in range(b0, b1) for h in range(h0, h1)]
    assert seen == [(b, h) for b in range(B) for h in range(H)]


def test_host_step_chunk_plan_errors():
    from entropic_ot_attention_b200.host_pipeline import plan_chunks
    with pytest.raises(ValueError):
        plan_chunks(2, 4, heads_per_chunk=3)
    with pytest.raises(ValueError):
        plan_chunks(2, 4, rows_per_chunk=3)
    with pytest.raises(ValueError):
        plan_chunks(2, 4, heads_per_chunk=1, rows_per_chunk=1)
