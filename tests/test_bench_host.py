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


# Algorithmic work of one call (the workload table of the measurement plan): MMA flops
# (T+R+2) 2d |Omega| forward and 5 2d |Omega| backward, roofline max(flops / 1630 TFLOP/s,
# bytes / 6547.2 GB/s) per pass.
@pytest.mark.parametrize("shape,omega,fwd_flops,bwd_flops,fwd_ms,bwd_ms,bounds", [
    # medium: B=4 H=8 L=4096 d=64 W=256 T=20 R=2; |Omega| = 32 (4096*257 - 128*129)
    ((4, 8, 4096, 64, 20, 2), 32 * (4096 * 257 - 128 * 129), 1.019e11, 2.12e10, 0.0625, 0.0191, ("tensor", "hbm")),
    # long: B=1 H=4 L=131072 d=128 W=1024 T=10 R=2; |Omega| = 4 (131072*1025 - 512*513)
    ((1, 4, 131072, 128, 10, 2), 4 * (131072 * 1025 - 512 * 513), 1.922e12, 6.87e11, 1.179, 0.421,
     ("tensor", "tensor")),
])
def test_algorithmic_work_and_roofline(shape, omega, fwd_flops, bwd_flops, fwd_ms, bwd_ms, bounds):
    B, H, L, d, T, R = shape
    w = bench.algorithmic_work(B, H, L, d, T, R, omega, 2)
    assert w["fwd_flops"] == pytest.approx(fwd_flops, rel=2e-3)
    assert w["bwd_flops"] == pytest.approx(bwd_flops, rel=2e-3)
    assert w["solve_flops"] == (T + R) * 2 * d * omega
    assert w["solve_flops"] + w["output_flops"] == w["fwd_flops"]
    tf, bf = bench.roofline_ms(w["fwd_flops"], w["fwd_bytes"], 1630.0, 6547.2)
    tb, bb = bench.roofline_ms(w["bwd_flops"], w["bwd_bytes"], 1630.0, 6547.2)
    assert tf == pytest.approx(fwd_ms, rel=5e-3) and bf == bounds[0]
    assert tb == pytest.approx(bwd_ms, rel=5e-3) and bb == bounds[1]


def test_dominant_kernel_counts_one_score_evaluation_per_iteration():
    """The forward solve of the long workload, timed at 4.893 ms per call, does 12 iterations of
    2d |Omega| flops: 337 TFLOP/s, 0.207 of the 1630 TFLOP/s burst peak."""
    omega = 4 * (131072 * 1025 - 512 * 513)
    w = bench.algorithmic_work(1, 4, 131072, 128, 10, 2, omega, 2)
    prof = {"fwd_sweep": (4.893, 2), "fwd_output": (0.498, 1), "bwd_sweep": (2.760, 6), "aux": (0.24, 12)}
    r = bench.dominant_kernel(prof, w, 10, 2, 1630.0, "measured", exp_passes=24, omega=omega, mufu_peak=4.65e12)
    assert r["kind"] == "fwd_sweep" and r["units_timed"] == 12
    assert r["achieved"] == pytest.approx(337.0, rel=2e-3)
    assert r["frac"] == pytest.approx(0.207, abs=1e-3)
    assert r["exp2_per_s"] == pytest.approx(24 * omega / 4.893e-3, rel=1e-9)
    prof["bwd_sweep"] = (6.0, 6)
    r = bench.dominant_kernel(prof, w, 10, 2, 1630.0, "measured", exp_passes=24, omega=omega, mufu_peak=4.65e12)
    assert r["kind"] == "bwd_sweep" and r["achieved"] == pytest.approx(w["bwd_flops"] / 6.0e-3 / 1e12)


def test_gpus_flag_spawns_that_many_ranks():
    """--gpus 2 without a launcher re-runs bench.py as two ranks; rank 0 alone prints one line
    whose n_gpus is 2 (host plumbing only: gloo, no GPU)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--dry-run"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert res.returncode == 0, res.stderr
    lines = [json.loads(x) for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["ranks_reporting"] == 2.0 and lines[0]["ms_per_step"] == 2.0
