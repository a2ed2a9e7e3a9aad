"""Sequence sharding of one unit over ranks (host logic, gloo on CPU): the row-range plan with
its W/2 halo, the per-half-step exchange of boundary potentials, and the (max, sum) merge of the
dense dustbin row.  A sharded solve over 2 and 3 ranks, each rank forming only its own rows'
and columns' band scores, must reproduce the single-rank oracle's potentials."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from entropic_ot_attention_b200.sharding import Shard, shard_plan
from oracle import eot_oracle as eo


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_shard_plan_covers_the_sequence_in_tiles():
    plan = shard_plan(640, 100, 2)
    assert [(s.r0, s.r1) for s in plan] == [(0, 384), (384, 640)]
    assert [(s.c0, s.c1) for s in plan] == [(0, 434), (334, 640)]
    plan = shard_plan(1280, 256, 3)
    assert [s.n for s in plan] == [512, 384, 384]
    assert plan[0].r0 == 0 and plan[-1].r1 == 1280
    assert all(a.r1 == b.r0 for a, b in zip(plan, plan[1:]))
    assert shard_plan(256, 1000, 1) == [Shard(0, 0, 256, 0, 256)]


@pytest.mark.parametrize("args", [(640, 100, 6), (200, 10, 1), (256, 600, 2), (256, -2, 1), (256, 10, 0)])
def test_shard_plan_rejects(args):
    with pytest.raises(ValueError):
        shard_plan(*args)


def _unit(L, d, W, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, d))
    k = rng.standard_normal((L, d))
    mask = (rng.random(L) > 0.15).astype(np.uint8)
    return q, k, mask


def _solve_worker(rank, world, port, L, d, W, T, R, out):
    import torch.distributed as dist
    from entropic_ot_attention_b200.sharding import sharded_solve, shard_plan
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    q, k, mask = _unit(L, d, W, seed=5)
    plan = shard_plan(L, W, world)
    sh = plan[rank]
    h, scale = W // 2, 1.0 / np.sqrt(d)
    act = mask.astype(bool)
    # uniform marginals over the active positions: the count is one scalar all-reduce
    n_act = torch.tensor([float(act[sh.r0:sh.r1].sum())], dtype=torch.float64)
    dist.all_reduce(n_act)
    log_a = -np.log(n_act.item())
    # this rank's band scores only: its rows against the halo columns, and its columns against
    # the halo rows (q and k rows of the halo copied once)
    rows = np.arange(sh.r0, sh.r1)
    halo = np.arange(sh.c0, sh.c1)
    band = (np.abs(rows[:, None] - halo[None, :]) <= h) & act[rows][:, None] & act[halo][None, :]
    S_rows = np.where(band, scale * q[rows] @ k[halo].T, -np.inf)   # S[i, j], i owned
    S_cols = np.where(band, scale * k[rows] @ q[halo].T, -np.inf)   # S[i, j]^T, j owned

    def row_step(v_halo):
        u = log_a - eo.lse(S_rows + v_halo.numpy()[None, :], axis=1)
        return torch.from_numpy(np.where(act[rows], u, 0.0))

    def col_step(u_halo):
        v = log_a - eo.lse(S_cols + u_halo.numpy()[None, :], axis=1)
        return torch.from_numpy(np.where(act[rows], v, 0.0))

    with np.errstate(invalid="ignore", divide="ignore"):
        ut, vt = sharded_solve(plan, rank, T, R, row_step, col_step)
    out[rank] = (sh.r0, sh.r1, ut.numpy(), vt.numpy())
    dist.destroy_process_group()


@pytest.mark.parametrize("world,L,W", [(2, 640, 100), (3, 1280, 256), (2, 512, 0)])
def test_sharded_solve_matches_single_rank_oracle(world, L, W):
    d, T, R = 16, 7, 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_solve_worker, args=(r, world, port, L, d, W, T, R, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    q, k, mask = _unit(L, d, W, seed=5)
    ref = eo.forward_unit(q, k, np.zeros((L, 1)), W, T, R, mask_row=mask)
    ut = np.zeros((R + 1, L))
    vt = np.zeros((R + 1, L))
    for r in range(world):
        r0, r1, u, v = out[r]
        ut[:, r0:r1] = u
        vt[:, r0:r1] = v
    assert np.max(np.abs(ut - ref.u_tail)) <= 1e-12
    assert np.max(np.abs(vt - ref.v_tail)) <= 1e-12


def _lse_worker(rank, world, port, out):
    import torch.distributed as dist
    from entropic_ot_attention_b200.sharding import allreduce_lse
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((world, 3, 50)) * 20.0
    x[:, 2, :] = -np.inf                      # an all -inf row: (-inf, 0)
    x[1:, 1, :] = -np.inf                     # only rank 0 holds row 1
    mine = x[rank]
    m = mine.max(axis=1)
    s = np.where(np.isfinite(m), np.exp(mine - np.where(np.isfinite(m), m, 0.0)[:, None]).sum(axis=1), 0.0)
    M, S = allreduce_lse(torch.from_numpy(m), torch.from_numpy(s))
    out[rank] = (M.numpy(), S.numpy())
    dist.destroy_process_group()


def test_allreduce_lse_matches_direct_log_sum_exp():
    world = 3
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_lse_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    rng = np.random.default_rng(11)
    x = rng.standard_normal((world, 3, 50)) * 20.0
    x[:, 2, :] = -np.inf
    x[1:, 1, :] = -np.inf
    want = eo.lse(np.concatenate(list(x), axis=1), axis=1)
    for r in range(world):
        M, S = out[r]
        with np.errstate(divide="ignore"):
            got = np.where(S > 0, M + np.log(np.where(S > 0, S, 1.0)), -np.inf)
        assert np.allclose(got[:2], want[:2], rtol=0, atol=1e-12)
        assert got[2] == -np.inf and S[2] == 0.0


def _unit_dustbin(L_real, d, seed):
    """Real positions [0, L_real), the dustbin at L_real, fillers up to the next tile."""
    rng = np.random.default_rng(seed)
    L = L_real + 128
    q = rng.standard_normal((L, d))
    k = rng.standard_normal((L, d))
    mask = np.zeros(L, np.uint8)
    mask[:L_real] = (rng.random(L_real) > 0.15).astype(np.uint8)
    return q, k, mask


def _lse_pair(x):
    """(max, sum exp(x - max)) of a 1-D array, (-inf, 0) when empty or all -inf."""
    x = x[np.isfinite(x)]
    if x.size == 0:
        return -np.inf, 0.0
    m = x.max()
    return m, float(np.exp(x - m).sum())


def _dustbin_worker(rank, world, port, L_real, d, W, T, R, mass, dself, out):
    import torch.distributed as dist
    from entropic_ot_attention_b200.sharding import sharded_solve_dustbin, shard_plan
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    q, k, mask = _unit_dustbin(L_real, d, seed=13)
    D = L_real
    plan = shard_plan(L_real, W, world)
    sh = plan[rank]
    h, scale = W // 2, 1.0 / np.sqrt(d)
    act = mask.astype(bool)
    n_act = torch.tensor([float(act[sh.r0:sh.r1].sum())], dtype=torch.float64)
    dist.all_reduce(n_act)
    log_a = np.log((1.0 - mass) / n_act.item())
    rows = np.arange(sh.r0, sh.r1)
    halo = np.arange(sh.c0, sh.c1)
    band = (np.abs(rows[:, None] - halo[None, :]) <= h) & act[rows][:, None] & act[halo][None, :]
    S_rows = np.where(band, scale * q[rows] @ k[halo].T, -np.inf)
    S_cols = np.where(band, scale * k[rows] @ q[halo].T, -np.inf)
    to_D = scale * q[rows] @ k[D]          # S_rD, owned rows
    from_D = scale * q[D] @ k[rows].T      # S_Dc, owned columns

    def row_step(v_halo, v_D):
        x = np.concatenate([S_rows + v_halo.numpy()[None, :], (to_D + v_D.item())[:, None]], axis=1)
        u = np.where(act[rows], log_a - eo.lse(x, axis=1), 0.0)
        m, s = _lse_pair(np.where(act[rows], from_D + v_halo.numpy()[sh.owned], -np.inf))
        return torch.from_numpy(u), torch.tensor(m, dtype=torch.float64), torch.tensor(s, dtype=torch.float64)

    def col_step(u_halo, u_D):
        x = np.concatenate([S_cols + u_halo.numpy()[None, :], (from_D + u_D.item())[:, None]], axis=1)
        v = np.where(act[rows], log_a - eo.lse(x, axis=1), 0.0)
        m, s = _lse_pair(np.where(act[rows], to_D + u_halo.numpy()[sh.owned], -np.inf))
        return torch.from_numpy(v), torch.tensor(m, dtype=torch.float64), torch.tensor(s, dtype=torch.float64)

    self_score = float(scale * q[D] @ k[D]) if dself else None
    with np.errstate(invalid="ignore", divide="ignore"):
        ut, vt, uD, vD = sharded_solve_dustbin(plan, rank, T, R, row_step, col_step, np.log(mass), self_score)
    out[rank] = (sh.r0, sh.r1, ut.numpy(), vt.numpy(), uD.numpy(), vD.numpy())
    dist.destroy_process_group()


@pytest.mark.parametrize("world,L_real,W,dself", [(2, 640, 100, True), (3, 1280, 256, False)])
def test_sharded_solve_with_dustbin_matches_single_rank_oracle(world, L_real, W, dself):
    d, T, R, mass = 16, 6, 2, 0.1
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_dustbin_worker, args=(r, world, port, L_real, d, W, T, R, mass, dself, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    q, k, mask = _unit_dustbin(L_real, d, seed=13)
    ref = eo.forward_unit(q, k, np.zeros((q.shape[0], 1)), W, T, R, mask_row=mask, dustbin=True,
                          dustbin_index=L_real, dustbin_mass=mass, dustbin_self=dself)
    ut = np.zeros((R + 1, L_real))
    vt = np.zeros((R + 1, L_real))
    for r in range(world):
        r0, r1, u, v, uD, vD = out[r]
        ut[:, r0:r1] = u
        vt[:, r0:r1] = v
        assert np.max(np.abs(uD - ref.u_tail[:, L_real])) <= 1e-12
        assert np.max(np.abs(vD - ref.v_tail[:, L_real])) <= 1e-12
    assert np.max(np.abs(ut - ref.u_tail[:, :L_real])) <= 1e-12
    assert np.max(np.abs(vt - ref.v_tail[:, :L_real])) <= 1e-12
