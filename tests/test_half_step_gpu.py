"""One band half-step through the C ABI (``eot_band_half_step``) against the oracle's row and
column steps ("Blockwise Differentiable Sinkhorn Attention" §2.1), and a sequence-sharded solve
of one unit whose ranks (gloo processes sharing cuda:0) take every half-step on the GPU.

Tolerance of one half-step: the scores are fp32 sums of d exact products of the (dtype-exact)
inputs, the sum of exponentials is fp32 with ex2.approx / lg2.approx (relative error about
2^-22 each), so a potential is off by well under 1e-5 of max(|potential|, 1); 1e-4 is the bar.
A solve of 2 (T + R) half-steps carries those errors through the iteration, which contracts
them: 1e-4 again."""
import os
import socket

import numpy as np
import pytest

import eot_inputs
from harness import pot_err
from oracle import eot_oracle as eo

pytestmark = pytest.mark.gpu

STEP_TOL = 1e-4


def _log_marg(mask, extra=0):
    """Uniform log marginals over the active positions of each batch row, as if the row were
    part of a sequence with ``extra`` more active positions elsewhere."""
    n = mask.sum(axis=1, keepdims=True).astype(np.float64) + extra
    with np.errstate(divide="ignore"):
        return np.where(mask.astype(bool), -np.log(np.maximum(n, 1.0)), -np.inf)


def _oracle_step(x, y, log_m, pot, W, scale, active):
    """The oracle's row step on the band support restricted to the active positions."""
    L = x.shape[0]
    st = eo.unit_structure(L, W, mask_row=active)
    S = eo.scores(x, y, scale, st.support)
    return eo.row_step(S, log_m, pot, active)


@pytest.mark.parametrize("dtype,d,W,L,impl", [
    ("bf16", 128, 256, 896, "auto"),      # several tiles, ragged masks
    ("bf16", 128, 1024, 1280, "auto"),    # a band wider than the tile pair
    ("bf16", 64, 100, 640, "auto"),       # d = 64, a band edge inside a tile
    ("bf16", 64, 0, 256, "auto"),         # W = 0: out_i = log m_i - (S_ii + in_i)
    ("fp32", 32, 60, 384, "auto"),        # CUDA-core path
    ("bf16", 64, 160, 512, "simt"),
])
def test_half_step_matches_oracle(dtype, d, W, L, impl):
    import torch
    from entropic_ot_attention_b200 import band_half_step
    B, H = 2, 2
    rng = np.random.default_rng(L + W + d)
    mask = (rng.random((B, L)) > 0.2).astype(np.uint8)
    mask[1, L - 200:] = 0                                   # a ragged tail
    case = eot_inputs.dense_case(B, H, L, d, W, 0, 0, dtype, seed=3, mask=mask)
    log_m = _log_marg(mask, extra=37)
    pot = (rng.standard_normal((B, H, L)) * 3.0).astype(np.float32)
    pot[np.broadcast_to(mask[:, None, :] == 0, pot.shape)] = 1.0e3   # must be ignored
    scale = 1.0 / np.sqrt(d)
    dev = torch.device("cuda:0")
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    q = torch.from_numpy(case.Q).to(dev).to(tdt).contiguous()
    k = torch.from_numpy(case.K).to(dev).to(tdt).contiguous()
    lm_t = torch.from_numpy(log_m.astype(np.float32)).to(dev)
    pin = torch.from_numpy(pot).to(dev)
    u = band_half_step(q, k, lm_t, pin, W, impl=impl).cpu().numpy()     # row half-step
    v = band_half_step(k, q, lm_t, pin, W, impl=impl).cpu().numpy()     # column half-step
    torch.cuda.synchronize()
    for b in range(B):
        act = mask[b].astype(bool)
        for h in range(H):
            x, y = case.Q[b, h].astype(np.float64), case.K[b, h].astype(np.float64)
            p_in = pot[b, h].astype(np.float64)
            want_u = _oracle_step(x, y, log_m[b], p_in, W, scale, act)
            st = eo.unit_structure(L, W, mask_row=act)
            want_v = eo.col_step(eo.scores(x, y, scale, st.support), log_m[b], p_in, act)
            assert pot_err(u[b, h], want_u) <= STEP_TOL, (b, h, pot_err(u[b, h], want_u))
            assert pot_err(v[b, h], want_v) <= STEP_TOL, (b, h, pot_err(v[b, h], want_v))
            assert np.all(u[b, h][~act] == 0.0) and np.all(v[b, h][~act] == 0.0)


@pytest.mark.parametrize("dtype,d,W,L", [("bf16", 128, 256, 896), ("bf16", 64, 100, 640), ("fp32", 32, 60, 384)])
def test_output_of_given_potentials_matches_oracle(dtype, d, W, L):
    import torch
    from entropic_ot_attention_b200 import band_output
    from harness import TOL, rel_err
    B, H = 2, 2
    rng = np.random.default_rng(L + W + d + 2)
    mask = (rng.random((B, L)) > 0.2).astype(np.uint8)
    case = eot_inputs.dense_case(B, H, L, d, W, 0, 0, dtype, seed=6, mask=mask)
    scale = 1.0 / np.sqrt(d)
    u = (rng.standard_normal((B, H, L)) * 0.5 - np.log(L)).astype(np.float32)
    vp = (rng.standard_normal((B, H, L)) * 0.5).astype(np.float32)
    dev = torch.device("cuda:0")
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    t = lambda a: torch.from_numpy(a).to(dev).to(tdt).contiguous()
    log_m = np.stack([eo.unit_structure(L, W, mask_row=mask[b]).log_a for b in range(B)]).astype(np.float32)
    O = band_output(t(case.Q), t(case.K), t(case.V), torch.from_numpy(log_m).to(dev), torch.from_numpy(u).to(dev),
                    torch.from_numpy(vp).to(dev), W).float().cpu().numpy()
    for b in range(B):
        st = eo.unit_structure(L, W, mask_row=mask[b])
        for h in range(H):
            S = eo.scores(case.Q[b, h], case.K[b, h], scale, st.support)
            want = eo.output(S, st, u[b, h].astype(np.float64), vp[b, h].astype(np.float64), case.V[b, h])
            assert rel_err(O[b, h], want) <= TOL[dtype], (b, h, rel_err(O[b, h], want))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _unit(L, d, dtype, seed):
    rng = np.random.default_rng(seed)
    mask = (rng.random((1, L)) > 0.15).astype(np.uint8)
    case = eot_inputs.dense_case(1, 1, L, d, 0, 0, 0, dtype, seed=seed, mask=mask)
    return case.Q[0, 0], case.K[0, 0], mask[0]


def _unit_v(L, d, dtype, seed):
    rng = np.random.default_rng(seed)
    mask = (rng.random((1, L)) > 0.15).astype(np.uint8)
    return eot_inputs.dense_case(1, 1, L, d, 0, 0, 0, dtype, seed=seed, mask=mask).V[0, 0]


def _gpu_solve_worker(rank, world, port, L, d, W, T, R, dtype, out):
    import torch
    import torch.distributed as dist
    from entropic_ot_attention_b200.sharding import device_half_steps, shard_plan, sharded_solve
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    q, k, mask = _unit(L, d, dtype, seed=9)
    vv = _unit_v(L, d, dtype, seed=9)
    plan = shard_plan(L, W, world)
    sh = plan[rank]
    act = mask.astype(bool)
    # uniform marginals of the whole sequence: the active count is one scalar all-reduce
    n_act = torch.tensor([float(act[sh.r0:sh.r1].sum())], dtype=torch.float64)
    dist.all_reduce(n_act)
    lm_halo = torch.from_numpy(np.where(act[sh.c0:sh.c1], -np.log(n_act.item()), -np.inf))
    dev = torch.device("cuda:0")
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    qh = torch.from_numpy(np.ascontiguousarray(q[sh.c0:sh.c1])).to(dev).to(tdt)
    kh = torch.from_numpy(np.ascontiguousarray(k[sh.c0:sh.c1])).to(dev).to(tdt)
    row_step, col_step = device_half_steps(sh, qh, kh, lm_halo, W)
    ut, vt = sharded_solve(plan, rank, T, R, row_step, col_step)
    # the owned rows' output from the last potentials over the halo
    from entropic_ot_attention_b200.sharding import device_output, halo_exchange
    vh = torch.from_numpy(np.ascontiguousarray(vv[sh.c0:sh.c1])).to(dev).to(tdt)
    O = device_output(sh, qh, kh, vh, lm_halo, halo_exchange(ut[R], plan, rank), halo_exchange(vt[R], plan, rank), W)
    torch.cuda.synchronize()
    out[rank] = (sh.r0, sh.r1, ut.numpy(), vt.numpy(), O.float().cpu().numpy())
    dist.destroy_process_group()


@pytest.mark.parametrize("world,L,W,d,dtype", [(2, 1280, 256, 64, "bf16"), (3, 1536, 300, 128, "bf16"),
                                               (2, 768, 100, 32, "fp32")])
def test_sharded_solve_on_gpu_matches_oracle(world, L, W, d, dtype):
    import torch.multiprocessing as mp
    T, R = 5, 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_gpu_solve_worker, args=(r, world, port, L, d, W, T, R, dtype, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    from harness import TOL, rel_err
    q, k, mask = _unit(L, d, dtype, seed=9)
    vv = _unit_v(L, d, dtype, seed=9)
    ref = eo.forward_unit(q, k, vv, W, T, R, mask_row=mask)
    ut = np.zeros((R + 1, L))
    vt = np.zeros((R + 1, L))
    O = np.zeros((L, d))
    for r in range(world):
        r0, r1, u, v, o = out[r]
        ut[:, r0:r1] = u
        vt[:, r0:r1] = v
        O[r0:r1] = o
    assert pot_err(ut, ref.u_tail) <= STEP_TOL, pot_err(ut, ref.u_tail)
    assert pot_err(vt, ref.v_tail) <= STEP_TOL, pot_err(vt, ref.v_tail)
    assert rel_err(O, ref.O) <= TOL[dtype], rel_err(O, ref.O)


@pytest.mark.parametrize("dtype,d,W,L_real,impl", [
    ("bf16", 128, 256, 768, "auto"),
    ("bf16", 64, 100, 640, "auto"),
    ("fp32", 32, 60, 384, "auto"),
])
def test_half_step_with_dustbin_matches_oracle(dtype, d, W, L_real, impl):
    import torch
    from entropic_ot_attention_b200 import band_half_step
    B, H, mass = 2, 2, 0.1
    L, D = L_real + 128, L_real
    rng = np.random.default_rng(L + W + d + 1)
    real = np.zeros((B, L), np.uint8)
    real[:, :L_real] = (rng.random((B, L_real)) > 0.2).astype(np.uint8)
    case = eot_inputs.dense_case(B, H, L, d, W, 0, 0, dtype, seed=4)
    with np.errstate(divide="ignore"):
        log_m = np.where(real.astype(bool), np.log((1.0 - mass) / (real.sum(axis=1, keepdims=True) + 37.0)), -np.inf)
    log_m[:, D] = np.log(mass)
    pot = (rng.standard_normal((B, H, L)) * 3.0).astype(np.float32)
    scale = 1.0 / np.sqrt(d)
    dev = torch.device("cuda:0")
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    q = torch.from_numpy(case.Q).to(dev).to(tdt).contiguous()
    k = torch.from_numpy(case.K).to(dev).to(tdt).contiguous()
    lm_t = torch.from_numpy(log_m.astype(np.float32)).to(dev)
    pin = torch.from_numpy(pot).to(dev)
    lo, hi = 128, L_real - 128
    u, part = band_half_step(q, k, lm_t, pin, W, impl=impl, dustbin_index=D, own=(lo, hi))
    u_all, part_all = band_half_step(q, k, lm_t, pin, W, impl=impl, dustbin_index=D)
    u, part, part_all = u.cpu().numpy(), part.cpu().numpy(), part_all.cpu().numpy()
    torch.cuda.synchronize()
    for b in range(B):
        act = real[b].astype(bool)
        st = eo.unit_structure(L, W, mask_row=real[b], dustbin=True, dustbin_index=D, dustbin_mass=mass)
        for h in range(H):
            x, y = case.Q[b, h].astype(np.float64), case.K[b, h].astype(np.float64)
            S = eo.scores(x, y, scale, st.support)
            want = eo.row_step(S, log_m[b], pot[b, h].astype(np.float64), st.active)
            assert pot_err(u[b, h, :D], want[:D]) <= STEP_TOL, (b, h, pot_err(u[b, h, :D], want[:D]))
            # the dustbin's partial over [lo, hi), and over every real position with (D, D) added
            xs = S[D, :D] + pot[b, h, :D]
            sel = act[:D] & (np.arange(D) >= lo) & (np.arange(D) < hi)
            want_part = eo.lse(xs[sel], axis=0)
            got_part = part[b, h, 0] + np.log(part[b, h, 1])
            assert abs(got_part - want_part) <= STEP_TOL * max(abs(want_part), 1.0)
            self_term = S[D, D] + pot[b, h, D]
            got_D = log_m[b, D] - eo.lse(np.array([part_all[b, h, 0] + np.log(part_all[b, h, 1]), self_term]), axis=0)
            assert abs(got_D - want[D]) <= STEP_TOL * max(abs(want[D]), 1.0)


def _gpu_dustbin_worker(rank, world, port, L_real, d, W, T, R, mass, dtype, out):
    import torch
    import torch.distributed as dist
    from entropic_ot_attention_b200.sharding import device_half_steps_dustbin, shard_plan, sharded_solve_dustbin
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    q, k, mask = _unit_dustbin(L_real, d, dtype, seed=21)
    D = L_real
    plan = shard_plan(L_real, W, world)
    sh = plan[rank]
    act = mask.astype(bool)
    n_act = torch.tensor([float(act[sh.r0:sh.r1].sum())], dtype=torch.float64)
    dist.all_reduce(n_act)
    lm_halo = torch.from_numpy(np.where(act[sh.c0:sh.c1], np.log((1.0 - mass) / n_act.item()), -np.inf))
    dev = torch.device("cuda:0")
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(tdt)
    row_step, col_step = device_half_steps_dustbin(sh, to_dev(q[sh.c0:sh.c1]), to_dev(k[sh.c0:sh.c1]), to_dev(q[D]),
                                                   to_dev(k[D]), lm_halo, float(np.log(mass)), W)
    self_score = float(np.float64(q[D]) @ np.float64(k[D]) / np.sqrt(d))
    ut, vt, uD, vD = sharded_solve_dustbin(plan, rank, T, R, row_step, col_step, float(np.log(mass)), self_score)
    torch.cuda.synchronize()
    out[rank] = (sh.r0, sh.r1, ut.numpy(), vt.numpy(), uD.numpy(), vD.numpy())
    dist.destroy_process_group()


def _unit_dustbin(L_real, d, dtype, seed):
    rng = np.random.default_rng(seed)
    L = L_real + 128
    mask = np.zeros((1, L), np.uint8)
    mask[0, :L_real] = (rng.random(L_real) > 0.15).astype(np.uint8)
    case = eot_inputs.dense_case(1, 1, L, d, 0, 0, 0, dtype, seed=seed)
    return case.Q[0, 0], case.K[0, 0], mask[0]


@pytest.mark.parametrize("world,L_real,W,d,dtype", [(2, 1280, 256, 64, "bf16"), (3, 1536, 300, 128, "bf16")])
def test_sharded_solve_with_dustbin_on_gpu_matches_oracle(world, L_real, W, d, dtype):
    import torch.multiprocessing as mp
    T, R, mass = 5, 2, 0.1
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_gpu_dustbin_worker, args=(r, world, port, L_real, d, W, T, R, mass, dtype, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    q, k, mask = _unit_dustbin(L_real, d, dtype, seed=21)
    ref = eo.forward_unit(q, k, np.zeros((q.shape[0], 1)), W, T, R, mask_row=mask, dustbin=True,
                          dustbin_index=L_real, dustbin_mass=mass, dustbin_self=True)
    ut = np.zeros((R + 1, L_real))
    vt = np.zeros((R + 1, L_real))
    for r in range(world):
        r0, r1, u, v, uD, vD = out[r]
        ut[:, r0:r1] = u
        vt[:, r0:r1] = v
        assert pot_err(uD, ref.u_tail[:, L_real]) <= STEP_TOL
        assert pot_err(vD, ref.v_tail[:, L_real]) <= STEP_TOL
    assert pot_err(ut, ref.u_tail[:, :L_real]) <= STEP_TOL, pot_err(ut, ref.u_tail[:, :L_real])
    assert pot_err(vt, ref.v_tail[:, :L_real]) <= STEP_TOL, pot_err(vt, ref.v_tail[:, :L_real])
