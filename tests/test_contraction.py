"""Projective contraction certificate of the band's strictly positive blocks (BDSA §2.4, second
certificate: Hilbert's projective metric shows the strictly positive active blocks of the
Sinkhorn map contract).

CPU: the oracle's diameter (``oracle.contraction``) against its definition by brute force,
closed forms, the Birkhoff-Hopf bound itself on random positive vectors, and the symmetry of
the diameter under transposition.  GPU: the library's per-tile ratios against the oracle's.
"""
import math

import numpy as np
import pytest

import eot_inputs
from oracle import contraction as oc


@pytest.mark.parametrize("shape,seed", [((3, 4), 0), ((5, 5), 1), ((4, 2), 2), ((6, 3), 3)])
def test_diameter_equals_its_definition(shape, seed):
    B = np.random.default_rng(seed).standard_normal(shape) * 2.0
    assert oc.block_diameter(B) == pytest.approx(oc.block_diameter_brute(B), rel=1e-13, abs=1e-13)


def test_rank_one_and_two_by_two_closed_forms():
    rng = np.random.default_rng(4)
    a, b = rng.standard_normal(7), rng.standard_normal(5)
    assert oc.block_diameter(a[:, None] + b[None, :]) == pytest.approx(0.0, abs=1e-12)   # one ray
    for x in (0.3, -1.7, 5.0):
        assert oc.block_diameter(np.array([[0.0, 0.0], [0.0, x]])) == pytest.approx(abs(x))
    assert oc.block_diameter(np.ones((1, 6))) == 0.0 and oc.block_diameter(np.ones((6, 1))) == 0.0


@pytest.mark.parametrize("seed", [5, 6, 7])
def test_birkhoff_hopf_bound_holds(seed):
    """d_H(K x, K y) <= tanh(Delta / 4) d_H(x, y) for K = exp(B) and positive x, y."""
    rng = np.random.default_rng(seed)
    B = rng.standard_normal((8, 6))
    K = np.exp(B)
    kappa = math.tanh(oc.block_diameter(B) / 4.0)
    assert 0.0 < kappa < 1.0
    worst = 0.0
    for _ in range(2000):
        x, y = np.exp(rng.standard_normal(6) * 2), np.exp(rng.standard_normal(6) * 2)
        ratio = oc.hilbert_distance(K @ x, K @ y) / oc.hilbert_distance(x, y)
        assert ratio <= kappa + 1e-12
        worst = max(worst, ratio)
    assert worst > 0.2 * kappa   # the bound is not vacuous on this block


def test_tiles_transpose_symmetry_and_edges():
    """Delta(B) = Delta(B^T): tile (I, I + o) of (q, k) equals tile (I + o, I) of (k, q).  Tiles
    out of range and tiles without active tokens are -1; a band narrower than a tile has none."""
    rng = np.random.default_rng(8)
    L, d, W, t = 40, 3, 24, 4                      # tile 4: m = (12 - 3) // 4 = 2
    q, k = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    mask = np.ones(L, np.uint8)
    mask[8:12] = 0                                 # tile 2 wholly inactive
    a = oc.contraction_tiles(q, k, W, mask_row=mask, tile=t)
    b = oc.contraction_tiles(k, q, W, mask_row=mask, tile=t)
    m = oc.offsets(W, t)
    assert m == 2 and a.shape == (10, 5)
    for I in range(10):
        for o in range(-m, m + 1):
            J = I + o
            if 0 <= J < 10:
                assert a[I, o + m] == pytest.approx(b[J, -o + m], abs=1e-13)
            else:
                assert a[I, o + m] == -1.0
    assert np.all(a[2] == -1.0) and a[0, 2 + m] == -1.0   # rows of tile 2, columns of tile 2
    assert ((a == -1.0) | ((a >= 0.0) & (a < 1.0))).all()
    assert oc.contraction_tiles(q, k, 4, tile=t).shape == (10, 0)   # W // 2 = 2 < t - 1


def _ragged(B, L, seed):
    rng = np.random.default_rng(seed)
    m = np.zeros((B, L), np.uint8)
    for b in range(B):
        n = int(rng.integers(L // 2, L + 1))
        m[b, :n] = 1
        m[b, rng.choice(n, size=max(1, n // 40), replace=False)] = 0
    return m


@pytest.mark.gpu
@pytest.mark.parametrize("kind", ["fp32_d40_masked", "bf16_d64_W1024", "bf16_dustbin_masked", "narrow_band"])
def test_contraction_matches_oracle(kind):
    """eot_contraction's per-tile ratios equal the oracle's (float64 scores from the same
    inputs); the -1 entries (pairs out of range or without active tokens) match exactly."""
    import torch
    from entropic_ot_attention_b200 import contraction_certificate
    D = None
    if kind == "fp32_d40_masked":
        case = eot_inputs.dense_case(2, 2, 640, 40, 700, 1, 1, "fp32", seed=31, mask=_ragged(2, 640, 31))
    elif kind == "bf16_d64_W1024":
        case = eot_inputs.dense_case(2, 1, 768, 64, 1024, 1, 1, "bf16", seed=32)
    elif kind == "bf16_dustbin_masked":
        case = eot_inputs.dustbin_case(1, 2, 500, 32, 600, 1, 1, "bf16", seed=33, mask=_ragged(1, 500, 33)[0:1])
        D = case.dustbin_index
    else:
        case = eot_inputs.dense_case(1, 1, 256, 32, 200, 1, 1, "fp32", seed=34)
    dev = torch.device("cuda:0")
    tdt = torch.float32 if case.dtype == "fp32" else torch.bfloat16
    q, k = (torch.from_numpy(x).to(dev).to(tdt).contiguous() for x in (case.Q, case.K))
    mask = None if case.mask is None else torch.from_numpy(case.mask).to(dev)
    kappa = contraction_certificate(q, k, case.W, mask=mask, scale=case.scale, dustbin_index=D)
    torch.cuda.synchronize()
    got = kappa.cpu().numpy()
    B, H = case.Q.shape[:2]
    for b in range(B):
        for h in range(H):
            want = oc.contraction_tiles(case.Q[b, h].astype(np.float64), case.K[b, h].astype(np.float64), case.W,
                                        case.scale, None if case.mask is None else case.mask[b],
                                        -1 if D is None else D)
            assert got[b, h].shape == want.shape
            assert np.array_equal(got[b, h] == -1.0, want == -1.0)
            np.testing.assert_allclose(got[b, h], want, atol=1e-4, rtol=0)
    if kind == "narrow_band":
        assert got.shape[-1] == 0
    else:
        assert (got > 0.0).any()


def test_offsets_and_argument_errors():
    """eot_contraction_offsets follows |o| 128 + 127 <= W / 2; null tensors are refused before
    anything is launched (no GPU needed)."""
    import torch
    from entropic_ot_attention_b200 import _abi, api
    for W, n in ((1024, 7), (254, 1), (253, 0), (0, 0), (700, 3)):
        p = api.make_problem(1, 2, 1024, 64, W, 1, 1, torch.bfloat16)
        assert _abi.eot_contraction_offsets(p) == n == max(2 * oc.offsets(W) + 1, 0)
    bad = api.make_problem(1, 2, 1000, 64, 512, 1, 1, torch.bfloat16)   # L not a multiple of 128
    assert _abi.eot_contraction_offsets(bad) == -1
    p = api.make_problem(1, 2, 1024, 64, 1024, 1, 1, torch.bfloat16)
    assert _abi.lib.eot_contraction(__import__("ctypes").byref(p), None, None, None, None, None) == \
        _abi.EOT_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("W,t", [(24, 4), (23, 4), (30, 5), (1024, 128)])
def test_reported_pairs_are_exactly_the_wholly_supported_ones(W, t):
    """The tile pairs the certificate reports (|o| <= m) are those on which the band support of
    eot_oracle.unit_structure is complete, so exp(S) is strictly positive there; at |o| = m + 1
    some entry of the pair lies outside the band."""
    from oracle import eot_oracle as eo
    L = 12 * t
    sup = eo.unit_structure(L, W).support
    m = oc.offsets(W, t)
    I = 5
    for o in range(0, m + 2):
        J = I + o
        full = bool(sup[I * t:(I + 1) * t, J * t:(J + 1) * t].all())
        assert full == (o <= m), (o, m)
