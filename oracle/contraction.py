"""Projective contraction certificate of the band's strictly positive blocks.

TEST INFRASTRUCTURE ONLY, under the same rules as ``eot_oracle``: only ``tests/`` may import
it; the product path never does.

Source: "Blockwise Differentiable Sinkhorn Attention" (gist.science 2605.08123) §2.4, second
certificate: with Hilbert's projective metric, the strictly positive active blocks of the
Sinkhorn map are contractions.

Reading (the pages name the metric and nothing more).  A positive matrix K contracts
Hilbert's projective metric d_H(x, y) = log max_i(x_i / y_i) - log min_i(x_i / y_i) by the
Birkhoff-Hopf ratio kappa(K) = tanh(Delta(K) / 4), where Delta(K) is the projective diameter
of K's image, max over rows i, i' and columns j, j' of log(K_ij K_i'j' / (K_ij' K_i'j)).  With
K = exp(S) on a block that is
    Delta = max_{i, i', j, j'} (S_ij + S_i'j' - S_ij' - S_i'j)
          = max_{i, i'} [ max_j (S_ij - S_i'j) - min_j (S_ij - S_i'j) ].
On a band the kernel is strictly positive only on tile pairs that lie wholly inside it: tile
I (positions [b I, b I + b)) against tile J = I + o with |o| b + b - 1 <= W // 2, i.e.
|o| <= m = (W // 2 - b + 1) // b.  A block is restricted to its active real tokens (the dustbin
and the fillers after it are left out); a tile pair with no active row or column has no block.
"""
from __future__ import annotations

import math

import numpy as np


def block_diameter(B: np.ndarray) -> float:
    """Delta of exp(B) for a float64 score block [rows, cols] (0 for a single row or column)."""
    B = np.asarray(B, np.float64)
    if B.shape[0] < 2 or B.shape[1] < 2:
        return 0.0
    best = 0.0
    for i in range(B.shape[0]):
        diff = B[i][None, :] - B          # row i minus every row i'
        best = max(best, float(np.max(diff.max(axis=1) - diff.min(axis=1))))
    return best


def block_diameter_brute(B: np.ndarray) -> float:
    """Delta by its definition, over every (i, i', j, j') (tiny blocks only)."""
    B = np.asarray(B, np.float64)
    r, c = B.shape
    best = 0.0
    for i in range(r):
        for i2 in range(r):
            for j in range(c):
                for j2 in range(c):
                    best = max(best, B[i, j] + B[i2, j2] - B[i, j2] - B[i2, j])
    return best


def hilbert_distance(x: np.ndarray, y: np.ndarray) -> float:
    """d_H(x, y) for strictly positive vectors."""
    r = np.log(np.asarray(x, np.float64)) - np.log(np.asarray(y, np.float64))
    return float(r.max() - r.min())


def offsets(W: int, tile: int = 128) -> int:
    """m: tile offsets -m..m lie wholly inside the band (-1: none)."""
    h = W // 2
    return (h - tile + 1) // tile if h >= tile - 1 else -1


def contraction_tiles(q, k, W: int, scale: float | None = None, mask_row=None, dustbin_index: int = -1,
                      tile: int = 128) -> np.ndarray:
    """kappa [nT, 2m + 1] for one unit: entry (I, o + m) is tanh(Delta / 4) of the active block of
    tiles (I, I + o), or -1 where I + o is out of range or the block has no active row or column."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    S = scale * (q @ k.T)
    act = np.ones(L, bool) if mask_row is None else np.asarray(mask_row).astype(bool).copy()
    if dustbin_index >= 0:
        act[dustbin_index:] = False
    nT = (L + tile - 1) // tile
    m = offsets(W, tile)
    out = np.full((nT, max(2 * m + 1, 0)), -1.0)
    for I in range(nT):
        for o in range(-m, m + 1):
            J = I + o
            if not 0 <= J < nT:
                continue
            rows = np.arange(I * tile, min(L, I * tile + tile))
            cols = np.arange(J * tile, min(L, J * tile + tile))
            rows, cols = rows[act[rows]], cols[act[cols]]
            if rows.size == 0 or cols.size == 0:
                continue
            out[I, o + m] = math.tanh(block_diameter(S[np.ix_(rows, cols)]) / 4.0)
    return out
