"""Seeded synthetic inputs for band Sinkhorn attention, shared by the oracle and the GPU path.

This module holds none of the method's arithmetic: it only draws random tensors, rounds
them to the run's input dtype, and builds masks.  Both sides (the float64 oracle and the
CUDA library) are fed the exact same values.

Every generator uses numpy ``Generator(PCG64(seed))`` and draws float32 normals in a
fixed order (stated per workload).  bf16 inputs are rounded to nearest-even bf16 and kept
in float32 arrays, so converting them to torch.bfloat16 is exact.

Named workloads (sizes as used by tests and bench.py):

``tiny``      B=1 H=1 L=256 d=32 W=32 fp32, Q,K,V,dO ~ N(0,1), T=50 R=2
``medium``    B=4 H=8 L=4096 d=64 W=256 bf16, Q,K,V,dO ~ N(0,1), T=20 R=2
``dustbin``   B=2 H=8, 16384 real tokens + 1 dustbin + 127 fillers (L=16512), d=64 W=512 bf16,
              Q,K,V,dO ~ N(0,1) on real rows, one dustbin q/k/v per head ~ N(0,1),
              dustbin mass 0.1, T=20 R=2
``protein``   32 sequences, tokens uniform over 25 symbols, lengths uniform in [256, 2048]
              padded to 2048 (masked fillers), embedding tables E_q, E_k, E_v [25, H=4, 128]
              ~ N(0,1) (random init), bf16, W=128, T=30, R=2 (``protein_r4``: R=4)
``long``      B=1 H=4 L=131072 d=128 W=1024 bf16, Q,K,V ~ N(0, std 1/sqrt(d)), dO ~ N(0,1),
              T=10 R=2
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "fp32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return round_to_bf16(x)
    raise ValueError(f"unknown dtype {dtype}")


@dataclass
class Case:
    """One seeded problem instance.  Arrays are float32 holding dtype-exact values."""

    name: str
    Q: np.ndarray
    K: np.ndarray
    V: np.ndarray
    dO: np.ndarray
    mask: np.ndarray | None          # uint8 [B, L] (1 = active real token) or None
    W: int
    T: int
    R: int
    dtype: str                       # "fp32" | "bf16"
    dustbin: bool = False
    dustbin_index: int = -1
    dustbin_mass: float = 0.0
    scale: float | None = None       # None: 1/sqrt(d)
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        return self.Q.shape

    def oracle_kwargs(self) -> dict:
        return dict(W=self.W, T=self.T, R=self.R, scale=self.scale, mask=self.mask,
                    dustbin=self.dustbin, dustbin_index=self.dustbin_index,
                    dustbin_mass=self.dustbin_mass)


def _normal(rng, shape, std=1.0):
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def dense_case(B, H, L, d, W, T, R, dtype="bf16", seed=0, std=1.0, mask=None, name="custom",
               scale=None) -> Case:
    """Q, K, V, dO ~ N(0, std^2) (dO ~ N(0,1)), drawn in that order; masked rows zeroed."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Q = _normal(rng, (B, H, L, d), std)
    K = _normal(rng, (B, H, L, d), std)
    V = _normal(rng, (B, H, L, d), std)
    dO = _normal(rng, (B, H, L, d))
    if mask is not None:
        mask = np.ascontiguousarray(mask, np.uint8)
        z = (mask == 0)[:, None, :, None]
        Q[np.broadcast_to(z, Q.shape)] = 0
        K[np.broadcast_to(z, K.shape)] = 0
        V[np.broadcast_to(z, V.shape)] = 0
        dO[np.broadcast_to(z, dO.shape)] = 0
    return Case(name, to_dtype(Q, dtype), to_dtype(K, dtype), to_dtype(V, dtype), to_dtype(dO, dtype),
                mask, W, T, R, dtype, scale=scale)


def dustbin_case(B, H, L_real, d, W, T, R, dtype="bf16", seed=0, mass=0.1, tile=128, mask=None,
                 name="custom_dustbin") -> Case:
    """Real tokens, then one dustbin token at index L_real, then fillers up to a tile multiple.

    Draw order: Q, K, V, dO over [B,H,L_real,d], then dustbin q, k, v over [H, d]."""
    L = ((L_real + 1 + tile - 1) // tile) * tile
    rng = np.random.Generator(np.random.PCG64(seed))
    Qr = _normal(rng, (B, H, L_real, d))
    Kr = _normal(rng, (B, H, L_real, d))
    Vr = _normal(rng, (B, H, L_real, d))
    dOr = _normal(rng, (B, H, L_real, d))
    qD = _normal(rng, (H, d))
    kD = _normal(rng, (H, d))
    vD = _normal(rng, (H, d))
    Q = np.zeros((B, H, L, d), np.float32)
    K = np.zeros_like(Q)
    V = np.zeros_like(Q)
    dO = np.zeros_like(Q)
    Q[:, :, :L_real], K[:, :, :L_real], V[:, :, :L_real], dO[:, :, :L_real] = Qr, Kr, Vr, dOr
    Q[:, :, L_real] = qD[None]
    K[:, :, L_real] = kD[None]
    V[:, :, L_real] = vD[None]
    full_mask = None
    if mask is not None:
        full_mask = np.zeros((B, L), np.uint8)
        full_mask[:, :L_real] = mask
        z = (full_mask == 0)
        z[:, L_real] = False
        zz = z[:, None, :, None]
        for X in (Q, K, V, dO):
            X[np.broadcast_to(zz, X.shape)] = 0
    return Case(name, to_dtype(Q, dtype), to_dtype(K, dtype), to_dtype(V, dtype), to_dtype(dO, dtype),
                full_mask, W, T, R, dtype, dustbin=True, dustbin_index=L_real, dustbin_mass=mass,
                meta={"L_real": L_real})


def protein_case(n_seq=32, H=4, d=128, L=2048, min_len=256, W=128, T=30, R=2, dtype="bf16", seed=0,
                 n_symbols=25, name="protein") -> Case:
    """Protein-like ragged batch.  Draw order: lengths, tokens, E_q, E_k, E_v, dO."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lengths = rng.integers(min_len, L, size=n_seq, endpoint=True)
    tokens = rng.integers(0, n_symbols, size=(n_seq, L))
    Eq = _normal(rng, (n_symbols, H, d))
    Ek = _normal(rng, (n_symbols, H, d))
    Ev = _normal(rng, (n_symbols, H, d))
    dO = _normal(rng, (n_seq, H, L, d))
    mask = (np.arange(L)[None, :] < lengths[:, None]).astype(np.uint8)
    Q = np.ascontiguousarray(np.transpose(Eq[tokens], (0, 2, 1, 3)))
    K = np.ascontiguousarray(np.transpose(Ek[tokens], (0, 2, 1, 3)))
    V = np.ascontiguousarray(np.transpose(Ev[tokens], (0, 2, 1, 3)))
    z = (mask == 0)[:, None, :, None]
    for X in (Q, K, V, dO):
        X[np.broadcast_to(z, X.shape)] = 0
    return Case(name, to_dtype(Q, dtype), to_dtype(K, dtype), to_dtype(V, dtype), to_dtype(dO, dtype),
                mask, W, T, R, dtype, meta={"lengths": lengths})


def workload(name: str, seed: int = 0) -> Case:
    """The named workloads of the module docstring."""
    if name == "tiny":
        return dense_case(1, 1, 256, 32, 32, 50, 2, "fp32", seed, name=name)
    if name == "medium":
        return dense_case(4, 8, 4096, 64, 256, 20, 2, "bf16", seed, name=name)
    if name == "dustbin":
        return dustbin_case(2, 8, 16384, 64, 512, 20, 2, "bf16", seed, mass=0.1, name=name)
    if name == "protein_r2":
        return protein_case(R=2, seed=seed, name=name)
    if name == "protein_r4":
        return protein_case(R=4, seed=seed, name=name)
    if name == "long":
        return dense_case(1, 4, 131072, 128, 1024, 10, 2, "bf16", seed, std=128 ** -0.5, name=name)
    raise KeyError(name)


WORKLOADS = ("tiny", "medium", "dustbin", "protein_r2", "protein_r4", "long")


def band_entries(case: Case) -> int:
    """Nominal band entries B*H*L*W*(T+R) (the throughput unit); L counts real positions
    (the padded length for ragged batches, the real length for the dustbin layout)."""
    B, H, L, _ = case.Q.shape
    L = case.meta.get("L_real", L)
    return B * H * L * case.W * (case.T + case.R)
