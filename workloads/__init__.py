"""Seeded synthetic inputs for the ClusterAttention forward path.

This module only draws random tensors. It contains none of the method's
arithmetic, and both the fp64 oracle and the CUDA path read what it makes.

Every workload stands in for one of the paper's evaluation settings
(ClusterAttention: A training-free speedup of bidirectional attention,
Section 4 "Results"): the tabular TabPFN-3 rows and the Wan 2.1 video
latents are not available, so their shapes and statistics are imitated with
seeded Gaussian / sinusoidal data.

All draws use NumPy's PCG64 with ``seed = 1000 + config_id`` (or an explicit
seed), are made in float64 and are rounded once to the storage dtype:
bf16 by round-to-nearest-even applied directly to the float64 value, fp32 by
NumPy's own float64 -> float32 cast.

Returned tensors are head-major ``[B, H, N_alloc, d]`` numpy arrays:
* ``bf16`` workloads hold the bf16 values widened to float32 (exact), plus a
  ``*_bits`` uint16 view that is the bf16 bit pattern;
* ``fp32`` workloads hold float32 values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Workload",
    "round_to_bf16",
    "bf16_bits",
    "make_workload",
    "config_workload",
    "gaussian_mixture_qkv",
    "lowrank_qkv",
    "grid_sinusoid_qkv",
    "heavy_tail_mixture_qkv",
    "CONFIG_SHAPES",
]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), once.

    Returns float64 values that are exactly representable in bf16.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                 # x = m * 2**e, 0.5 <= |m| < 1
    # bf16 keeps 8 significant bits: scale the mantissa to [128, 256).
    r = np.rint(m * 256.0)             # numpy rint rounds half to even
    return np.ldexp(r / 256.0, e)


def bf16_bits(x_bf16_exact: np.ndarray) -> np.ndarray:
    """uint16 bit pattern of values already exactly representable in bf16."""
    f32 = np.ascontiguousarray(x_bf16_exact, dtype=np.float32)
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass
class Workload:
    """One synthetic attention-layer input."""
    name: str
    B: int
    H: int
    N_alloc: int
    n_valid: int
    d: int
    c: int
    k: int
    dtype: str                  # "bf16" or "fp32"
    compensate: bool
    Q: np.ndarray               # [B,H,N_alloc,d] float32 (bf16-exact when dtype == bf16)
    K: np.ndarray
    V: np.ndarray
    seed: int

    @property
    def C(self) -> int:
        return -(-self.n_valid // self.c)

    def bits(self, name: str) -> np.ndarray:
        """bf16 bit pattern of Q, K or V (bf16 workloads only)."""
        assert self.dtype == "bf16"
        return bf16_bits(getattr(self, name))


def _finish(x64: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(x64).astype(np.float32)
    if dtype == "fp32":
        return x64.astype(np.float32)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Generators. Each returns float64 [H, N, d] arrays for Q, K, V (one batch).
# ---------------------------------------------------------------------------

def gaussian_mixture_qkv(rng: np.random.Generator, H: int, N: int, d: int,
                         n_comp: int = 8, std: float = 0.3):
    """Gaussian mixture with component means ~ N(0, I_d), per-component std
    ``std``. Queries and keys share one label per token (q_i and k_i come from
    the same component, with independent noise); values use their own labels.
    """
    Q = np.empty((H, N, d)); K = np.empty((H, N, d)); V = np.empty((H, N, d))
    for h in range(H):
        mu = rng.standard_normal((n_comp, d))
        z = rng.integers(0, n_comp, size=N)
        Q[h] = mu[z] + std * rng.standard_normal((N, d))
        K[h] = mu[z] + std * rng.standard_normal((N, d))
        zv = rng.integers(0, n_comp, size=N)
        V[h] = mu[zv] + std * rng.standard_normal((N, d))
    return Q, K, V


def lowrank_qkv(rng: np.random.Generator, H: int, N: int, d: int,
                rank: int = 16, noise: float = 0.1):
    """Per-head low-rank Gaussian projections plus noise (tabular-shaped).

    A latent Z (N x rank, N(0,1)) is shared by Q and K of one head;
    Q = Z A_q + noise * E, K = Z A_k + noise * E', A entries ~ N(0, 1/rank).
    V ~ N(0, 1).
    """
    Q = np.empty((H, N, d)); K = np.empty((H, N, d)); V = np.empty((H, N, d))
    s = 1.0 / math.sqrt(rank)
    for h in range(H):
        Z = rng.standard_normal((N, rank))
        Aq = s * rng.standard_normal((rank, d))
        Ak = s * rng.standard_normal((rank, d))
        Q[h] = Z @ Aq + noise * rng.standard_normal((N, d))
        K[h] = Z @ Ak + noise * rng.standard_normal((N, d))
        V[h] = rng.standard_normal((N, d))
    return Q, K, V


def grid_sinusoid_qkv(rng: np.random.Generator, H: int, grid=(21, 45, 80),
                      N_alloc: Optional[int] = None, d: int = 128,
                      noise: float = 0.5):
    """Video-latent-shaped features on a (T, Hh, W) grid.

    Channel j of Q (and, with its own draws, of K) is
    sin(2*pi*(w_t t/T + w_h h/Hh + w_w w/W) + phi) with integer frequencies
    w ~ U{1..4} per axis and phase phi ~ U[0, 2pi), plus ``noise`` * N(0,1).
    The grid rows are shuffled by one seeded permutation shared by Q, K and V
    (so no spatial order survives). V ~ N(0,1). Rows past the grid
    (padding up to N_alloc) are zero.
    """
    T, Hh, W = grid
    n = T * Hh * W
    N_alloc = N_alloc or n
    tt, hh, ww = np.meshgrid(np.arange(T) / T, np.arange(Hh) / Hh,
                             np.arange(W) / W, indexing="ij")
    coords = np.stack([tt.ravel(), hh.ravel(), ww.ravel()], axis=1)  # [n,3]
    perm = rng.permutation(n)
    coords = coords[perm]
    Q = np.zeros((H, N_alloc, d)); K = np.zeros((H, N_alloc, d)); V = np.zeros((H, N_alloc, d))
    for h in range(H):
        for X in (Q, K):
            om = rng.integers(1, 5, size=(d, 3)).astype(np.float64)
            ph = rng.uniform(0.0, 2.0 * math.pi, size=d)
            X[h, :n] = np.sin(2.0 * math.pi * (coords @ om.T) + ph) \
                + noise * rng.standard_normal((n, d))
        V[h, :n] = rng.standard_normal((n, d))
    return Q, K, V


def heavy_tail_mixture_qkv(rng: np.random.Generator, H: int, N: int, d: int,
                           n_comp: int = 64, std: float = 0.3, nu: float = 3.0):
    """Gaussian mixture whose component weights are heavy-tailed:
    pi_j proportional to |t_j| with t_j ~ Student-t(nu). Means ~ N(0, I_d);
    Q and K share labels and means, with independent noise; V ~ N(0,1).
    """
    Q = np.empty((H, N, d)); K = np.empty((H, N, d)); V = np.empty((H, N, d))
    for h in range(H):
        mu = rng.standard_normal((n_comp, d))
        t = np.abs(rng.standard_t(nu, size=n_comp))
        pi = t / t.sum()
        z = rng.choice(n_comp, size=N, p=pi)
        Q[h] = mu[z] + std * rng.standard_normal((N, d))
        K[h] = mu[z] + std * rng.standard_normal((N, d))
        V[h] = rng.standard_normal((N, d))
    return Q, K, V


# ---------------------------------------------------------------------------
# The five workload configurations.
# ---------------------------------------------------------------------------

CONFIG_SHAPES = {
    # id: (B, H, N_alloc, n_valid, d, c, k, dtype)
    1: (1, 1, 1024, 1024, 64, 64, 4, "fp32"),
    2: (1, 8, 65536, 65536, 64, 128, 64, "bf16"),
    3: (1, 40, 76800, 75600, 128, 128, 89, "bf16"),
    4: (1, 4, 262144, 262144, 64, 256, 64, "bf16"),
}


def make_workload(kind: str, *, B: int = 1, H: int, N: int, d: int, c: int,
                  k: int, dtype: str = "bf16", seed: int = 0,
                  n_valid: Optional[int] = None, compensate: bool = True,
                  name: Optional[str] = None, **gen_kw) -> Workload:
    """Build a workload of any size with one of the generators.

    kind: "mixture" | "lowrank" | "grid" | "heavytail".
    For "grid", ``gen_kw['grid']`` gives (T, Hh, W) and N is N_alloc.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    Qs, Ks, Vs = [], [], []
    for _ in range(B):
        if kind == "mixture":
            q, kk, v = gaussian_mixture_qkv(rng, H, N, d, **gen_kw)
            nv = N if n_valid is None else n_valid
        elif kind == "lowrank":
            q, kk, v = lowrank_qkv(rng, H, N, d, **gen_kw)
            nv = N if n_valid is None else n_valid
        elif kind == "grid":
            grid = gen_kw.pop("grid", (21, 45, 80))
            q, kk, v = grid_sinusoid_qkv(rng, H, grid=grid, N_alloc=N, d=d, **gen_kw)
            nv = grid[0] * grid[1] * grid[2]
        elif kind == "heavytail":
            q, kk, v = heavy_tail_mixture_qkv(rng, H, N, d, **gen_kw)
            nv = N if n_valid is None else n_valid
        else:
            raise ValueError(kind)
        Qs.append(_finish(q, dtype)); Ks.append(_finish(kk, dtype)); Vs.append(_finish(v, dtype))
    Q = np.stack(Qs); K = np.stack(Ks); V = np.stack(Vs)
    if nv < N:
        # Rows past n_valid are padding: zero, never read as tokens.
        Q[:, :, nv:] = 0; K[:, :, nv:] = 0; V[:, :, nv:] = 0
    return Workload(name=name or f"{kind}-H{H}-N{N}-d{d}-c{c}-k{k}", B=B, H=H,
                    N_alloc=N, n_valid=nv, d=d, c=c, k=k, dtype=dtype,
                    compensate=compensate, Q=Q, K=K, V=V, seed=seed)


def config_workload(config_id: int, *, H: Optional[int] = None,
                    seed: Optional[int] = None, d: Optional[int] = None,
                    c: Optional[int] = None, keep: Optional[float] = None,
                    compensate: bool = True) -> Workload:
    """The named workload configurations.

    1: single head, N=1024, d=64, fp32, 8-component mixture (std 0.3), c=64, k=4.
    2: tabular-shaped, H=8, N=65,536, d=64, bf16, rank-16 low-rank + 0.1 noise, c=128, k=64.
    3: video-shaped, H=40, 21x45x80 = 75,600 tokens padded to 76,800, d=128,
       bf16, grid sinusoids + 0.5 noise, shuffled rows, c=128, k=ceil(0.15*591)=89.
    4: large tabular-shaped, H=4, N=262,144, d=64, bf16, 64-component mixture
       with Student-t(3) weights, c=256, k=64.
    5: sweep, H=8, N=32,768, d in {64,128}, bf16, config 2's generator,
       c in {64,128,256}, keep fraction in {1/32, 1/8, 1/4, 1}.

    ``H`` may be lowered (heads are independent draws in order, so the first
    h heads of a smaller draw equal the first h heads of the full one).
    """
    s = 1000 + config_id if seed is None else seed
    if config_id == 1:
        B, Hf, N, nv, dd, cc, kk, dt = CONFIG_SHAPES[1]
        return make_workload("mixture", B=B, H=H or Hf, N=N, d=dd, c=cc, k=kk,
                             dtype=dt, seed=s, compensate=compensate,
                             name="cfg1-mixture-N1024-d64-fp32", n_comp=8, std=0.3)
    if config_id == 2:
        B, Hf, N, nv, dd, cc, kk, dt = CONFIG_SHAPES[2]
        return make_workload("lowrank", B=B, H=H or Hf, N=N, d=dd, c=cc, k=kk,
                             dtype=dt, seed=s, compensate=compensate,
                             name="cfg2-lowrank-N65536-d64-bf16", rank=16, noise=0.1)
    if config_id == 3:
        B, Hf, N, nv, dd, cc, kk, dt = CONFIG_SHAPES[3]
        return make_workload("grid", B=B, H=H or Hf, N=N, d=dd, c=cc, k=kk,
                             dtype=dt, seed=s, compensate=compensate,
                             name="cfg3-grid-21x45x80-d128-bf16", grid=(21, 45, 80),
                             noise=0.5)
    if config_id == 4:
        B, Hf, N, nv, dd, cc, kk, dt = CONFIG_SHAPES[4]
        return make_workload("heavytail", B=B, H=H or Hf, N=N, d=dd, c=cc, k=kk,
                             dtype=dt, seed=s, compensate=compensate,
                             name="cfg4-heavytail-N262144-d64-bf16", n_comp=64,
                             std=0.3, nu=3.0)
    if config_id == 5:
        dd = d or 64
        cc = c or 128
        N = 32768
        C = -(-N // cc)
        f = 1.0 / 8 if keep is None else keep
        kk = max(1, math.ceil(f * C))
        return make_workload("lowrank", B=1, H=H or 8, N=N, d=dd, c=cc, k=kk,
                             dtype="bf16", seed=s, compensate=compensate,
                             name=f"cfg5-lowrank-N32768-d{dd}-c{cc}-k{kk}"
                                  f"-{'smc' if compensate else 'nosmc'}",
                             rank=16, noise=0.1)
    raise ValueError(config_id)
