"""Helpers shared by the parity tests: layout index maps written from the
comments of include/sa3.h, metrics, and the choice of sampled Q blocks.
Nothing here computes any step of the method."""
from __future__ import annotations

import numpy as np
import torch


def qk_sf_to_canonical(tiled: np.ndarray, B: int, H: int, Np: int, d: int) -> np.ndarray:
    """Scale atoms of Q or K -> canonical [B,H,Np,d/16] via the header's map
    (((bh*(Np/128) + t/128)*(d/64) + c/4)*512 + 16*(t%32) + 4*((t%128)/32) + c%4."""
    bh = np.arange(B * H)[:, None, None]
    t = np.arange(Np)[None, :, None]
    c = np.arange(d // 16)[None, None, :]
    off = (((bh * (Np // 128) + t // 128) * (d // 64) + c // 4) * 512
           + 16 * (t % 32) + 4 * ((t % 128) // 32) + c % 4)
    return tiled.reshape(-1)[off].reshape(B, H, Np, d // 16)


def vt_sf_to_canonical(tiled: np.ndarray, B: int, H: int, Np: int, d: int) -> np.ndarray:
    """Scale atoms of V^T -> canonical [B,H,d,Np/16] via the header's map
    (bh*(Np/64) + u/4)*512 + 16*(c%32) + 4*(c/32) + u%4."""
    bh = np.arange(B * H)[:, None, None]
    c = np.arange(d)[None, :, None]
    u = np.arange(Np // 16)[None, None, :]
    off = (bh * (Np // 64) + u // 4) * 512 + 16 * (c % 32) + 4 * (c // 32) + u % 4
    return tiled.reshape(-1)[off].reshape(B, H, d, Np // 16)


def vt_sf_padding(tiled: np.ndarray, B: int, H: int, Np: int, d: int) -> np.ndarray:
    """Bytes of the padding channels d..127 of every V^T scale atom."""
    if d >= 128:
        return np.zeros(0, np.uint8)
    bh = np.arange(B * H)[:, None, None]
    c = np.arange(d, 128)[None, :, None]
    u = np.arange(Np // 16)[None, None, :]
    off = (bh * (Np // 64) + u // 4) * 512 + 16 * (c % 32) + 4 * (c // 32) + u % 4
    return tiled.reshape(-1)[off]


def fp64_sum_is_exact(k: torch.Tensor) -> bool:
    """True if every per-(b,h,channel) fp64 sum of the bf16 K is exact (so
    any summation order gives the same bits): checked with int64 fixed
    point at the smallest exponent present."""
    kf = k.to(torch.float64)
    nz = kf[kf != 0].abs()
    if nz.numel() == 0:
        return True
    emin = int(torch.floor(torch.log2(nz.min())).item()) - 8
    scaled = kf * (2.0 ** -emin)
    if not torch.equal(scaled, torch.round(scaled)):
        return False
    if scaled.abs().max().item() * k.shape[2] >= 2.0 ** 62:
        return False
    ints = scaled.to(torch.int64).sum(dim=2)
    exact = ints.to(torch.float64) * (2.0 ** emin)  # exact: |ints| < 2^53 checked below
    fsum = kf.sum(dim=2)
    return bool(torch.equal(exact, fsum) and (ints.abs() < 2 ** 53).all())


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def bf16_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().numpy()


def bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


def sample_units(B: int, H: int, N: int, seed: int = 0, per_bh: int = 2, bh_list=None):
    """(bh, q_block) pairs: for each listed (b,h), Q blocks {0, last} plus
    `per_bh` seeded random ones (the last block holds the ragged tail)."""
    nqb = (N + 127) // 128
    rng = np.random.default_rng(seed)
    bhs = range(B * H) if bh_list is None else bh_list
    units = []
    for bh in bhs:
        blocks = {0, nqb - 1}
        if nqb > 2:
            blocks |= set(int(x) for x in rng.choice(np.arange(1, nqb - 1), size=min(per_bh, nqb - 2),
                                                      replace=False))
        units += [(bh, qb) for qb in sorted(blocks)]
    return units
