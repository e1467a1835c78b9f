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


# ------------------------------------------------- end-to-end parity chain
def gpu_canonical(qz, B: int, H: int, Nq: int, Nkv: int, d: int) -> dict:
    """The GPU's quantized operands in the oracle's canonical layout."""
    Npq = (Nq + 127) // 128 * 128
    Np = (Nkv + 127) // 128 * 128
    g = {f: getattr(qz, f).cpu().numpy() for f in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean")}
    return dict(q_codes=g["q_fp4"].reshape(B, H, Npq, d // 2), k_codes=g["k_fp4"].reshape(B, H, Np, d // 2),
                vt_codes=g["vt_fp4"].reshape(B, H, d, Np // 2), k_mean=g["k_mean"].reshape(B, H, d),
                q_sf=qk_sf_to_canonical(g["q_sf"], B, H, Npq, d), k_sf=qk_sf_to_canonical(g["k_sf"], B, H, Np, d),
                vt_sf=vt_sf_to_canonical(g["vt_sf"], B, H, Np, d), vt_sf_pad=vt_sf_padding(g["vt_sf"], B, H, Np, d))


def heads_of(t: torch.Tensor, bh_list) -> torch.Tensor:
    """Heads bh_list of a [B,H,N,d] tensor, stacked as [1, len, N, d]."""
    B, H, N, d = t.shape
    return t.reshape(B * H, N, d)[list(bh_list)].reshape(1, len(bh_list), N, d).contiguous()


def oracle_quantize_heads(oracle, q, k, v, bh_list, **kw) -> dict:
    """The oracle's own quantization of heads bh_list (one head's result does
    not depend on the others), as a B=1, H=len(bh_list) operand set."""
    return oracle.quantize_qkv(heads_of(q, bh_list), heads_of(k, bh_list), heads_of(v, bh_list), **kw)


def assert_quantized_equal(gpu: dict, ref: dict, bh_list) -> None:
    """Codes, scales and the K mean of the GPU (canonical, all heads) equal
    the oracle's (heads bh_list only), bit for bit."""
    idx = list(bh_list)
    for f in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf"):
        g = gpu[f].reshape((-1,) + gpu[f].shape[2:])[idx]
        r = ref[f].reshape((-1,) + ref[f].shape[2:])
        if not np.array_equal(g, r):
            bad = np.argwhere(g != r)
            raise AssertionError(f"{f}: {len(bad)} bytes differ from the oracle's, first (head, ...) "
                                 f"{[[idx[b[0]]] + b[1:].tolist() for b in bad[:4]]}")
    gm = gpu["k_mean"].reshape(-1, gpu["k_mean"].shape[-1])[idx]
    rm = ref["k_mean"].reshape(-1, ref["k_mean"].shape[-1])
    assert np.array_equal(gm.view(np.uint32), rm.view(np.uint32)), "k_mean differs from the oracle's"
    if "vt_sf_pad" in gpu:
        assert not gpu["vt_sf_pad"].any(), "padding channels of the V^T scale atoms are not 0"


def _forgive_ties(got: np.ndarray, ref: np.ndarray, ref32: np.ndarray, window: float = 2.0 ** -16):
    """got with every element that is a bf16 rounding tie replaced by ref:
    got and ref are adjacent bf16 values and the oracle's fp32 value before
    its rounding, ref32, lies within `window` (relative) of their midpoint,
    so that an fp32 difference far below any meaningful error (an ulp of the
    row sum, say) decides the rounding either way.  Returns (adjusted got,
    number of elements forgiven)."""
    g = np.ascontiguousarray(got, np.float32)
    r = np.ascontiguousarray(ref, np.float32)
    gb = (g.view(np.uint32) >> 16).astype(np.int64)
    rb = (r.view(np.uint32) >> 16).astype(np.int64)
    mid = (g.astype(np.float64) + r.astype(np.float64)) / 2
    tie = (np.abs(gb - rb) == 1) & ((gb >> 15) == (rb >> 15)) & \
          (np.abs(ref32.astype(np.float64) - mid) <= window * np.abs(mid))
    return np.where(tie, r, g), int(tie.sum())


def blockwise_rel_l2(got: np.ndarray, ref: np.ndarray, blocks, tol: float, live=None, label: str = "",
                     ref32: np.ndarray | None = None) -> float:
    """rel-L2 of got against ref for every (head, Q block) in ``blocks``
    (got, ref: [heads, Nq, d] float arrays; blocks: (head index, q_block)
    pairs; live: optional [Nq] mask of rows that see a key).  With ref32 (the
    oracle's fp32 outputs before their bf16 rounding), bf16 rounding ties are
    not counted as errors (see _forgive_ties).  Fails on any block above
    ``tol``; prints the worst block, the worst single element and the number
    of ties.  Returns the worst block's error."""
    ties = 0
    if ref32 is not None:
        got, ties = _forgive_ties(got, ref, ref32)
    Nq = got.shape[1]
    worst, where = 0.0, None
    for h, qb in blocks:
        rows = np.arange(qb * 128, min(Nq, qb * 128 + 128))
        if live is not None:
            rows = rows[live[rows]]
        if rows.size == 0:
            continue
        g = got[h, rows].astype(np.float64)
        r = ref[h, rows].astype(np.float64)
        nr = np.linalg.norm(r)
        err = np.linalg.norm(g - r) / nr if nr > 0 else np.linalg.norm(g)
        if err > worst:
            worst, where = err, (h, qb)
    dif = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    if live is not None:
        dif = dif[:, live]
    e = np.unravel_index(np.argmax(dif), dif.shape) if dif.size else ()
    print(f"{label} worst block rel-L2 {worst:.3e} at (head, q_block) {where}; "
          f"worst element |diff| {dif.max() if dif.size else 0.0:.3e} at {tuple(int(x) for x in e)}; "
          f"{ties} bf16 ties")
    assert worst <= tol, f"{label} block {where}: rel-L2 {worst:.3e} > {tol}"
    return worst
