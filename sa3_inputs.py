"""Seeded synthetic Q, K, V for microscaled-FP4 attention.

This module holds no arithmetic of the attention method: it only draws
random tensors.  Both the CUDA path's tests/bench and the CPU oracle's tests
take their inputs from here, so the two sides see the same bytes.

The workloads stand in for the pages' LLM-prefill and video-DiT attention
layers ("SageAttention" summary, "Key results": Llama2, CogvideoX, ...),
whose datasets and weights are not available; the shapes and distributions
are fixed below.

Recipe (one torch CPU generator, seed 0 unless given):
  1. draw the base of Q, then K, then V, each per (b, h) slice in order,
     in fp32: standard normal, or Student-t(nu) = Z / sqrt(chi2_nu / nu)
     with chi2_nu the sum of nu squared normals drawn right after Z,
     optionally scaled by sqrt((nu - 2) / nu) to unit variance;
  2. draw outlier channels, per (b, h) without replacement, for Q then K
     (torch.randperm, first n_out entries) and multiply those channels by
     the factor;
  3. draw the per-(b, h, channel) K offset ~ N(0, std^2), shared by all
     tokens, and add it to K;
  4. round to bf16 (round to nearest even) last.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dist: str = "normal"          # "normal" or "student_t"
    nu: int = 0                    # Student-t degrees of freedom
    unit_var: bool = False         # scale Student-t to unit variance
    k_offset_std: float = 2.0      # K per-channel offset ~ N(0, std^2)
    q_outliers: tuple = (0, 1.0)   # (channels per (b,h), factor)
    k_outliers: tuple = (0, 1.0)

    @property
    def ops(self) -> float:
        """Attention operations 4*B*H*N^2*d, halved for the causal mask."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f


WORKLOADS = {
    # tiny non-causal case the oracle finishes in seconds
    "tiny_b1h2n256d64": Workload("tiny_b1h2n256d64", 1, 2, 256, 64, False),
    # non-causal, the headline throughput case
    "noncausal_b2h16n4096d128": Workload("noncausal_b2h16n4096d128", 2, 16, 4096, 128, False,
                                         q_outliers=(4, 20.0)),
    # video-DiT shaped, ragged tail (17776 = 138*128 + 112)
    "videodit_b1h30n17776d64": Workload("videodit_b1h30n17776d64", 1, 30, 17776, 64, False,
                                        dist="student_t", nu=3, unit_var=True, k_offset_std=3.0),
    # LLM prefill, causal
    "prefill_b4h32n8192d128_causal": Workload("prefill_b4h32n8192d128_causal", 4, 32, 8192, 128, True,
                                              q_outliers=(8, 30.0), k_outliers=(8, 30.0)),
    # long context, causal, heavy tails (not rescaled)
    "longctx_b1h32n32768d128_causal": Workload("longctx_b1h32n32768d128_causal", 1, 32, 32768, 128, True,
                                               dist="student_t", nu=4, unit_var=False),
}
ORDER = list(WORKLOADS)


def _base(g: torch.Generator, w: Workload, n: int, d: int) -> torch.Tensor:
    z = torch.randn((n, d), generator=g, dtype=torch.float32)
    if w.dist == "normal":
        return z
    chi2 = torch.zeros((n, d), dtype=torch.float32)
    for _ in range(w.nu):
        e = torch.randn((n, d), generator=g, dtype=torch.float32)
        chi2.addcmul_(e, e)
    z.div_(torch.sqrt(chi2 / w.nu))
    if w.unit_var:
        z.mul_(math.sqrt((w.nu - 2) / w.nu))
    return z


def make_qkv(w: Workload | str, seed: int = 0, shape_override: dict | None = None):
    """Return bf16 CPU tensors q, k, v of shape [B, H, N, d].

    ``shape_override`` (e.g. ``{"N": 129}``) keeps the distribution of ``w``
    but changes its sizes; used for edge cases."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if shape_override:
        w = dataclasses.replace(w, **shape_override)
    g = torch.Generator().manual_seed(seed)
    B, H, N, d = w.B, w.H, w.N, w.d
    out = []
    for _name in ("q", "k", "v"):
        t = torch.empty((B, H, N, d), dtype=torch.float32)
        for b in range(B):
            for h in range(H):
                t[b, h] = _base(g, w, N, d)
        out.append(t)
    q, k, v = out
    for t, (n_out, factor) in ((q, w.q_outliers), (k, w.k_outliers)):
        if n_out <= 0:
            continue
        for b in range(B):
            for h in range(H):
                ch = torch.randperm(d, generator=g)[:n_out]
                t[b, h][:, ch] *= factor
    off = torch.randn((B, H, 1, d), generator=g, dtype=torch.float32) * w.k_offset_std
    k += off
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
