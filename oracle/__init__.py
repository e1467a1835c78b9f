"""CPU oracle for microscaled-FP4 attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, the smoke check in ``__graft_entry__.py`` and the
``cpu_baseline`` / ``--impl reference`` leg of ``bench.py`` may import this
package.  The product path (``bit_quantized_attention_sa3_b200``) never
imports, links or calls it, and this package imports nothing from the
product.  The arithmetic lives in ``sa3_oracle.c`` (plain C, compiled with
``-O2 -fno-fast-math -ffp-contract=off`` so that every fp32 operation is
rounded exactly as written); this file only builds and marshals.

Functions follow the method's steps in order:
  kmean            K smoothing: mean of K over tokens
  quantize_qkv     E2M1 codes + E4M3 scales per 16-element block
  attn_fwd         tiled online-softmax attention on the quantized operands
  attn_exact       fp64 softmax attention on the bf16 inputs (no quantization)
  quantize_qkv_i8,
  attn_fwd_i8      the 8-bit variant: INT8 Q, K per 128-token block, FP16 P, V;
                   optionally the per-row log-sum-exp of the training forward
Layouts are the canonical ones documented in ``sa3_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa3_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BLK = 128
VEC = 16


def gcc_command(src: str, out: str) -> list[str]:
    """The compiler command for the oracle: no fast math, no FMA contraction."""
    return ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
            "-Wno-unused-parameter", src, "-o", out, "-lm"]


def build(force: bool = False) -> str:
    """Compile sa3_oracle.c into liboracle.so next to it (gcc + OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(gcc_command(_SRC, tmp), check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        # SA3_ORACLE_LIB: a library built elsewhere from a copy of the source
        # (the pin suite's own mutation test runs the pins against copies
        # with a planted mistake); unset, the in-tree build
        lib = ctypes.CDLL(os.environ.get("SA3_ORACLE_LIB") or build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        F = ctypes.c_float
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e2m1_value.argtypes = [I]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [I]
        lib.oracle_e2m1_rn.restype = I
        lib.oracle_e2m1_rn.argtypes = [F]
        lib.oracle_e4m3_rn_sat.restype = I
        lib.oracle_e4m3_rn_sat.argtypes = [F]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_f32_to_bf16.argtypes = [F]
        lib.oracle_padded_len.restype = I
        lib.oracle_padded_len.argtypes = [I]
        lib.oracle_kmean.restype = None
        lib.oracle_kmean.argtypes = [P, I, I, I, I, P]
        lib.oracle_quantize_qkv.restype = None
        lib.oracle_quantize_qkv.argtypes = [P, P, P, I, I, I, I, I, I, I] + [P] * 8
        lib.oracle_attn_fwd.restype = None
        lib.oracle_attn_fwd.argtypes = [P] * 6 + [I, I, I, I, I, I, F, I, P, P, I, P, P]
        lib.oracle_attn_exact.restype = None
        lib.oracle_attn_exact.argtypes = [P, P, P, I, I, I, I, I, I, F, P, P, I, P]
        lib.oracle_f32_to_f16.restype = ctypes.c_uint16
        lib.oracle_f32_to_f16.argtypes = [F]
        lib.oracle_quantize_qkv_i8.restype = None
        lib.oracle_quantize_qkv_i8.argtypes = [P, P, P, I, I, I, I, I] + [P] * 6
        lib.oracle_attn_fwd_i8.restype = None
        lib.oracle_attn_fwd_i8.argtypes = [P] * 5 + [I, I, I, I, I, I, F, P, I, P, P]
        lib.oracle_num_threads.restype = I
        lib.oracle_num_threads.argtypes = []
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_u16(x) -> np.ndarray:
    """Accept a bf16 torch tensor or a uint16 numpy array of bf16 bits."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def padded_len(n: int) -> int:
    return (n + BLK - 1) // BLK * BLK


def num_threads() -> int:
    return _load().oracle_num_threads()


def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(code)


def e2m1_rn(x: float) -> int:
    return _load().oracle_e2m1_rn(x)


def e4m3_rn_sat(x: float) -> int:
    return _load().oracle_e4m3_rn_sat(x)


def f32_to_bf16(x: float) -> int:
    return _load().oracle_f32_to_bf16(x)


def kmean(k) -> np.ndarray:
    k = _as_u16(k)
    B, H, N, d = k.shape
    out = np.zeros((B, H, d), np.float32)
    _load().oracle_kmean(_ptr(k), B, H, N, d, _ptr(out))
    return out


def quantize_qkv(q, k, v, smooth_k: bool = True, smooth_v: bool = False) -> dict:
    """Returns canonical-layout arrays: q_codes [B,H,Np(Nq),d/2], q_sf
    [B,H,Np(Nq),d/16], k_codes/k_sf the same over Np(Nkv), vt_codes
    [B,H,d,Np(Nkv)/2], vt_sf [B,H,d,Np(Nkv)/16], k_mean [B,H,d]; and the
    lengths n_q, n_kv; with smooth_v also v_mean [B,H,d] (V quantized after
    subtracting it).  q is [B,H,Nq,d], k and v are [B,H,Nkv,d]."""
    q, k, v = _as_u16(q), _as_u16(k), _as_u16(v)
    B, H, Nq, d = q.shape
    N = k.shape[2]
    assert k.shape == v.shape and k.shape[:2] == (B, H) and k.shape[3] == d
    Npq = padded_len(Nq)
    Np = padded_len(N)
    r = dict(
        q_codes=np.zeros((B, H, Npq, d // 2), np.uint8),
        q_sf=np.zeros((B, H, Npq, d // VEC), np.uint8),
        k_codes=np.zeros((B, H, Np, d // 2), np.uint8),
        k_sf=np.zeros((B, H, Np, d // VEC), np.uint8),
        vt_codes=np.zeros((B, H, d, Np // 2), np.uint8),
        vt_sf=np.zeros((B, H, d, Np // VEC), np.uint8),
        k_mean=np.zeros((B, H, d), np.float32),
        v_mean=np.zeros((B, H, d), np.float32),
    )
    _load().oracle_quantize_qkv(
        _ptr(q), _ptr(k), _ptr(v), B, H, Nq, N, d, int(bool(smooth_k)), int(bool(smooth_v)),
        _ptr(r["q_codes"]), _ptr(r["q_sf"]), _ptr(r["k_codes"]), _ptr(r["k_sf"]),
        _ptr(r["vt_codes"]), _ptr(r["vt_sf"]), _ptr(r["k_mean"]), _ptr(r["v_mean"]))
    if not smooth_v:
        del r["v_mean"]
    r["n_q"], r["n_kv"] = Nq, N
    return r


def _units_arr(units):
    if units is None:
        return None, 0
    u = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 2))
    return u, u.shape[0]


def attn_fwd(qz: dict, N: int, causal: bool, sm_scale: float | None = None,
             units=None, out: np.ndarray | None = None, n_kv: int | None = None,
             p_two_level: bool = False, out32: np.ndarray | None = None) -> np.ndarray:
    """Tiled FP4 attention on canonical-layout quantized operands with N
    query rows and ``n_kv`` key columns (default: qz["n_kv"] if present,
    else N).  Returns bf16 bits uint16 [B,H,N,d]; rows outside ``units``
    stay as in ``out`` (zeros by default).  ``units`` lists (b*H+h,
    q_block) pairs.  p_two_level: P pre-scaled by 2^11 before microscaling
    (R14); qz["v_mean"], if present, is added back after O / l (R13).
    out32 (float32 [B,H,N,d]), if given, receives the same outputs in fp32
    just before their bf16 rounding."""
    if n_kv is None:
        n_kv = qz.get("n_kv", N)
    B, H, Np, dh = qz["q_codes"].shape
    d = dh * 2
    if sm_scale is None:
        sm_scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = np.zeros((B, H, N, d), np.uint16)
    u, nu = _units_arr(units)
    arrs = [np.ascontiguousarray(qz[n]) for n in
            ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf")]
    vm = qz.get("v_mean")
    if vm is not None:
        vm = np.ascontiguousarray(vm, dtype=np.float32)
    if out32 is not None:
        assert out32.dtype == np.float32 and out32.shape == out.shape and out32.flags["C_CONTIGUOUS"]
    _load().oracle_attn_fwd(*[_ptr(a) for a in arrs], B, H, N, n_kv, d, int(bool(causal)),
                            float(sm_scale), int(bool(p_two_level)), _ptr(vm), _ptr(u), nu, _ptr(out), _ptr(out32))
    return out


def attn_exact(q, k, v, causal: bool, sm_scale: float | None = None,
               k_sub: np.ndarray | None = None, units=None) -> np.ndarray:
    """fp64 softmax attention of the bf16 inputs (q [B,H,Nq,d], k and v
    [B,H,Nkv,d]); returns float64 [B,H,Nq,d] (rows outside ``units`` are
    zero)."""
    q, k, v = _as_u16(q), _as_u16(k), _as_u16(v)
    B, H, N, d = q.shape
    Nkv = k.shape[2]
    if sm_scale is None:
        sm_scale = 1.0 / float(np.sqrt(d))
    out = np.zeros((B, H, N, d), np.float64)
    if k_sub is not None:
        k_sub = np.ascontiguousarray(k_sub, dtype=np.float32)
    u, nu = _units_arr(units)
    _load().oracle_attn_exact(_ptr(q), _ptr(k), _ptr(v), B, H, N, Nkv, d, int(bool(causal)),
                              float(sm_scale), _ptr(k_sub), _ptr(u), nu, _ptr(out))
    return out


def f32_to_f16(x: float) -> int:
    return _load().oracle_f32_to_f16(x)


def quantize_qkv_i8(q, k, v) -> dict:
    """8-bit variant (readings I1, I2): q_i8 [B,H,Np(Nq),d] int8, q_scale
    [B,H,Np(Nq)/128] fp32 (one per 128-token block), k_i8 / k_scale the same
    over Np(Nkv) after K smoothing, vt_f16 [B,H,d,Np(Nkv)] fp16 bits (uint16),
    k_mean [B,H,d]; lengths n_q, n_kv."""
    q, k, v = _as_u16(q), _as_u16(k), _as_u16(v)
    B, H, Nq, d = q.shape
    N = k.shape[2]
    Npq, Np = padded_len(Nq), padded_len(N)
    r = dict(q_i8=np.zeros((B, H, Npq, d), np.int8), q_scale=np.zeros((B, H, Npq // BLK), np.float32),
             k_i8=np.zeros((B, H, Np, d), np.int8), k_scale=np.zeros((B, H, Np // BLK), np.float32),
             vt_f16=np.zeros((B, H, d, Np), np.uint16), k_mean=np.zeros((B, H, d), np.float32))
    _load().oracle_quantize_qkv_i8(_ptr(q), _ptr(k), _ptr(v), B, H, Nq, N, d, _ptr(r["q_i8"]), _ptr(r["q_scale"]),
                                   _ptr(r["k_i8"]), _ptr(r["k_scale"]), _ptr(r["vt_f16"]), _ptr(r["k_mean"]))
    r["n_q"], r["n_kv"] = Nq, N
    return r


def attn_fwd_i8(qz: dict, N: int, causal: bool, sm_scale: float | None = None, units=None,
                n_kv: int | None = None, return_lse: bool = False):
    """8-bit variant attention (readings I3-I5) on quantize_qkv_i8 operands;
    N query rows, n_kv keys (default qz["n_kv"] or N); bf16 bits [B,H,N,d].
    With return_lse, also the per-row log-sum-exp of the training forward
    (reading I6): (out, lse) with lse float32 [B,H,N]."""
    if n_kv is None:
        n_kv = qz.get("n_kv", N)
    B, H, _, d = qz["q_i8"].shape
    if sm_scale is None:
        sm_scale = 1.0 / float(np.sqrt(d))
    out = np.zeros((B, H, N, d), np.uint16)
    lse = np.full((B, H, N), np.nan, np.float32) if return_lse else None
    u, nu = _units_arr(units)
    arrs = [np.ascontiguousarray(qz[n]) for n in ("q_i8", "q_scale", "k_i8", "k_scale", "vt_f16")]
    _load().oracle_attn_fwd_i8(*[_ptr(a) for a in arrs], B, H, N, n_kv, d, int(bool(causal)), float(sm_scale),
                               _ptr(u), nu, _ptr(out), _ptr(lse))
    return (out, lse) if return_lse else out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float32 (exact)."""
    return (a.astype(np.uint32) << 16).view(np.float32)
