"""libsa3 Python binding: microscaled-FP4 attention forward on B200.

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels of ``libsa3.so`` (C ABI in ``include/sa3.h``); PyTorch provides the
device memory and the current stream.  There is no CPU fallback: if the
library is missing or a call fails, an exception is raised.

    qz = quantize_qkv(q, k, v)          # K smoothing + FP4 microscaling
    out = attn_fwd(qz, causal=False)    # FP4 attention, bf16 out
    out = sa3_attention(q, k, v)        # both in one call

    q8 = quantize_qkv_i8(q, k, v)       # 8-bit variant: INT8 Q, K; FP16 V^T
    out, lse = attn_fwd_i8(q8, causal=True, lse=True)   # training forward

q may be shorter or longer than k and v (the *_lens calls).  Every call is
asynchronous on the current torch stream (or ``stream=``); buffers can be
passed in (``out=``, ``workspace=``) so that a step allocates nothing and can
be recorded into a CUDA graph.  ``device_status()`` synchronizes and reports
whether a bounded device wait gave up.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa3.so")

SA3_OK = 0
SA3_ERR_INVALID_ARG = 1
SA3_ERR_UNSUPPORTED = 2
SA3_ERR_CUDA = 3
SA3_ERR_TIMEOUT = 4
SA3_P_TWO_LEVEL = 1
SA3_V_SMOOTH = 2
SA3_SKIP_Q = 4
SA3_Q_ON_LOAD = 8
_NAMES = {0: "SA3_OK", 1: "SA3_ERR_INVALID_ARG", 2: "SA3_ERR_UNSUPPORTED", 3: "SA3_ERR_CUDA",
          4: "SA3_ERR_TIMEOUT"}

BLK = 128


class Sa3Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {_NAMES.get(code, code)}")
        self.code = code


class _QKV(ctypes.Structure):
    _fields_ = [("q_fp4", ctypes.c_void_p), ("q_sf", ctypes.c_void_p),
                ("k_fp4", ctypes.c_void_p), ("k_sf", ctypes.c_void_p),
                ("vt_fp4", ctypes.c_void_p), ("vt_sf", ctypes.c_void_p),
                ("k_mean", ctypes.c_void_p)]


class _QKVI8(ctypes.Structure):
    _fields_ = [("q_i8", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("k_i8", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("vt_f16", ctypes.c_void_p), ("k_mean", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libsa3.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:  # loaded: no lock on the per-call path
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m bit_quantized_attention_sa3_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            L.sa3_version.restype = ctypes.c_char_p
            L.sa3_version.argtypes = []
            L.sa3_quantize_qkv.restype = I
            L.sa3_quantize_qkv.argtypes = [P, P, P, I, I, I, I, ctypes.POINTER(_QKV), P, ctypes.c_size_t, P]
            L.sa3_attn_fwd.restype = I
            L.sa3_attn_fwd.argtypes = [ctypes.POINTER(_QKV), I, I, I, I, I, F, P, P]
            L.sa3_quantize_qkv_lens.restype = I
            L.sa3_quantize_qkv_lens.argtypes = [P, P, P, I, I, I, I, I, ctypes.POINTER(_QKV), P, ctypes.c_size_t, P]
            L.sa3_attn_fwd_lens.restype = I
            L.sa3_attn_fwd_lens.argtypes = [ctypes.POINTER(_QKV), I, I, I, I, I, I, F, ctypes.c_uint, P, P]
            L.sa3_quantize_qkv_i8.restype = I
            L.sa3_quantize_qkv_i8.argtypes = [P, P, P, I, I, I, I, I, ctypes.POINTER(_QKVI8), P, ctypes.c_size_t, P]
            L.sa3_attn_fwd_i8.restype = I
            L.sa3_attn_fwd_i8.argtypes = [ctypes.POINTER(_QKVI8), I, I, I, I, I, I, F, P, P]
            L.sa3_attn_fwd_i8_lse.restype = I
            L.sa3_attn_fwd_i8_lse.argtypes = [ctypes.POINTER(_QKVI8), I, I, I, I, I, I, F, P, P, P]
            L.sa3_device_status.restype = I
            L.sa3_device_status.argtypes = [P]
            L.sa3_quantize_qkv_ex.restype = I
            L.sa3_quantize_qkv_ex.argtypes = [P, P, P, I, I, I, I, I, ctypes.c_uint, ctypes.POINTER(_QKV), P, P,
                                              ctypes.c_size_t, P]
            L.sa3_attn_fwd_ex.restype = I
            L.sa3_attn_fwd_ex.argtypes = [ctypes.POINTER(_QKV), P, P, I, I, I, I, I, I, F, ctypes.c_uint, P, P]
            L.sa3_probe_fp4_mma.restype = I
            L.sa3_probe_fp4_mma.argtypes = [I, I, I, P, P]
            _lib = L
    return _lib


def version() -> str:
    return lib().sa3_version().decode()


# ---------------------------------------------------------------- sizes
def padded_len(N: int) -> int:
    return (N + BLK - 1) // BLK * BLK


def kmean_chunk(N: int) -> int:
    return 512 * (((N + 511) // 512 + 15) // 16)


def quant_workspace_bytes(B: int, H: int, N: int, d: int, v_smooth: bool = False) -> int:
    """sa3_quant_workspace_bytes (sa3_quant_workspace_bytes_ex with
    SA3_V_SMOOTH when v_smooth) of include/sa3.h."""
    c = kmean_chunk(N)
    return B * H * ((N + c - 1) // c) * d * 8 * (2 if v_smooth else 1)


@dataclasses.dataclass
class QuantizedQKV:
    """Device buffers of the quantized operands (layouts: include/sa3.h).
    N is the key/value length; Nq the query length (None: equal to N).
    q_fp4 and q_sf are None when Q was left to the attention kernel
    (skip_q: it quantizes Q on load)."""
    q_fp4: torch.Tensor | None   # u8 [B,H,Np(Nq),d/2]
    q_sf: torch.Tensor | None    # u8, 128x4 scale atoms
    k_fp4: torch.Tensor   # u8 [B,H,Np,d/2]
    k_sf: torch.Tensor
    vt_fp4: torch.Tensor  # u8 [B,H,d,Np/2]
    vt_sf: torch.Tensor
    k_mean: torch.Tensor  # f32 [B,H,d]
    B: int
    H: int
    N: int
    d: int
    Nq: int | None = None
    v_mean: torch.Tensor | None = None  # f32 [B,H,d]: V smoothed (SA3_V_SMOOTH), else None

    @property
    def n_q(self) -> int:
        return self.N if self.Nq is None else self.Nq

    @property
    def device(self) -> torch.device:
        return self.k_fp4.device

    def check(self, device: torch.device | None = None) -> None:
        """Raise ValueError unless every buffer is a contiguous tensor of the
        dtype and byte size that include/sa3.h gives for (B, H, Nq, N, d), all
        on one device (``device``, if given).  The kernels trust these sizes."""
        dev = self.device if device is None else device
        Npq, Np = padded_len(self.n_q), padded_len(self.N)
        B, H, d = self.B, self.H, self.d
        if (self.q_fp4 is None) != (self.q_sf is None):
            raise ValueError("q_fp4 and q_sf must both be given or both be None")
        if self.q_fp4 is not None:
            _check_buffer(self.q_fp4, "q_fp4", torch.uint8, B * H * Npq * d // 2, dev)
            _check_buffer(self.q_sf, "q_sf", torch.uint8, B * H * Npq * d // 16, dev)
        _check_buffer(self.k_fp4, "k_fp4", torch.uint8, B * H * Np * d // 2, dev)
        _check_buffer(self.k_sf, "k_sf", torch.uint8, B * H * Np * d // 16, dev)
        _check_buffer(self.vt_fp4, "vt_fp4", torch.uint8, B * H * d * Np // 2, dev)
        _check_buffer(self.vt_sf, "vt_sf", torch.uint8, B * H * Np * 8, dev)
        _check_buffer(self.k_mean, "k_mean", torch.float32, B * H * d, dev)
        if self.v_mean is not None:
            _check_buffer(self.v_mean, "v_mean", torch.float32, B * H * d, dev)

    def struct(self) -> _QKV:
        qp = 0 if self.q_fp4 is None else self.q_fp4.data_ptr()
        qs = 0 if self.q_sf is None else self.q_sf.data_ptr()
        return _QKV(qp, qs, self.k_fp4.data_ptr(),
                    self.k_sf.data_ptr(), self.vt_fp4.data_ptr(), self.vt_sf.data_ptr(),
                    self.k_mean.data_ptr())


def empty_quantized(B: int, H: int, N: int, d: int, device="cuda", Nq: int | None = None,
                    v_smooth: bool = False, skip_q: bool = False) -> QuantizedQKV:
    """Buffers for keys/values of length N and queries of length Nq (default N);
    with v_smooth also the mean of V (V smoothing); with skip_q no Q buffers
    (Q quantized on load by the attention kernel)."""
    Np = padded_len(N)
    Npq = padded_len(N if Nq is None else Nq)
    u8 = dict(dtype=torch.uint8, device=device)
    return QuantizedQKV(
        q_fp4=None if skip_q else torch.empty((B, H, Npq, d // 2), **u8),
        q_sf=None if skip_q else torch.empty(B * H * Npq * d // 16, **u8),
        k_fp4=torch.empty((B, H, Np, d // 2), **u8), k_sf=torch.empty(B * H * Np * d // 16, **u8),
        vt_fp4=torch.empty((B, H, d, Np // 2), **u8), vt_sf=torch.empty(B * H * Np * 8, **u8),
        k_mean=torch.empty((B, H, d), dtype=torch.float32, device=device), B=B, H=H, N=N, d=d,
        Nq=None if Nq is None or Nq == N else Nq,
        v_mean=torch.empty((B, H, d), dtype=torch.float32, device=device) if v_smooth else None)


def _stream_ptr(stream, device: torch.device) -> int:
    """The cudaStream_t to enqueue on: ``stream``, else the current stream
    of ``device``.  A stream of another device is rejected."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the operands on {device}")
    return stream.cuda_stream


def _check_buffer(t: torch.Tensor, name: str, dtype: torch.dtype, numel: int, device: torch.device,
                  shape: tuple | None = None) -> None:
    """A caller's buffer must be contiguous, of ``dtype``, on ``device`` and
    hold exactly ``numel`` elements (and ``shape``, if given): the kernels
    write or read that many bytes through its pointer."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() != numel or (shape is not None and tuple(t.shape) != tuple(shape)):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected "
                         f"{tuple(shape) if shape is not None else f'{numel} elements'}")


def _check_input(t: torch.Tensor, name: str):
    if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
        raise ValueError(f"{name} must be a contiguous 4-D bf16 CUDA tensor [B,H,N,d]")


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.device:
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_input(t, n)
    if not (k.shape == v.shape and q.shape[:2] == k.shape[:2] and q.shape[3] == k.shape[3]):
        raise ValueError("q must be [B,H,Nq,d] and k, v [B,H,N,d]")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k and v must be on one device")
    return q.device


def _check_workspace(ws: torch.Tensor, nbytes: int, device: torch.device) -> int:
    """Byte size of a caller's workspace (any dtype, contiguous, on device)."""
    if ws.device != device or not ws.is_contiguous():
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    size = ws.numel() * ws.element_size()
    if size < nbytes:
        raise ValueError(f"workspace holds {size} bytes, needs {nbytes}")
    return size


def _check_out(out: torch.Tensor, shape: tuple, device: torch.device) -> None:
    _check_buffer(out, "out", torch.bfloat16, math.prod(shape), device, shape)


def quantize_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 out: QuantizedQKV | None = None, workspace: torch.Tensor | None = None,
                 stream=None, v_smooth: bool = False, skip_q: bool = False) -> QuantizedQKV:
    """sa3_quantize_qkv: K smoothing, then E2M1 codes + E4M3 scales of Q, K, V.
    q is [B,H,Nq,d]; k and v are [B,H,N,d] (N may differ from Nq:
    sa3_quantize_qkv_lens).  v_smooth: V is smoothed like K and its mean
    kept in the result (sa3_quantize_qkv_ex with SA3_V_SMOOTH); attn_fwd
    then adds it back.  skip_q: Q is not quantized here (SA3_SKIP_Q); pass
    q to attn_fwd, which quantizes it on load."""
    dev = _check_qkv(q, k, v)
    B, H, Nq, d = q.shape
    N = k.shape[2]
    with torch.cuda.device(dev):
        if out is None:
            out = empty_quantized(B, H, N, d, dev, Nq=Nq, v_smooth=v_smooth, skip_q=skip_q)
        if (out.B, out.H, out.d, out.n_q, out.N) != (B, H, d, Nq, N):
            raise ValueError("out was sized for another shape")
        if v_smooth != (out.v_mean is not None):
            raise ValueError("out must hold v_mean exactly when v_smooth is set")
        if not skip_q and out.q_fp4 is None:
            raise ValueError("out has no Q buffers: quantize with skip_q=True")
        out.check(dev)
        nbytes = quant_workspace_bytes(B, H, N, d, v_smooth)
        if workspace is None:
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        ws_bytes = _check_workspace(workspace, nbytes, dev)
        sp = _stream_ptr(stream, dev)
        st = out.struct()
        if v_smooth or skip_q:
            flags = (SA3_V_SMOOTH if v_smooth else 0) | (SA3_SKIP_Q if skip_q else 0)
            rc = lib().sa3_quantize_qkv_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, Nq, N, d, flags,
                                           ctypes.byref(st), out.v_mean.data_ptr() if v_smooth else None,
                                           workspace.data_ptr(), ws_bytes, sp)
        elif Nq == N:
            rc = lib().sa3_quantize_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, N, d, ctypes.byref(st),
                                        workspace.data_ptr(), ws_bytes, sp)
        else:
            rc = lib().sa3_quantize_qkv_lens(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, Nq, N, d,
                                             ctypes.byref(st), workspace.data_ptr(), ws_bytes, sp)
    if rc != SA3_OK:
        raise Sa3Error(rc, "sa3_quantize_qkv")
    return out


def attn_fwd(qz: QuantizedQKV, causal: bool = False, sm_scale: float | None = None,
             out: torch.Tensor | None = None, stream=None, p_two_level: bool = False,
             q: torch.Tensor | None = None) -> torch.Tensor:
    """sa3_attn_fwd: FP4 attention of quantized operands; bf16 [B,H,Nq,d].
    With Nq != N (sa3_attn_fwd_lens) the causal mask aligns the last query
    with the last key; a row that sees no key is 0.  p_two_level: P scaled
    by 2^11 before it is microscaled (SA3_P_TWO_LEVEL).  Operands quantized
    with v_smooth carry V's mean, which is added back (sa3_attn_fwd_ex with
    SA3_V_SMOOTH).  q (bf16 [B,H,Nq,d]): the kernel quantizes Q on load
    (SA3_Q_ON_LOAD) instead of reading qz's Q codes; required when qz was
    made with skip_q."""
    B, H, N, d, Nq = qz.B, qz.H, qz.N, qz.d, qz.n_q
    dev = qz.device
    if dev.type != "cuda":
        raise ValueError("the quantized operands must be CUDA tensors")
    qz.check(dev)
    if q is not None:
        _check_input(q, "q")
        if tuple(q.shape) != (B, H, Nq, d) or q.device != dev:
            raise ValueError("q must be bf16 [B,H,Nq,d] on the operands' device")
    elif qz.q_fp4 is None:
        raise ValueError("qz holds no Q codes (skip_q): pass q to quantize it on load")
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=dev)
        _check_out(out, (B, H, Nq, d), dev)
        # sm_scale 0 asks the library for its default, 1/sqrt(d)
        scale = 0.0 if sm_scale is None else float(sm_scale)
        sp = _stream_ptr(stream, dev)
        st = qz.struct()
        if qz.v_mean is not None or q is not None:
            flags = ((SA3_V_SMOOTH if qz.v_mean is not None else 0) | (SA3_P_TWO_LEVEL if p_two_level else 0)
                     | (SA3_Q_ON_LOAD if q is not None else 0))
            rc = lib().sa3_attn_fwd_ex(ctypes.byref(st), q.data_ptr() if q is not None else None,
                                       qz.v_mean.data_ptr() if qz.v_mean is not None else None, B, H, Nq, N, d,
                                       int(bool(causal)), scale, flags, out.data_ptr(), sp)
        elif Nq == N and not p_two_level:
            rc = lib().sa3_attn_fwd(ctypes.byref(st), B, H, N, d, int(bool(causal)), scale, out.data_ptr(), sp)
        else:
            flags = SA3_P_TWO_LEVEL if p_two_level else 0
            rc = lib().sa3_attn_fwd_lens(ctypes.byref(st), B, H, Nq, N, d, int(bool(causal)), scale,
                                         flags, out.data_ptr(), sp)
    if rc != SA3_OK:
        raise Sa3Error(rc, "sa3_attn_fwd")
    return out


# ------------------------------------------------------- 8-bit variant
@dataclasses.dataclass
class QuantizedQKVI8:
    """Operands of the 8-bit variant (layouts: include/sa3.h): INT8 Q and
    smoothed K with one fp32 scale per 128-token tile, FP16 V^T."""
    q_i8: torch.Tensor     # int8 [B,H,Np(Nq),d]
    q_scale: torch.Tensor  # f32 [B,H,Np(Nq)/128]
    k_i8: torch.Tensor     # int8 [B,H,Np(N),d]
    k_scale: torch.Tensor  # f32 [B,H,Np(N)/128]
    vt_f16: torch.Tensor   # f16 [B,H,d,Np(N)]
    k_mean: torch.Tensor   # f32 [B,H,d]
    B: int
    H: int
    N: int
    d: int
    Nq: int

    @property
    def device(self) -> torch.device:
        return self.q_i8.device

    def check(self, device: torch.device | None = None) -> None:
        """As QuantizedQKV.check, for the 8-bit operands."""
        dev = self.device if device is None else device
        Npq, Np = padded_len(self.Nq), padded_len(self.N)
        B, H, d = self.B, self.H, self.d
        _check_buffer(self.q_i8, "q_i8", torch.int8, B * H * Npq * d, dev)
        _check_buffer(self.q_scale, "q_scale", torch.float32, B * H * (Npq // BLK), dev)
        _check_buffer(self.k_i8, "k_i8", torch.int8, B * H * Np * d, dev)
        _check_buffer(self.k_scale, "k_scale", torch.float32, B * H * (Np // BLK), dev)
        _check_buffer(self.vt_f16, "vt_f16", torch.float16, B * H * d * Np, dev)
        _check_buffer(self.k_mean, "k_mean", torch.float32, B * H * d, dev)

    def struct(self) -> _QKVI8:
        return _QKVI8(self.q_i8.data_ptr(), self.q_scale.data_ptr(), self.k_i8.data_ptr(), self.k_scale.data_ptr(),
                      self.vt_f16.data_ptr(), self.k_mean.data_ptr())


def empty_quantized_i8(B: int, H: int, N: int, d: int, device="cuda", Nq: int | None = None) -> QuantizedQKVI8:
    Nq = N if Nq is None else Nq
    Npq, Np = padded_len(Nq), padded_len(N)
    f32 = dict(dtype=torch.float32, device=device)
    return QuantizedQKVI8(
        q_i8=torch.empty((B, H, Npq, d), dtype=torch.int8, device=device), q_scale=torch.empty((B, H, Npq // BLK), **f32),
        k_i8=torch.empty((B, H, Np, d), dtype=torch.int8, device=device), k_scale=torch.empty((B, H, Np // BLK), **f32),
        vt_f16=torch.empty((B, H, d, Np), dtype=torch.float16, device=device), k_mean=torch.empty((B, H, d), **f32),
        B=B, H=H, N=N, d=d, Nq=Nq)


def quantize_qkv_i8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: QuantizedQKVI8 | None = None,
                    workspace: torch.Tensor | None = None, stream=None) -> QuantizedQKVI8:
    """sa3_quantize_qkv_i8: K smoothing, INT8 Q and K per 128-token tile, FP16 V^T."""
    dev = _check_qkv(q, k, v)
    B, H, Nq, d = q.shape
    N = k.shape[2]
    with torch.cuda.device(dev):
        if out is None:
            out = empty_quantized_i8(B, H, N, d, dev, Nq=Nq)
        if (out.B, out.H, out.d, out.Nq, out.N) != (B, H, d, Nq, N):
            raise ValueError("out was sized for another shape")
        out.check(dev)
        nbytes = quant_workspace_bytes(B, H, N, d)
        if workspace is None:
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        ws_bytes = _check_workspace(workspace, nbytes, dev)
        sp = _stream_ptr(stream, dev)
        st = out.struct()
        rc = lib().sa3_quantize_qkv_i8(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, Nq, N, d, ctypes.byref(st),
                                       workspace.data_ptr(), ws_bytes, sp)
    if rc != SA3_OK:
        raise Sa3Error(rc, "sa3_quantize_qkv_i8")
    return out


def attn_fwd_i8(qz: QuantizedQKVI8, causal: bool = False, sm_scale: float | None = None,
                out: torch.Tensor | None = None, stream=None, lse: torch.Tensor | bool | None = None):
    """sa3_attn_fwd_i8: 8-bit attention (INT8 QK^T, FP16 P V); bf16 [B,H,Nq,d].

    With ``lse`` (True, or a float32 [B,H,Nq] tensor to fill) this is the
    training forward, sa3_attn_fwd_i8_lse: it also writes each row's
    log-sum-exp and returns ``(out, lse)``."""
    B, H, N, d, Nq = qz.B, qz.H, qz.N, qz.d, qz.Nq
    dev = qz.device
    if dev.type != "cuda":
        raise ValueError("the quantized operands must be CUDA tensors")
    qz.check(dev)
    scale = 0.0 if sm_scale is None else float(sm_scale)  # 0: the library's default 1/sqrt(d)
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=dev)
        _check_out(out, (B, H, Nq, d), dev)
        sp = _stream_ptr(stream, dev)
        st = qz.struct()
        if lse is None or lse is False:
            rc = lib().sa3_attn_fwd_i8(ctypes.byref(st), B, H, Nq, N, d, int(bool(causal)), scale,
                                       out.data_ptr(), sp)
            if rc != SA3_OK:
                raise Sa3Error(rc, "sa3_attn_fwd_i8")
            return out
        if lse is True:
            lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
        _check_buffer(lse, "lse", torch.float32, B * H * Nq, dev)
        rc = lib().sa3_attn_fwd_i8_lse(ctypes.byref(st), B, H, Nq, N, d, int(bool(causal)), scale,
                                       out.data_ptr(), lse.data_ptr(), sp)
    if rc != SA3_OK:
        raise Sa3Error(rc, "sa3_attn_fwd_i8_lse")
    return out, lse


def device_status(stream=None, device=None) -> int:
    """Synchronizes the stream (default: the current stream of ``device``,
    default the current device); SA3_ERR_TIMEOUT if a bounded wait gave up."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if stream is not None:
        dev = stream.device
    with torch.cuda.device(dev):
        return lib().sa3_device_status(_stream_ptr(stream, dev))


def probe_fp4_mma(n: int = 128, iters: int = 4096, ctas: int | None = None, out: torch.Tensor | None = None,
                  stream=None, device=None) -> torch.Tensor:
    """sa3_probe_fp4_mma: enqueue the block-scaled FP4 MMA rate probe (M=128,
    N=n, K=64, ``iters`` MMAs per CTA, one CTA per SM by default) and return
    its check values, fp32 [2*ctas], each 64*iters once it has run.  Time it
    with CUDA events around this call: 2*128*n*64 * iters * ctas operations."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        if ctas is None:
            ctas = torch.cuda.get_device_properties(dev).multi_processor_count
        if out is None:
            out = torch.empty(2 * ctas, dtype=torch.float32, device=dev)
        _check_buffer(out, "out", torch.float32, 2 * ctas, dev)
        rc = lib().sa3_probe_fp4_mma(ctas, n, iters, out.data_ptr(), _stream_ptr(stream, dev))
    if rc != SA3_OK:
        raise Sa3Error(rc, "sa3_probe_fp4_mma")
    return out


def sa3_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                  sm_scale: float | None = None, v_smooth: bool = False) -> torch.Tensor:
    """Plug-in attention: quantize then attend; bf16 [B,H,N,d] in and out."""
    return attn_fwd(quantize_qkv(q, k, v, v_smooth=v_smooth), causal=causal, sm_scale=sm_scale)
