"""The C ABI without a GPU: libsa3.so loads, exports every function that
include/sa3.h declares, returns its version, and rejects bad arguments
before touching the device."""
import ctypes
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sa3.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int|char|void)\s*\*?\s*(sa3_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from bit_quantized_attention_sa3_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_boundary():
    assert _declared() == ["sa3_attn_fwd", "sa3_attn_fwd_ex", "sa3_attn_fwd_i8", "sa3_attn_fwd_i8_lse",
                           "sa3_attn_fwd_lens", "sa3_device_status", "sa3_probe_fp4_mma", "sa3_quantize_qkv",
                           "sa3_quantize_qkv_ex", "sa3_quantize_qkv_i8", "sa3_quantize_qkv_lens",
                           "sa3_quantize_qkv_noalloc", "sa3_selftest_wait_timeout", "sa3_version"]


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


@pytest.mark.skipif(shutil.which("nm") is None, reason="needs binutils nm")
def test_library_exports_only_the_declared_symbols(lib):
    """The kernels, their launchers and the host helpers' caches stay inside
    the library: a second build loaded into the same process (or another
    library with the same template instances) must not bind to them."""
    from bit_quantized_attention_sa3_b200 import build
    r = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True, check=True)
    syms = [ln.split() for ln in r.stdout.splitlines() if len(ln.split()) == 3]
    assert sorted(name for _, kind, name in syms if kind in "TtWwVvuBDR") == _declared()
    assert not [name for _, kind, name in syms if kind == "u"], "process-wide unique symbols"


def test_version(lib):
    lib.sa3_version.restype = ctypes.c_char_p
    assert lib.sa3_version().decode().startswith("libsa3")


def test_argument_checks_need_no_gpu(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.sa3_quantize_qkv.restype = I
    lib.sa3_quantize_qkv.argtypes = [P, P, P, I, I, I, I, P, P, ctypes.c_size_t, P]
    lib.sa3_attn_fwd.restype = I
    lib.sa3_attn_fwd.argtypes = [P, I, I, I, I, I, ctypes.c_float, P, P]
    # d unsupported
    assert lib.sa3_quantize_qkv(16, 16, 16, 1, 1, 8, 96, None, None, 0, None) == 2
    # null pointers / bad sizes
    assert lib.sa3_quantize_qkv(None, None, None, 1, 1, 8, 64, None, None, 0, None) == 1
    assert lib.sa3_quantize_qkv(16, 16, 16, 0, 1, 8, 64, None, None, 0, None) == 1
    assert lib.sa3_attn_fwd(None, 1, 1, 8, 64, 0, 0.0, None, None) == 1
    assert lib.sa3_attn_fwd(None, 1, 1, 8, 100, 0, 0.0, None, None) == 2
    # B*H is limited only through B*H*N_p*d/2 < 2^31 (grids are 1-D):
    # 100000 heads of 8 tokens pass the shape check (then fail on null)
    assert lib.sa3_attn_fwd(None, 1000, 100, 8, 64, 0, 0.0, None, None) == 1
    assert lib.sa3_attn_fwd(None, 1 << 16, 1 << 9, 8, 64, 0, 0.0, None, None) == 2
    lib.sa3_selftest_wait_timeout.restype = I
    lib.sa3_selftest_wait_timeout.argtypes = [ctypes.c_uint, P]
    assert lib.sa3_selftest_wait_timeout(0, None) == 1
    lib.sa3_probe_fp4_mma.restype = I
    lib.sa3_probe_fp4_mma.argtypes = [I, I, I, P, P]
    assert lib.sa3_probe_fp4_mma(148, 192, 16, 16, None) == 1     # n must be 128 or 256
    assert lib.sa3_probe_fp4_mma(148, 128, 0, 16, None) == 1      # iters >= 1
    assert lib.sa3_probe_fp4_mma(148, 128, 1 << 19, 16, None) == 1
    assert lib.sa3_probe_fp4_mma(148, 128, 16, None, None) == 1
    # separate query / key lengths: each is checked
    lib.sa3_quantize_qkv_lens.restype = I
    lib.sa3_quantize_qkv_lens.argtypes = [P, P, P, I, I, I, I, I, P, P, ctypes.c_size_t, P]
    lib.sa3_attn_fwd_lens.restype = I
    lib.sa3_attn_fwd_lens.argtypes = [P, I, I, I, I, I, I, ctypes.c_float, ctypes.c_uint, P, P]
    assert lib.sa3_quantize_qkv_lens(16, 16, 16, 1, 1, 8, 0, 64, None, None, 0, None) == 1
    assert lib.sa3_quantize_qkv_lens(16, 16, 16, 1, 1, 0, 8, 64, None, None, 0, None) == 1
    assert lib.sa3_quantize_qkv_lens(16, 16, 16, 1, 1, 8, 8, 96, None, None, 0, None) == 2
    assert lib.sa3_attn_fwd_lens(None, 1, 1, 8, 0, 64, 0, 0.0, 0, None, None) == 1
    assert lib.sa3_attn_fwd_lens(None, 1, 1, 8, 8, 64, 0, 0.0, 0, None, None) == 1
    # size limit B*H*N_p*d/2 < 2^31: exactly at it -> unsupported; one tile
    # below passes the shape check and fails on the null pointers instead
    at = 1 << 25  # N_p * 128 / 2 = 2^31 with B = H = 1, d = 128
    assert lib.sa3_quantize_qkv(16, 16, 16, 1, 1, at, 128, None, None, 0, None) == 2
    assert lib.sa3_attn_fwd(None, 1, 1, at, 128, 0, 0.0, None, None) == 2
    assert lib.sa3_attn_fwd(None, 1, 1, at - 128, 128, 0, 0.0, None, None) == 1
    assert lib.sa3_attn_fwd_lens(None, 1, 1, 8, at, 128, 0, 0.0, 0, None, None) == 2


def test_outputs_that_alias_inputs_are_rejected_without_a_gpu(lib):
    """The aliasing checks run on addresses alone, before any launch: an
    attention output overlapping the Q it quantizes on load, or one of the
    quantized operands, and an 8-bit output overlapping its log-sum-exp."""
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.sa3_attn_fwd_ex.restype = I
    lib.sa3_attn_fwd_ex.argtypes = [P, P, P, I, I, I, I, I, I, F, ctypes.c_uint, P, P]
    lib.sa3_attn_fwd_i8_lse.restype = I
    lib.sa3_attn_fwd_i8_lse.argtypes = [P, I, I, I, I, I, I, F, P, P, P]
    B, H, N, d = 1, 2, 256, 64
    mb = 1 << 20
    # seven buffers 1 MiB apart (fake, 16-byte aligned addresses; never touched)
    bufs = [(i + 1) * mb for i in range(7)]

    class QKV(ctypes.Structure):
        _fields_ = [(n, ctypes.c_void_p) for n in ("q_fp4", "q_sf", "k_fp4", "k_sf", "vt_fp4", "vt_sf", "k_mean")]

    st = QKV(*bufs)
    q = 16 * mb
    q_on_load = 8
    # in place: out = q
    assert lib.sa3_attn_fwd_ex(ctypes.byref(st), q, None, B, H, N, N, d, 0, 0.0, q_on_load, q, None) == 1
    # out reaching into q's last bytes
    assert lib.sa3_attn_fwd_ex(ctypes.byref(st), q, None, B, H, N, N, d, 0, 0.0, q_on_load, q - 16, None) == 1
    # out over the K codes (two-pass path)
    assert lib.sa3_attn_fwd_ex(ctypes.byref(st), None, None, B, H, N, N, d, 0, 0.0, 0, bufs[2] + 64, None) == 1

    class QKV8(ctypes.Structure):
        _fields_ = [(n, ctypes.c_void_p) for n in ("q_i8", "q_scale", "k_i8", "k_scale", "vt_f16", "k_mean")]

    st8 = QKV8(*bufs[:6])
    out = 16 * mb
    assert lib.sa3_attn_fwd_i8_lse(ctypes.byref(st8), B, H, N, N, d, 0, 0.0, out, out + 64, None) == 1
    assert lib.sa3_attn_fwd_i8_lse(ctypes.byref(st8), B, H, N, N, d, 0, 0.0, bufs[4], None, None) == 1


def test_binding_loads_the_library_and_reports_its_version():
    """The Python binding's own loader (no GPU needed to load or to ask the
    version) sets every declared signature."""
    import bit_quantized_attention_sa3_b200 as sa3
    from bit_quantized_attention_sa3_b200 import build
    build.build()
    assert sa3.version().startswith("libsa3")
    L = sa3.lib()
    assert sa3.lib() is L
    for name in _declared():
        if name not in ("sa3_selftest_wait_timeout", "sa3_quantize_qkv_noalloc", "sa3_version"):
            assert getattr(L, name).argtypes, name  # ctypes leaves argtypes None unless set


def test_binding_sizes_match_the_header(tmp_path):
    """The binding's size helpers restate the header's inline functions:
    compile the header's own into a host program and compare."""
    import shutil

    sa3 = pytest.importorskip("bit_quantized_attention_sa3_b200")
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("needs a C compiler")
    shapes = [(1, 1, 1, 64), (2, 16, 4096, 128), (1, 30, 17776, 64), (4, 32, 8192, 128), (1, 256, 8192, 128),
              (1, 32, 32768, 128), (3, 7, 1000, 64)]
    src = tmp_path / "sizes.c"
    lines = ['#include "sa3.h"', "#include <stdio.h>", "int main(void) {"]
    for B, H, N, d in shapes:
        lines.append(f'  printf("%lld %lld %lld %lld\\n", (long long)sa3_padded_len({N}), '
                     f"(long long)sa3_kmean_chunk({N}), (long long)sa3_quant_workspace_bytes({B}, {H}, {N}, {d}), "
                     f"(long long)sa3_quant_workspace_bytes_ex({B}, {H}, {N}, {d}, SA3_V_SMOOTH));")
    lines.append('  printf("%u\\n", (unsigned)SA3_NOALLOC_SCRATCH_BYTES);')
    lines.append("  return 0;\n}")
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "sizes"
    r = subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    for (B, H, N, d), line in zip(shapes, out):
        got = [int(x) for x in line.split()]
        want = [sa3.padded_len(N), sa3.kmean_chunk(N), sa3.quant_workspace_bytes(B, H, N, d),
                sa3.quant_workspace_bytes(B, H, N, d, v_smooth=True)]
        assert got == want, (B, H, N, d)
    # the no-alloc scratch holds exactly 256 heads of 8192 tokens at d = 128
    assert int(out[len(shapes)]) == sa3.quant_workspace_bytes(1, 256, 8192, 128)
