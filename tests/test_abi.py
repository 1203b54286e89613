"""The C-ABI library loads, exports every symbol include/dq.h declares, and
rejects invalid arguments before touching the GPU (CPU only)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "dq.h")


def declared_functions():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"DQ_API\s+[\w\s\*]+?\b(dq_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def L():
    from w4a4_post_quantization_dual_b200 import build, dq
    build.build()
    return dq.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(os.path.join(ROOT, "w4a4_post_quantization_dual_b200", "lib", "libdq.so"))
    for n in names:
        assert hasattr(lib, n), n
    from w4a4_post_quantization_dual_b200 import dq
    assert set(names) == set(dq.SIGNATURES), "binding and header disagree"


def test_status_strings_and_groups(L):
    for s in range(6):
        assert L.dq_status_string(s)
    assert [L.dq_native_group(f) for f in range(4)] == [64, 32, 32, 16]
    assert L.dq_version() >= 100


def test_scales_bytes_matches_layout_definition(L, orc):
    for rows, k, f, G in [(1, 4096, 3, 16), (300, 5120, 3, 16), (4096, 14336, 2, 32),
                          (129, 256, 1, 32)]:
        assert L.dq_scales_bytes(rows, k, f, G) == orc.sf_bytes(rows, k // G)
    assert L.dq_scales_bytes(10, 256, 0, 128) == 10 * 2 * 2
    assert L.dq_scales_bytes(10, 250, 3, 16) == 0  # k % G != 0
    assert L.dq_scales_bytes(10, 256, 3, 32) == 0  # NVFP4 block must be 16


def test_invalid_arguments_rejected_without_launch(L):
    from w4a4_post_quantization_dual_b200.dq import SIGNATURES  # noqa: F401
    fake = ctypes.c_void_p(0x1000)   # never dereferenced: validation fails first
    ws = ctypes.c_void_p(0x2000)
    # null W
    assert L.dq_solve_scales(None, 1, 64, 64, 3, 16, 5, fake, fake, fake, None, ws, 4096, None) == 1
    # n not a multiple of G
    assert L.dq_solve_scales(fake, 1, 64, 40, 3, 16, 5, fake, fake, fake, None, ws, 4096, None) == 1
    # workspace too small
    assert L.dq_solve_scales(fake, 1, 64, 64, 3, 16, 5, fake, fake, fake, None, ws, 8, None) == 5
    # ablation flags: both arms at once, or an unknown bit; misaligned r0
    for flags in (3, 8, 1 | 16):
        assert L.dq_solve_scales_ex(fake, 1, 64, 64, 3, 16, 5, flags, None, None, fake, fake,
                                    fake, None, ws, 4096, None) == 1
    assert L.dq_solve_scales_ex(fake, 1, 64, 64, 3, 16, 5, 0, ctypes.c_void_p(0x1002), None,
                                fake, fake, fake, None, ws, 4096, None) == 1
    assert L.dq_solve_scales_ex(fake, 1, 64, 64, 3, 16, 5, 4, None, None, fake, fake, fake, None,
                                ws, 8, None) == 5
    # batched solver: empty batch, n % G, unknown flag, workspace too small
    arr = lambda *v: (ctypes.c_void_p * len(v))(*v)
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)
    two = arr(0x1000, 0x2000)
    assert L.dq_solve_batched_workspace_size(2, 5) == 2 * L.dq_solve_workspace_size(5)
    assert L.dq_solve_scales_batched(0, two, 1, i64(64, 64), i64(64, 64), 3, 16, 5, 0, two, two,
                                     two, None, ws, 4096, None) == 1
    assert L.dq_solve_scales_batched(2, two, 1, i64(64, 64), i64(64, 40), 3, 16, 5, 0, two, two,
                                     two, None, ws, 4096, None) == 1
    assert L.dq_solve_scales_batched(2, two, 1, i64(64, 64), i64(64, 64), 3, 16, 5, 8, two, two,
                                     two, None, ws, 4096, None) == 1
    assert L.dq_solve_scales_batched(2, two, 1, i64(64, 64), i64(64, 64), 3, 16, 5, 0, two, two,
                                     two, None, ws, 100, None) == 5
    # 8-bit formats: INT8 has no tensor-core linear; MXFP8 follows the MX shape rules
    assert L.dq_w4a4_linear(fake, fake, fake, fake, fake, fake, None, fake, 1, 16, 128, 256,
                            4, None) == 2
    assert L.dq_w4a4_linear(fake, fake, None, fake, fake, None, None, fake, 1, 16, 100, 256,
                            6, None) == 1
    assert L.dq_scales_bytes(10, 256, 4, 128) == 10 * 2 * 2          # INT8: bf16 row-major
    assert L.dq_scales_bytes(130, 256, 6, 32) == 2 * 2 * 512          # MXFP8: padded atoms
    assert [L.dq_native_group(f) for f in (4, 5, 6)] == [128, 32, 32]
    # more column blocks than one launch grid holds: refused before anything is enqueued
    wide = 16 * 65536
    assert L.dq_solve_scales(fake, 1, 64, wide, 3, 16, 5, fake, fake, fake, None, ws, 4096,
                             None) == 2
    assert L.dq_solve_scales_batched(2, two, 1, i64(64, 64), i64(64, wide), 3, 16, 5, 0, two, two,
                                     two, None, ws, 4096, None) == 2
    # bad group for the format
    assert L.dq_quantize_weight(fake, 1, 64, 64, 2, 16, fake, fake, fake, fake, fake, None) == 1
    # NVFP4 weight packing needs the tensor scale pointer
    assert L.dq_quantize_weight(fake, 1, 64, 64, 3, 16, fake, fake, None, fake, fake, None) == 1
    # NVFP4 activations need s_tok; K must be a multiple of 4*G for the MMA layout
    assert L.dq_quantize_act(fake, 1, 4, 64, None, 3, 16, fake, fake, None, None) == 1
    assert L.dq_quantize_act(fake, 1, 4, 48, None, 3, 16, fake, fake, fake, None) == 1
    # GEMM: INT4 (bf16 group scales) has no block-scaled tensor-core form on sm_100a
    assert L.dq_w4a4_linear(fake, fake, fake, fake, fake, fake, None, fake, 1, 16, 128, 256,
                            0, None) == 2
    # GEMM shape rules: N % 128, K % 256, 16-byte alignment
    assert L.dq_w4a4_linear(fake, fake, fake, fake, fake, fake, None, fake, 1, 16, 100, 256,
                            3, None) == 1
    assert L.dq_w4a4_linear(fake, fake, fake, fake, fake, fake, None, fake, 1, 16, 128, 128,
                            3, None) == 1
    # N must stay below 2^31 (the kernels index output columns with 32-bit ints)
    assert L.dq_w4a4_linear(fake, fake, fake, fake, fake, fake, None, fake, 1, 16, 1 << 31, 256,
                            3, None) == 1
    assert L.dq_w4a4_linear_fused(fake, 1, None, fake, fake, fake, None, fake, 1, 16, 1 << 31,
                                  256, 3, None) == 1
    odd = ctypes.c_void_p(0x1001)
    assert L.dq_w4a4_linear(odd, fake, fake, fake, fake, fake, None, fake, 1, 16, 128, 256,
                            3, None) == 1


def test_header_is_plain_c_and_links(L, tmp_path):
    """include/dq.h compiles as strict C99 and a C program linked against
    libdq.so gets the documented results from calls that need no GPU."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.join(ROOT, "w4a4_post_quantization_dual_b200", "lib")
    exe = str(tmp_path / "c_abi_check")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe,
                    "-L", libdir, "-ldq", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert "c abi ok" in out.stdout
