"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "libattn.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as ea
    return ea.lib()


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for n in ("attn_fwd", "attn_fwd_masked", "attn_bwd", "attn_bwd_workspace_bytes", "attn_status",
              "attn_bwd_deterministic", "attn_bwd_deterministic_workspace_bytes", "attn_bwd_noalloc",
              "attn_strerror", "attn_fwd_varlen", "attn_bwd_varlen", "attn_fwd_blocksparse",
              "attn_bwd_blocksparse", "attn_fwd_fp8", "attn_fwd_fp8_masked", "attn_fwd_fp8_varlen",
              "attn_fwd_fp8_blocksparse"):
        assert n in names


@pytest.mark.parametrize("name", ["libattn.so", "libattn_debug.so"])
def test_every_declared_symbol_is_exported(L, name):
    path = os.path.join(ROOT, "exact_attention_123_b200", name)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    handle = ctypes.CDLL(path)
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(handle, n)
    # nothing else of ours leaks out of the library
    ours = {e for e in exported if e.startswith("attn")}
    assert ours == set(declared_functions())


def test_release_and_debug_libraries_identify_themselves(L):
    import exact_attention_123_b200 as ea
    lib_dir = os.path.join(ROOT, "exact_attention_123_b200")
    assert ctypes.CDLL(os.path.join(lib_dir, "libattn.so")).attn_debug_checks() == 0
    assert ctypes.CDLL(os.path.join(lib_dir, "libattn_debug.so")).attn_debug_checks() == 1
    prev = ea.use_debug_library(True)
    try:
        assert ea.attn_debug_checks()
        assert ea.attn_debug_corrupt_tag(5) == -1 and ea.attn_debug_corrupt_tag(-1) == 5  # host-side hook only
    finally:
        ea.use_debug_library(prev)
    assert not ea.attn_debug_checks()


def test_header_compiles_as_c(tmp_path):
    c = tmp_path / "t.c"
    c.write_text('#include "libattn.h"\nint main(void){return ATTN_OK;}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-c", str(c),
                    "-o", str(tmp_path / "t.o")], check=True)


def test_strerror_and_workspace_sizes(L):
    import exact_attention_123_b200 as ea
    for code in range(0, 8):
        assert isinstance(ea.attn_strerror(code), str) and ea.attn_strerror(code)
    # two fp32 terms (D and lse*log2 e) per query row and head
    assert ea.attn_bwd_workspace_bytes(2, 16, 4096, 128) >= 2 * (2 * 16 * 4096 * 4)
    assert ea.attn_bwd_workspace_bytes(1, 1, 1, 96) == 0
    assert ea.attn_bwd_workspace_bytes(0, 1, 1, 64) == 0
    assert ea.attn_bwd_varlen_workspace_bytes(1000, 4, 64) >= 2 * (1000 * 4 * 4)
    # the deterministic backward needs only the two per-row terms, and never more than attn_bwd
    assert ea.attn_bwd_deterministic_workspace_bytes(2, 16, 4096, 128) == 2 * (2 * 16 * 4096 * 4)
    assert ea.attn_bwd_deterministic_workspace_bytes(2, 16, 4096, 128) <= ea.attn_bwd_workspace_bytes(2, 16, 4096, 128)
    assert ea.attn_bwd_deterministic_workspace_bytes(1, 1, 1, 96) == 0


def test_noalloc_size_limit_is_exact(L):
    # ATTN_NOALLOC_SCRATCH_BYTES = 8 MiB holds the two fp32 terms of exactly 1,048,576
    # query rows x heads; one more row is refused on the host, before any device work
    # (so the fake pointers are never read and no GPU is needed).
    import exact_attention_123_b200 as ea
    limit = 8 << 20
    assert ea.attn_bwd_deterministic_workspace_bytes(1, 1, 1048576, 128) <= limit
    assert ea.attn_bwd_deterministic_workspace_bytes(1, 1, 1048577, 128) > limit
    assert ea.attn_bwd_deterministic_workspace_bytes(1, 1, 1048577, 64) > limit
    vp = ctypes.c_void_p
    for shape in ((1, 1, 1048577, 128), (2, 1, 524289, 64)):
        rc = L.attn_bwd_noalloc(*[vp(FAKE)] * 9, *shape, ctypes.c_float(0.088), 1, None, None, None)
        assert rc == ea.ATTN_ERR_WORKSPACE, shape


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case below fails host validation first


def fwd(L, ptrs, B=1, H=1, N=16, d=64, scale=0.125):
    vp = [ctypes.c_void_p(p) if p else None for p in ptrs]
    return L.attn_fwd(*vp, B, H, N, d, ctypes.c_float(scale), 1, None, None)


def test_host_argument_errors(L):
    import exact_attention_123_b200 as ea
    good = [FAKE] * 5
    assert fwd(L, [0, FAKE, FAKE, FAKE, FAKE]) == ea.ATTN_ERR_INVALID_ARG
    assert fwd(L, good, B=0) == ea.ATTN_ERR_INVALID_ARG
    assert fwd(L, good, N=-3) == ea.ATTN_ERR_INVALID_ARG
    assert fwd(L, good, scale=0.0) == ea.ATTN_ERR_INVALID_ARG
    assert fwd(L, good, scale=float("nan")) == ea.ATTN_ERR_INVALID_ARG
    assert fwd(L, good, d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert fwd(L, good, d=256) == ea.ATTN_ERR_UNSUPPORTED
    assert fwd(L, [FAKE + 8] + [FAKE] * 4) == ea.ATTN_ERR_MISALIGNED
    vp = ctypes.c_void_p
    # varlen entry points need cu_seqlens
    assert L.attn_fwd_varlen(vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), 2, 10, 8, 1, 64,
                             ctypes.c_float(0.1), 1, None, None, None) == ea.ATTN_ERR_INVALID_ARG
    # backward: workspace missing / too small / misaligned
    args = [vp(FAKE)] * 9 + [1, 1, 16, 64, ctypes.c_float(0.125), 1, None, None]
    assert L.attn_bwd(*args, None, 0, None) == ea.ATTN_ERR_WORKSPACE
    assert L.attn_bwd(*args, vp(FAKE), 16, None) == ea.ATTN_ERR_WORKSPACE
    need = ea.attn_bwd_workspace_bytes(1, 1, 16, 64)
    assert L.attn_bwd(*args, vp(FAKE + 16), need, None) == ea.ATTN_ERR_MISALIGNED


def test_blocksparse_host_argument_errors(L):
    import exact_attention_123_b200 as ea
    vp = ctypes.c_void_p
    f = ctypes.c_float(0.1)
    # the tile mask is required, and a mask row must fit the kernels' 64 bits (N <= 8192)
    assert L.attn_fwd_blocksparse(*[vp(FAKE)] * 5, 1, 1, 256, 64, f, 0, None, None) == ea.ATTN_ERR_INVALID_ARG
    assert L.attn_fwd_blocksparse(*[vp(FAKE)] * 5, 1, 1, 8193, 64, f, 0, vp(FAKE), None) == ea.ATTN_ERR_UNSUPPORTED
    assert L.attn_fwd_blocksparse(*[vp(FAKE)] * 5, 1, 1, 256, 96, f, 0, vp(FAKE), None) == ea.ATTN_ERR_UNSUPPORTED
    need = ea.attn_bwd_workspace_bytes(1, 1, 256, 64)
    args = [vp(FAKE)] * 9 + [1, 1, 256, 64, f, 0]
    assert L.attn_bwd_blocksparse(*args, None, vp(FAKE), need, None) == ea.ATTN_ERR_INVALID_ARG
    args[11] = 8320
    assert L.attn_bwd_blocksparse(*args, vp(FAKE), vp(FAKE), need, None) == ea.ATTN_ERR_UNSUPPORTED
    args[11] = 256
    assert L.attn_bwd_blocksparse(*args, vp(FAKE), None, 0, None) == ea.ATTN_ERR_WORKSPACE


def test_fp8_host_argument_errors(L):
    import exact_attention_123_b200 as ea
    vp, f = ctypes.c_void_p, ctypes.c_float

    def call(ptrs=(FAKE,) * 5, scales=(1.0, 1.0, 1.0), d=128, scale=0.1, B=1):
        p = [vp(x) if x else None for x in ptrs]
        return L.attn_fwd_fp8(p[0], p[1], p[2], f(scales[0]), f(scales[1]), f(scales[2]), p[3], p[4], B, 1, 256,
                              d, f(scale), 1, None)
    assert call(ptrs=(FAKE, 0, FAKE, FAKE, FAKE)) == ea.ATTN_ERR_INVALID_ARG
    assert call(scales=(1.0, 0.0, 1.0)) == ea.ATTN_ERR_INVALID_ARG
    assert call(scales=(1.0, 1.0, float("inf"))) == ea.ATTN_ERR_INVALID_ARG
    assert call(scale=-1.0) == ea.ATTN_ERR_INVALID_ARG
    assert call(d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert call(ptrs=(FAKE, FAKE, FAKE + 4, FAKE, FAKE)) == ea.ATTN_ERR_MISALIGNED
    assert call(ptrs=(FAKE, FAKE, FAKE, FAKE, FAKE + 8)) == ea.ATTN_ERR_MISALIGNED
    assert call(B=0) == ea.ATTN_ERR_INVALID_ARG
    # packed layout: cu_seqlens is required; masked dense layout: d must be 64 or 128
    p5 = [vp(FAKE)] * 3
    assert L.attn_fwd_fp8_varlen(*p5, f(1.0), f(1.0), f(1.0), vp(FAKE), vp(FAKE), 2, 100, 64, 1, 128, f(0.1), 1,
                                 None, None, None) == ea.ATTN_ERR_INVALID_ARG
    assert L.attn_fwd_fp8_masked(*p5, f(1.0), f(1.0), f(1.0), vp(FAKE), vp(FAKE), 1, 1, 256, 96, f(0.1), 1,
                                 vp(FAKE), None) == ea.ATTN_ERR_UNSUPPORTED
    # with a tile mask: the mask is required, N <= 8192, and the scales are checked as above
    def sparse(mask, N=256, d=128, scales=(1.0, 1.0, 1.0)):
        return L.attn_fwd_fp8_blocksparse(*p5, *(f(x) for x in scales), vp(FAKE), vp(FAKE), 1, 1, N, d, f(0.1), 1,
                                          mask, None)
    assert sparse(None) == ea.ATTN_ERR_INVALID_ARG
    assert sparse(vp(FAKE), N=8193) == ea.ATTN_ERR_UNSUPPORTED
    assert sparse(vp(FAKE), d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert sparse(vp(FAKE), scales=(1.0, 1.0, -2.0)) == ea.ATTN_ERR_INVALID_ARG


def test_wait_limit_and_fault_hook_setters(L):
    import exact_attention_123_b200 as ea
    prev = ea.attn_set_wait_limit_ms(1234)
    assert ea.attn_set_wait_limit_ms(prev) == 1234
    assert ea.attn_debug_skip_load(5) == -1
    assert ea.attn_debug_skip_load(-1) == 5
    assert ea.attn_debug_force_band(3) == 0
    assert ea.attn_debug_force_band(-2) == 3  # (non-positive: automatic)
    assert ea.attn_debug_force_band(0) == 0


def test_product_package_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "exact_attention_123_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle", txt, re.M), f
                assert "liboracle" not in txt, f
