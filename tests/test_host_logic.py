"""CPU-only checks of host-side logic: the test helpers' vectorised scale
placement, the input generators' recipe, and the C library's exports and
argument validation (no kernel launches)."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import nvfp4_oracle as o
from qad_nvfp4_quantize_b200 import inputs
from tests.util import tiled

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_vectorised_tiling_matches_oracle_loop():
    rng = np.random.default_rng(0)
    for rows, nb in [(1, 4), (130, 8), (256, 80)]:
        s = rng.integers(0, 127, (rows, nb)).astype(np.uint8)
        assert np.array_equal(tiled(s), o.scales_to_tiled(s))


def test_input_recipe_is_seeded_and_shaped():
    a = inputs.tiny_linear(0)
    b = inputs.tiny_linear(0)
    assert a["x"].shape == (128, 256) and a["w"].shape == (256, 256)
    assert (a["x"] == b["x"]).all()
    f = inputs.four_over_six_linear(0, M=8, N=64, K=256)
    w = f["w"].float().numpy()
    assert (np.abs(w) > 0.2).sum() >= 1        # the x20 entries are present
    m = inputs.moe_experts(0, T=32, H=256, E=8, topk=2, I=128)
    ids = m["topk_ids"].numpy()
    assert ids.shape == (32, 2) and (ids[:, 0] != ids[:, 1]).all()
    assert np.allclose(m["topk_w"].numpy().sum(1), 1.0, atol=1e-6)


def _header_symbols():
    with open(os.path.join(ROOT, "include", "nvfp4.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def clib():
    import qad_nvfp4_quantize_b200 as nv
    if not os.path.exists(nv.library_path):
        pytest.fail("libnvfp4.so is not built")
    return ctypes.CDLL(nv.library_path)


def test_library_exports_every_declared_symbol(clib):
    missing = [s for s in _header_symbols() if not hasattr(clib, s)]
    assert not missing, f"not exported: {missing}"
    assert len(_header_symbols()) >= 14


def test_bounds_checking_build_exports_the_same_symbols():
    path = os.path.join(ROOT, "qad_nvfp4_quantize_b200", "libnvfp4_debug.so")
    if not os.path.exists(path):
        pytest.fail("libnvfp4_debug.so is not built")
    dbg = ctypes.CDLL(path)
    missing = [s for s in _header_symbols() if not hasattr(dbg, s)]
    assert not missing, f"not exported by the bounds-checking build: {missing}"
    dbg.nvfp4_status_string.restype = ctypes.c_char_p
    assert dbg.nvfp4_status_string(8).startswith(b"a computed index")


def test_host_side_queries_and_validation(clib):
    import qad_nvfp4_quantize_b200 as nv
    L = nv.lib()
    assert L.nvfp4_version() >= 100
    assert L.nvfp4_scale_bytes(128, 256) == 512 * 4
    assert L.nvfp4_scale_bytes(129, 64) == 2 * 512
    assert L.nvfp4_scale_bytes(128, 100) == 0
    assert L.nvfp4_quantize_workspace_bytes(128, 256) > 0
    # invalid arguments are rejected before any device work
    assert L.nvfp4_quantize(None, 128, 100, 0, None, None, None, None, None, None, 0, None) == 1
    assert L.nvfp4_quantize(None, -1, 64, 0, None, None, None, None, None, None, 0, None) == 1
    assert L.nvfp4_quantize(None, 1, 64, 7, None, None, None, None, None, None, 0, None) == 1
    assert L.nvfp4_gemm(None, None, None, None, None, None, 1, 24, 64, None, None) == 1
    assert L.nvfp4_gemm(None, None, None, None, None, None, 1, 32, 96, None, None) == 1
    assert L.nvfp4_fake_quant(None, 4, 64, 0, None, ctypes.c_void_p(16), None, None, 0, None) == 1
    assert L.nvfp4_status_string(6) == b"device wait timed out"


def _chunk_index_params(shapes, tmp_path):
    """Run the library's host-side chunk-index helpers (kernels.h) for each
    (M, K) through a small g++-built program: (narrow?, 32-bit magic, 64-bit
    magic)."""
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    cuda_inc = "/usr/local/cuda/include"
    if gxx is None or not os.path.isdir(cuda_inc):
        pytest.skip("g++ or the CUDA headers are not available")
    src = tmp_path / "chunk_params.cpp"
    src.write_text(
        '#include <cstdio>\n#include "kernels.h"\n'
        "int main() { long long M, K;\n"
        "  while (std::scanf(\"%lld %lld\", &M, &K) == 2)\n"
        "    std::printf(\"%d %llu %llu\\n\", (int)nvfp4::narrow_chunks(M, K),\n"
        "                (unsigned long long)nvfp4::chunk_magic_narrow(K), (unsigned long long)nvfp4::chunk_magic(K));\n"
        "  return 0; }\n")
    exe = tmp_path / "chunk_params"
    csrc = os.path.join(ROOT, "qad_nvfp4_quantize_b200", "csrc")
    subprocess.run([gxx, "-std=c++17", "-O1", f"-I{csrc}", f"-I{cuda_inc}", str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], input="".join(f"{m} {k}\n" for m, k in shapes), capture_output=True,
                         text=True, check=True).stdout.split("\n")
    return [tuple(int(v) for v in line.split()) for line in out if line.strip()]


def test_chunk_row_division_is_exact_where_32bit_is_chosen(tmp_path):
    # The kernels divide a chunk index ch by cpr (chunks per row) as
    # umulhi(ch, magic): exact for every chunk of every tensor the host sends
    # down the 32-bit path; the 64-bit magic is exact everywhere.
    shapes = [(1, 64), (1, 512), (7, 513), (4096, 5120), (16384, 14336), (16384, 4096), (65536, 2048),
              (1 << 20, 512), (3, 1 << 22), (4, (1 << 24) + 64), (1, 1 << 25), (262144, 8192),
              (2047, 65536), (65535, 32768)]
    rng = np.random.default_rng(5)
    for (M, K), (narrow, m32, m64) in zip(shapes, _chunk_index_params(shapes, tmp_path)):
        cpr = (K + 511) // 512
        n = M * cpr
        chs = {0, cpr - 1, cpr, n - 1, max(n - cpr, 0), n // 2}
        chs |= set(int(c) for c in rng.integers(0, n, 200))
        if narrow:
            # every element index and scale-byte offset fits, and the division is exact
            assert (M + 128) * cpr * 512 < 1 << 31
            for ch in chs:
                r = ch if cpr == 1 else (ch * m32) >> 32
                assert r == ch // cpr, (M, K, ch)
        for ch in chs:
            r = ch if cpr == 1 else (ch * m64) >> 64
            assert r == ch // cpr, (M, K, ch)
    # shapes near the limits take the 64-bit path
    flags = dict(zip(shapes, [p[0] for p in _chunk_index_params(shapes, tmp_path)]))
    assert flags[(4096, 5120)] == 1 and flags[(16384, 14336)] == 1
    assert flags[(4, (1 << 24) + 64)] == 0 and flags[(1, 1 << 25)] == 0 and flags[(262144, 8192)] == 0
