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
