"""The test-side converters of the tiled NVFP4 key-scale layout (the layout `csa.h`
documents for the key cache and the index-key scales), checked against an explicit
construction of that layout and for being a bijection."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from helpers import nvfp4_key_scale_index, nvfp4_scales_from_tiled, nvfp4_scales_to_tiled


def _tiled_by_loops(rows):
    """The layout spelled out: per tile of 128 entries and per 64-element K block kb,
    512 bytes in which lane l (entry % 32) holds 16 bytes: for row group q = (entry % 128)
    // 32, bytes 4q .. 4q+3 are the scales of blocks 4kb .. 4kb+3 of that entry."""
    E, nb = rows.shape
    assert E % 128 == 0 and nb % 4 == 0
    out = np.zeros(E * nb, dtype=rows.dtype)
    for tile in range(E // 128):
        for kb in range(nb // 4):
            base = tile * 128 * nb + kb * 512
            for l in range(32):
                for q in range(4):
                    for j in range(4):
                        out[base + l * 16 + q * 4 + j] = rows[tile * 128 + q * 32 + l, 4 * kb + j]
    return out.reshape(E, nb)


def test_index_matches_the_spelled_out_layout():
    rng = np.random.default_rng(0)
    rows = rng.integers(0, 256, size=(256, 16), dtype=np.uint8)   # 2 tiles, c = 256 (4 K blocks)
    np.testing.assert_array_equal(nvfp4_scales_to_tiled(rows), _tiled_by_loops(rows))


def test_index_is_a_bijection_on_whole_tiles_and_injective_on_ragged_ones():
    for E, c in ((128, 64), (384, 128), (1000, 128), (129, 64)):
        idx = nvfp4_key_scale_index(E, c).reshape(-1)
        e_pad = (E + 127) // 128 * 128
        assert len(np.unique(idx)) == idx.size                     # no two scales share a byte
        assert idx.min() >= 0 and idx.max() < e_pad * (c // 16)    # inside the padded area
        if E % 128 == 0:
            assert np.array_equal(np.sort(idx), np.arange(E * (c // 16)))


def test_round_trip_with_batch_dims_and_ragged_length():
    rng = np.random.default_rng(1)
    rows = rng.integers(0, 256, size=(3, 1000, 8), dtype=np.uint8)
    tiled = nvfp4_scales_to_tiled(rows, E_cap=1100)
    assert tiled.shape == (3, 1152, 8)
    np.testing.assert_array_equal(nvfp4_scales_from_tiled(tiled, 1000), rows)


def test_kernel_layout_function_matches_the_helpers(tmp_path):
    """The kernels' own offset function (host-callable, in the CUDA sources) against the
    helper, on a host-only program built with nvcc: no GPU is touched."""
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "layout.cu"
    src.write_text(
        '#include <cstdio>\n#include "common.cuh"\n'
        "int main() {\n"
        "  const int cs[2] = {64, 128};\n"
        "  for (int ci = 0; ci < 2; ++ci)\n"
        "    for (long long e = 0; e < 300; ++e)\n"
        "      for (int blk = 0; blk < cs[ci] / 16; ++blk)\n"
        '        std::printf("%zu\\n", csa::nvfp4_key_scale_offset(e, blk, cs[ci]));\n'
        '  std::printf("%zu %zu\\n", csa::nvfp4_key_scale_seq_bytes(300, 64),\n'
        "              csa::nvfp4_key_scale_seq_bytes(256, 128));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([nvcc, "-std=c++17", "-I", os.path.join(root, "include"),
                    "-I", os.path.join(root, "long_context_sparse_05_b200", "csrc"),
                    str(src), "-o", str(exe)], check=True, capture_output=True, timeout=300)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                         timeout=60).stdout.split("\n")
    got = np.array([int(v) for v in out[:-2]])
    want = np.concatenate([nvfp4_key_scale_index(300, c).reshape(-1) for c in (64, 128)])
    np.testing.assert_array_equal(got, want)
    assert out[-2].split() == [str(3 * 128 * 4), str(2 * 128 * 8)]   # ceil(E/128) tiles of 8c bytes
