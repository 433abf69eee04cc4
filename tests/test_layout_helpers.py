"""The test-side converters of the tiled NVFP4 key-scale layout (the layout `csa.h`
documents for the key cache and the index-key scales), checked against an explicit
construction of that layout and for being a bijection."""

import numpy as np

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
