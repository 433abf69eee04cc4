"""The oracle's FP8 (E4M3) and FP4 (E2M1) codecs and its bf16 rounding against CUDA's
own conversion routines (`cuda_fp8.h`, `cuda_fp4.h`, `cuda_bf16.h`, host-callable),
called from a host-only program built with nvcc: every code value decoded, and
encodings of random values, every tie between neighbouring codes, and out-of-range
values.  No GPU is used."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import codecs

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include <vector>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
int main(int argc, char** argv) {
  std::vector<float> x;
  FILE* f = std::fopen(argv[1], "rb");
  float v;
  while (std::fread(&v, 4, 1, f) == 1) x.push_back(v);
  std::fclose(f);
  FILE* o = std::fopen(argv[2], "wb");
  for (int c = 0; c < 256; ++c) {
    const float y = __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3)));
    std::fwrite(&y, 4, 1, o);
  }
  for (int c = 0; c < 16; ++c) {
    const float y = __half2float(__half(__nv_cvt_fp4_to_halfraw((__nv_fp4_storage_t)c, __NV_E2M1)));
    std::fwrite(&y, 4, 1, o);
  }
  for (float xi : x) {
    const uint8_t c = __nv_cvt_float_to_fp8(xi, __NV_SATFINITE, __NV_E4M3);
    std::fwrite(&c, 1, 1, o);
  }
  for (float xi : x) {
    const uint8_t c = __nv_cvt_float_to_fp4(xi, __NV_E2M1, cudaRoundNearest);
    std::fwrite(&c, 1, 1, o);
  }
  for (float xi : x) {
    const unsigned short b = __bfloat16_as_ushort(__float2bfloat16_rn(xi));
    std::fwrite(&b, 2, 1, o);
  }
  std::fclose(o);
  return 0;
}
"""


def _neighbour_ties(values):
    pos = np.unique(values[np.isfinite(values) & (values >= 0)])
    mids = (pos[:-1] + pos[1:]) / 2
    return np.concatenate([pos, -pos, mids, -mids])


@pytest.fixture(scope="module")
def cuda_codecs(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("codecs")
    src, exe = d / "codecs.cu", d / "codecs"
    src.write_text(PROGRAM)
    subprocess.run([nvcc, "-std=c++17", str(src), "-o", str(exe)], check=True,
                   capture_output=True, timeout=300)
    rng = np.random.default_rng(5)
    e4m3_vals = codecs.e4m3_decode(np.arange(256, dtype=np.uint8))
    e2m1_vals = codecs.e2m1_decode(np.arange(16, dtype=np.uint8))
    x = np.concatenate([
        rng.uniform(-448, 448, 4000), rng.normal(0, 0.01, 4000), rng.uniform(-7, 7, 4000),
        _neighbour_ties(e4m3_vals), _neighbour_ties(e2m1_vals),
        [0.0, -0.0, 500.0, -500.0, 1e30, -1e30, 6.5, -6.5, 100.0],
    ]).astype(np.float32)
    # float32 values at, just below and just above a bf16 rounding tie, all exponents
    hi = rng.integers(0, 1 << 16, 3000, dtype=np.uint32) << 16
    hi = hi[((hi >> 23) & 0xFF) != 0xFF]                       # finite only
    ties = np.concatenate([hi | 0x8000, hi | 0x7FFF, hi | 0x8001]).view(np.float32)
    x = np.concatenate([x, ties, np.float32([3.3895e38, 3.4e38, -3.4e38, 1e-40, -1e-40])])
    (d / "x.bin").write_bytes(x.tobytes())
    subprocess.run([str(exe), str(d / "x.bin"), str(d / "out.bin")], check=True, timeout=60)
    raw = (d / "out.bin").read_bytes()
    dec8 = np.frombuffer(raw[:1024], dtype=np.float32)
    dec4 = np.frombuffer(raw[1024:1088], dtype=np.float32)
    enc8 = np.frombuffer(raw[1088:1088 + x.size], dtype=np.uint8)
    enc4 = np.frombuffer(raw[1088 + x.size:1088 + 2 * x.size], dtype=np.uint8)
    bf = np.frombuffer(raw[1088 + 2 * x.size:1088 + 4 * x.size], dtype=np.uint16)
    return dict(x=x, dec8=dec8, dec4=dec4, enc8=enc8, enc4=enc4, bf16=bf)


def test_e4m3_decode_every_code(cuda_codecs):
    ours = codecs.e4m3_decode(np.arange(256, dtype=np.uint8))
    ref = cuda_codecs["dec8"].astype(np.float64)
    nan = np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(ours), nan)
    np.testing.assert_array_equal(ours[~nan], ref[~nan])


def test_e2m1_decode_every_code(cuda_codecs):
    ours = codecs.e2m1_decode(np.arange(16, dtype=np.uint8))
    np.testing.assert_array_equal(ours, cuda_codecs["dec4"].astype(np.float64))


def test_e4m3_encode_round_to_nearest_even_and_saturation(cuda_codecs):
    ours = codecs.e4m3_encode(cuda_codecs["x"])
    np.testing.assert_array_equal(ours, cuda_codecs["enc8"])


def test_e2m1_encode_round_to_nearest_even_and_saturation(cuda_codecs):
    ours = codecs.e2m1_encode(cuda_codecs["x"])
    np.testing.assert_array_equal(ours, cuda_codecs["enc4"])


def test_bf16_round_to_nearest_even(cuda_codecs):
    x = cuda_codecs["x"]
    ours = codecs.bf16_bits(codecs.round_to_bf16(x.astype(np.float64)))
    np.testing.assert_array_equal(ours, cuda_codecs["bf16"])
