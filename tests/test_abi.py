"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, its structs match the ctypes mirrors, and argument errors come back as
CSA_ERR_INVALID_ARG before any CUDA call (so these run without a GPU)."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import long_context_sparse_05_b200 as csa
from long_context_sparse_05_b200 import _lib as L
from long_context_sparse_05_b200 import runner, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from long_context_sparse_05_b200 import build
    build.build()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(csa_\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 12, names
    lib = ctypes.CDLL(L.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    assert set(declared_functions()) <= set(L._SIGS), set(declared_functions()) - set(L._SIGS)


def test_page_size_matches_header():
    m = re.search(r"#define\s+CSA_PAGE_ENTRIES\s+(\d+)", open(HEADER).read())
    assert m and int(m.group(1)) == L.PAGE_ENTRIES


def test_noalloc_scratch_size_matches_header():
    """The binding's copy of the fixed scratch size is the header's (the tests rely on it)."""
    m = re.search(r"#define\s+CSA_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)",
                  open(HEADER).read())
    assert m, "CSA_NOALLOC_SCRATCH_BYTES not found"
    assert L.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_struct_layouts_match_c():
    structs = {"csa_compress_params": L.CompressParams, "csa_index_params": L.IndexParams,
               "csa_attn_params": L.AttnParams, "csa_decode_params": L.DecodeParams,
               "csa_decode_tensors": L.DecodeTensors, "csa_prefill_params": L.PrefillParams,
               "csa_paged_params": L.PagedParams, "csa_paged_tensors": L.PagedTensors,
               "csa_prefill_tensors": L.PrefillTensors}
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "csa.h"', "int main(void){"]
    for cname, py in structs.items():
        prog.append('printf("%s %%zu\\n", sizeof(%s));' % (cname, cname))
        for fname, _ in py._fields_:
            prog.append('printf("%s.%s %%zu\\n", offsetof(%s, %s));' % (cname, fname, cname, fname))
    prog.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write("\n".join(prog))
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-I",
                               "/usr/local/cuda/include", c, "-o", exe])
        out = subprocess.check_output([exe], text=True).split("\n")
    got = dict(line.split() for line in out if line)
    for cname, py in structs.items():
        assert int(got[cname]) == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert int(got["%s.%s" % (cname, fname)]) == getattr(py, fname).offset, (cname, fname)


def test_status_strings():
    assert csa.csa_status_string(0) == "CSA_OK"
    assert "INVALID" in csa.csa_status_string(1)
    assert L.lib().csa_version() >= 100


def test_invalid_arguments_rejected_on_host():
    lib = L.lib()
    p = L.CompressParams(m=0, overlap=1, c=64, d_rope=16, rope_theta=1e4, eps=1e-6, apply_norm=1,
                         in_dtype=0, out_dtype=0)
    fake = 1 << 20   # never dereferenced: validation fails first
    assert lib.csa_compress(ctypes.byref(p), fake, fake, fake, fake, fake, fake, 1, 64, 0, 16, 16,
                            fake, None, None) == 1
    p.m = 4
    p.d_rope = 7   # odd rotary width
    assert lib.csa_compress(ctypes.byref(p), fake, fake, fake, fake, fake, fake, 1, 64, 0, 16, 16,
                            fake, None, None) == 1
    p.d_rope = 16
    # more entries than the raw rows can complete
    assert lib.csa_compress(ctypes.byref(p), fake, fake, fake, fake, fake, fake, 1, 64, 0, 17, 17,
                            fake, None, None) == 1
    # unaligned pointer
    assert lib.csa_compress(ctypes.byref(p), fake + 2, fake, fake, fake, fake, fake, 1, 64, 0, 16,
                            16, fake, None, None) == 1
    # zero work is a no-op success
    assert lib.csa_compress(ctypes.byref(p), None, None, None, None, None, None, 0, 64, 0, 16, 16,
                            None, None, None) == 0
    ip = L.IndexParams(H_I=4, d_I=20, m=4, qk_dtype=0, score_dtype=0)   # d_I not a multiple of 16
    assert lib.csa_index_scores(ctypes.byref(ip), fake, None, fake, fake, None, fake, 1, 1, 8, 8,
                                fake, None) == 1
    assert lib.csa_topk(fake, 5, fake, 4, 1, 1, 8, 2, fake, fake, None, 0, None) == 1
    ap = L.AttnParams(H=4, d=64, n_w=16, scale=0.125, m=4, k=0, dtype=0)
    assert lib.csa_sparse_attn(ctypes.byref(ap), fake, fake, 8, fake, fake, fake, 64, fake, fake,
                               1, 1, fake, None, None, 0, None) == 1   # idx given with k = 0
    assert lib.csa_quantize(1, 2, fake, 4, 24, fake, fake, None) == 1  # d not a multiple of 16
    # NVFP4 index keys keep their scales in 64-element K blocks: widths must be multiples of 64
    p4 = L.CompressParams(m=4, overlap=1, c=32, d_rope=16, rope_theta=1e4, eps=1e-6,
                          apply_norm=1, in_dtype=1, out_dtype=L.CSA_NVFP4)
    assert lib.csa_compress(ctypes.byref(p4), fake, fake, fake, fake, fake, fake, 1, 64, 0, 16,
                            16, fake, fake, None) == 1
    ip4 = L.IndexParams(H_I=4, d_I=32, m=4, qk_dtype=L.CSA_NVFP4, score_dtype=L.CSA_BF16)
    assert lib.csa_index_scores(ctypes.byref(ip4), fake, fake, fake, fake, fake, fake, 1, 1, 8, 8,
                                fake, None) == 1
    # the tensor-core indexer shapes (64 heads x 128 dims) need 16-byte aligned operands and
    # FP8 key-scale rows that are whole 16-byte runs: rejected, never run on a slower kernel
    for fmt in (L.CSA_FP8_E4M3, L.CSA_NVFP4):
        ipt = L.IndexParams(H_I=64, d_I=128, m=4, qk_dtype=fmt, score_dtype=L.CSA_BF16)
        assert lib.csa_index_scores(ctypes.byref(ipt), fake, fake, fake, fake + 8, fake, fake, 1,
                                    1, 1024, 1024, fake, None) == 1
    ipt = L.IndexParams(H_I=64, d_I=128, m=4, qk_dtype=L.CSA_FP8_E4M3, score_dtype=L.CSA_BF16)
    assert lib.csa_index_scores(ctypes.byref(ipt), fake, fake, fake, fake, fake, fake, 1, 1, 1026,
                                1026, fake, None) == 1
    dp = runner.decode_params(workloads.CSA_DECODE_1M)
    dp.c_I = 96                                        # the only defect: every pointer is set
    x = L.DecodeTensors(**{n: fake for n, _ in L.DecodeTensors._fields_})
    assert L.lib().csa_decode(ctypes.byref(dp), ctypes.byref(x), 1 << 20, 1 << 30, None) == 1
    # CSA2 modes: an unknown mode, Reuse without a selection, Reindex without a pool or with
    # an empty one, and any mode but Full for HCA
    for mode, P, drop, hca in ((7, 0, None, 0), (L.CSA_MODE_REUSE, 0, "idx_in", 0),
                               (L.CSA_MODE_REINDEX, 2048, "pool_count", 0),
                               (L.CSA_MODE_REINDEX, 0, None, 0), (L.CSA_MODE_REUSE, 0, None, 1)):
        dp = runner.decode_params(workloads.CSA_DECODE_1M)
        dp.mode, dp.P, dp.hca = mode, P, hca
        x = L.DecodeTensors(**{n: fake for n, _ in L.DecodeTensors._fields_})
        if drop:
            setattr(x, drop, None)
        assert L.lib().csa_decode(ctypes.byref(dp), ctypes.byref(x), 1 << 20, 1 << 34, None) == 1
    # the pool top-k: a pool of length 0, a missing pool count, too small a workspace
    ip = L.IndexParams(H_I=64, d_I=128, m=4, qk_dtype=L.CSA_FP8_E4M3, score_dtype=L.CSA_BF16)
    args = [fake] * 6 + [1, 1, 4096, 4096, fake, fake, 1024, 64, fake, fake, fake, 1 << 30, None]
    bad = list(args); bad[12] = 0
    assert lib.csa_pool_topk(ctypes.byref(ip), *bad) == 1
    bad = list(args); bad[11] = None
    assert lib.csa_pool_topk(ctypes.byref(ip), *bad) == 1
    bad = list(args); bad[17] = 16
    assert lib.csa_pool_topk(ctypes.byref(ip), *bad) == 1


def test_workspace_sizes_are_host_only_and_positive():
    for w in workloads.ALL.values():
        if w.kind == "csa_prefill":
            n = L.csa_prefill_workspace_size(runner.prefill_params(w))
        else:
            n = L.csa_decode_workspace_size(runner.decode_params(w))
        assert n > 0
    # a too-small workspace is an argument error
    w = workloads.CSA_DECODE_64K
    p = runner.decode_params(w)
    x = L.DecodeTensors()
    assert L.lib().csa_decode(ctypes.byref(p), ctypes.byref(x), 1 << 20, 16, None) == 1


def test_product_path_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", "/nonexistent/libcsa.so")
    with pytest.raises(L.CsaError):
        L.lib()


def test_noalloc_scratch_size_matches_the_header():
    # the binding's copy of the no-alloc scratch size is the header's CSA_NOALLOC_SCRATCH_BYTES
    hdr = open(HEADER).read()
    m = re.search(r"#define CSA_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m, "CSA_NOALLOC_SCRATCH_BYTES not found in csa.h"
    assert int(m.group(1)) << int(m.group(2)) == L.NOALLOC_SCRATCH_BYTES
