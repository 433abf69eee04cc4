"""ctypes binding of libcsa.so (the C ABI in include/csa.h).

Argument marshalling only: torch tensors become device pointers, Python
numbers become C scalars, the stream defaults to torch's current stream.
Every computation happens in the CUDA library; if it is missing or fails to
load, every call raises.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_F32, CSA_BF16, CSA_FP8_E4M3, CSA_NVFP4 = 0, 1, 2, 3
DTYPE = {"f32": CSA_F32, "bf16": CSA_BF16, "fp8": CSA_FP8_E4M3, "nvfp4": CSA_NVFP4}

c_int, c_float, c_double, c_size_t, c_void_p = (ctypes.c_int, ctypes.c_float, ctypes.c_double,
                                                 ctypes.c_size_t, ctypes.c_void_p)


class CsaError(RuntimeError):
    pass


class CompressParams(ctypes.Structure):
    _fields_ = [("m", c_int), ("overlap", c_int), ("c", c_int), ("d_rope", c_int),
                ("rope_theta", c_double), ("eps", c_float), ("apply_norm", c_int),
                ("in_dtype", c_int), ("out_dtype", c_int), ("out_entry_offset", c_int)]


class IndexParams(ctypes.Structure):
    _fields_ = [("H_I", c_int), ("d_I", c_int), ("m", c_int), ("qk_dtype", c_int),
                ("score_dtype", c_int)]


class AttnParams(ctypes.Structure):
    _fields_ = [("H", c_int), ("d", c_int), ("n_w", c_int), ("scale", c_float), ("m", c_int),
                ("k", c_int), ("dtype", c_int), ("d_rope_out", c_int), ("rope_theta", c_double)]


class DecodeParams(ctypes.Structure):
    _fields_ = [("b", c_int), ("L", c_int), ("m", c_int), ("c", c_int), ("H", c_int),
                ("c_I", c_int), ("H_I", c_int), ("d_rope", c_int), ("d_rope_I", c_int),
                ("rope_theta", c_double), ("eps", c_float), ("k", c_int), ("n_w", c_int),
                ("scale", c_float), ("kv_dtype", c_int), ("idx_dtype", c_int), ("hca", c_int),
                ("E_cap", c_int), ("mode", c_int), ("P", c_int), ("inv_rope", c_int)]


CSA_MODE_FULL, CSA_MODE_REUSE, CSA_MODE_REINDEX = 0, 1, 2


_DECODE_TENSORS = ["C_a", "Z_a", "C_b", "Z_b", "B_a", "B_b", "CI_a", "ZI_a", "CI_b", "ZI_b",
                   "BI_a", "BI_b", "kv_cache", "kI_cache", "kI_scales", "kv_win", "q", "q_I", "w",
                   "sink", "out", "lse", "idx_out", "count_out", "idx_in", "count_in", "pool",
                   "pool_count"]


class DecodeTensors(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in _DECODE_TENSORS]


class PagedParams(ctypes.Structure):
    _fields_ = [("b", c_int), ("m", c_int), ("c", c_int), ("H", c_int), ("c_I", c_int),
                ("H_I", c_int), ("d_rope", c_int), ("d_rope_I", c_int), ("rope_theta", c_double),
                ("eps", c_float), ("k", c_int), ("n_w", c_int), ("scale", c_float),
                ("kv_dtype", c_int), ("idx_dtype", c_int), ("hca", c_int), ("max_pages", c_int),
                ("num_pages", c_int), ("L_max", c_int), ("inv_rope", c_int)]


_PAGED_TENSORS = ["kv_pages", "kI_pages", "kI_scales", "block_table", "win", "tail_C_a",
                  "tail_Z_a", "tail_C_b", "tail_Z_b", "tail_CI_a", "tail_ZI_a", "tail_CI_b",
                  "tail_ZI_b", "pos", "new_C_a", "new_Z_a", "new_C_b", "new_Z_b", "new_CI_a",
                  "new_ZI_a", "new_CI_b", "new_ZI_b", "new_win", "B_a", "B_b", "BI_a", "BI_b",
                  "q", "q_I", "w", "sink", "out", "lse", "idx_out", "count_out"]


class PagedTensors(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in _PAGED_TENSORS]


PAGE_ENTRIES = 256


class PrefillParams(ctypes.Structure):
    _fields_ = [("b", c_int), ("n", c_int), ("m", c_int), ("c", c_int), ("H", c_int),
                ("c_I", c_int), ("H_I", c_int), ("d_rope", c_int), ("d_rope_I", c_int),
                ("rope_theta", c_double), ("eps", c_float), ("k", c_int), ("n_w", c_int),
                ("scale", c_float), ("kv_dtype", c_int), ("idx_dtype", c_int),
                ("score_dtype", c_int), ("inv_rope", c_int)]


_PREFILL_TENSORS = ["C_a", "Z_a", "C_b", "Z_b", "B_a", "B_b", "CI_a", "ZI_a", "CI_b", "ZI_b",
                    "BI_a", "BI_b", "kv_win", "q", "q_I", "w", "sink", "kv_cache", "kI_cache",
                    "kI_scales", "out", "lse", "idx_out", "count_out"]


class PrefillTensors(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in _PREFILL_TENSORS]


_lib = None

_SIGS = {
    "csa_status_string": (ctypes.c_char_p, [c_int]),
    "csa_version": (c_int, []),
    "csa_device_error": (c_int, [c_void_p]),
    "csa_selftest_bounded_wait": (c_int, [c_int, c_void_p]),
    "csa_compress": (c_int, [ctypes.POINTER(CompressParams)] + [c_void_p] * 6 +
                     [c_int] * 5 + [c_void_p, c_void_p, c_void_p]),
    "csa_quantize": (c_int, [c_int, c_int, c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "csa_index_scores": (c_int, [ctypes.POINTER(IndexParams)] + [c_void_p] * 6 + [c_int] * 4 +
                         [c_void_p, c_void_p]),
    "csa_topk": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p,
                         c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa_topk_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "csa_pool_topk": (c_int, [ctypes.POINTER(IndexParams)] + [c_void_p] * 6 + [c_int] * 4 +
                      [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p, c_size_t,
                       c_void_p]),
    "csa_pool_topk_workspace_size": (c_size_t, [ctypes.POINTER(IndexParams), c_int, c_int, c_int,
                                                c_int]),
    "csa_out_proj": (c_int, [c_void_p, c_void_p] + [c_int] * 5 + [c_void_p, c_void_p, c_size_t,
                                                                 c_void_p]),
    "csa_out_proj_workspace_size": (c_size_t, [c_int] * 5),
    "csa_sparse_attn": (c_int, [ctypes.POINTER(AttnParams), c_void_p, c_void_p, c_int, c_void_p,
                                c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_int,
                                c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "csa_sparse_attn_workspace_size": (c_size_t, [ctypes.POINTER(AttnParams), c_int, c_int, c_int]),
    "csa_sparse_attn_noalloc": (c_int, [ctypes.POINTER(AttnParams), c_void_p, c_void_p, c_int,
                                        c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                                        c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "csa_decode": (c_int, [ctypes.POINTER(DecodeParams), ctypes.POINTER(DecodeTensors), c_void_p,
                           c_size_t, c_void_p]),
    "csa_decode_workspace_size": (c_size_t, [ctypes.POINTER(DecodeParams)]),
    "csa_prefill": (c_int, [ctypes.POINTER(PrefillParams), ctypes.POINTER(PrefillTensors),
                            c_void_p, c_size_t, c_void_p]),
    "csa_prefill_workspace_size": (c_size_t, [ctypes.POINTER(PrefillParams)]),
    "csa_decode_launch_count": (c_int, [ctypes.POINTER(DecodeParams)]),
    "csa_decode_paged": (c_int, [ctypes.POINTER(PagedParams), ctypes.POINTER(PagedTensors),
                                 c_void_p, c_size_t, c_void_p]),
    "csa_decode_paged_workspace_size": (c_size_t, [ctypes.POINTER(PagedParams)]),
    "csa_decode_paged_launch_count": (c_int, [ctypes.POINTER(PagedParams)]),
    "csa_prefill_launch_count": (c_int, [ctypes.POINTER(PrefillParams)]),
    "csa_cp_candidates": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_int,
                                  c_void_p, c_void_p, c_void_p]),
    "csa_cp_merge_workspace_size": (c_size_t, [c_int, c_int, c_int]),
    "csa_cp_merge": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_size_t, c_void_p]),
    "csa_cp_pack_rows": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                 c_int, c_int, c_void_p, c_void_p]),
}


def lib():
    """The loaded CUDA library; raises if it is missing (no CPU fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise CsaError("libcsa.so is not built (%s); run "
                           "`python -m long_context_sparse_05_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        if x.device.type != "cuda":
            raise CsaError("tensor arguments must be CUDA tensors (got %s)" % x.device)
        if not x.is_contiguous():
            raise CsaError("tensor arguments must be contiguous")
        return x.data_ptr()
    return int(x)


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def _check(status):
    if status != 0:
        raise CsaError(lib().csa_status_string(status).decode())


def csa_device_error(stream=None):
    """Synchronise and read/clear the device error word (0 = no bounded wait gave up)."""
    return int(lib().csa_device_error(_stream(stream)))


def csa_selftest_bounded_wait(limit_us, stream=None):
    _check(lib().csa_selftest_bounded_wait(limit_us, _stream(stream)))


def csa_status_string(status):
    return lib().csa_status_string(status).decode()


def csa_compress(p, C_a, Z_a, B_a, C_b, Z_b, B_b, b, n, entry_begin, entry_count,
                 out_entries_per_seq, out, out_scales=None, stream=None):
    _check(lib().csa_compress(ctypes.byref(p), _ptr(C_a), _ptr(Z_a), _ptr(B_a), _ptr(C_b),
                              _ptr(Z_b), _ptr(B_b), b, n, entry_begin, entry_count,
                              out_entries_per_seq, _ptr(out), _ptr(out_scales), _stream(stream)))


def csa_quantize(in_dtype, out_dtype, x, rows, d, codes, scales, stream=None):
    _check(lib().csa_quantize(in_dtype, out_dtype, _ptr(x), rows, d, _ptr(codes), _ptr(scales),
                              _stream(stream)))


def csa_index_scores(p, q_I, q_scales, w, k_I, k_scales, q_pos, b, T, E_cap, E, scores,
                     stream=None):
    _check(lib().csa_index_scores(ctypes.byref(p), _ptr(q_I), _ptr(q_scales), _ptr(w), _ptr(k_I),
                                  _ptr(k_scales), _ptr(q_pos), b, T, E_cap, E, _ptr(scores),
                                  _stream(stream)))


def csa_topk(scores, score_dtype, q_pos, m, b, T, E, k, idx, count, ws=None, ws_bytes=0,
             stream=None):
    _check(lib().csa_topk(_ptr(scores), score_dtype, _ptr(q_pos), m, b, T, E, k, _ptr(idx),
                          _ptr(count), _ptr(ws), ws_bytes, _stream(stream)))


def csa_topk_workspace_size(score_dtype, b, T, E, k):
    return int(lib().csa_topk_workspace_size(score_dtype, b, T, E, k))


def csa_pool_topk_workspace_size(p, b, T, P, k):
    return int(lib().csa_pool_topk_workspace_size(ctypes.byref(p), b, T, P, k))


def csa_pool_topk(p, q_I, q_scales, w, k_I, k_scales, q_pos, b, T, E_cap, E, pool, pool_count,
                  P, k, idx, count, ws, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    _check(lib().csa_pool_topk(ctypes.byref(p), _ptr(q_I), _ptr(q_scales), _ptr(w), _ptr(k_I),
                               _ptr(k_scales), _ptr(q_pos), b, T, E_cap, E, _ptr(pool),
                               _ptr(pool_count), P, k, _ptr(idx), _ptr(count), _ptr(ws), ws_bytes,
                               _stream(stream)))


def csa_out_proj_workspace_size(T, H, d, g, d_g):
    return int(lib().csa_out_proj_workspace_size(T, H, d, g, d_g))


def csa_out_proj(o, W, T, H, d, g, d_g, y, ws=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(lib().csa_out_proj(_ptr(o), _ptr(W), T, H, d, g, d_g, _ptr(y), _ptr(ws), ws_bytes,
                              _stream(stream)))


def csa_sparse_attn_workspace_size(p, b, T, E_cap):
    return int(lib().csa_sparse_attn_workspace_size(ctypes.byref(p), b, T, E_cap))


def csa_sparse_attn(p, q, kv_comp, E_cap, idx, count, kv_win, n, q_pos, sink, b, T, out, lse=None,
                    ws=None, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 0
    _check(lib().csa_sparse_attn(ctypes.byref(p), _ptr(q), _ptr(kv_comp), E_cap, _ptr(idx),
                                 _ptr(count), _ptr(kv_win), n, _ptr(q_pos), _ptr(sink), b, T,
                                 _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def csa_sparse_attn_noalloc(p, q, kv_comp, E_cap, idx, count, kv_win, n, q_pos, sink, b, T, out,
                            lse=None, stream=None):
    """csa_sparse_attn without a workspace: the library's fixed scratch array is used."""
    _check(lib().csa_sparse_attn_noalloc(ctypes.byref(p), _ptr(q), _ptr(kv_comp), E_cap, _ptr(idx),
                                         _ptr(count), _ptr(kv_win), n, _ptr(q_pos), _ptr(sink), b,
                                         T, _ptr(out), _ptr(lse), _stream(stream)))


def _fill(struct_cls, names, tensors):
    s = struct_cls()
    for n in names:
        setattr(s, n, _ptr(tensors.get(n)))
    return s


def csa_decode_workspace_size(p):
    return int(lib().csa_decode_workspace_size(ctypes.byref(p)))


def csa_decode(p, tensors, ws, ws_bytes=None, stream=None):
    """tensors: dict with the csa_decode_tensors field names (missing -> NULL)."""
    x = _fill(DecodeTensors, _DECODE_TENSORS, tensors)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    _check(lib().csa_decode(ctypes.byref(p), ctypes.byref(x), _ptr(ws), ws_bytes, _stream(stream)))


def csa_prefill_workspace_size(p):
    return int(lib().csa_prefill_workspace_size(ctypes.byref(p)))


def csa_prefill(p, tensors, ws, ws_bytes=None, stream=None):
    x = _fill(PrefillTensors, _PREFILL_TENSORS, tensors)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    _check(lib().csa_prefill(ctypes.byref(p), ctypes.byref(x), _ptr(ws), ws_bytes,
                             _stream(stream)))



def csa_decode_launch_count(p):
    return int(lib().csa_decode_launch_count(ctypes.byref(p)))


def csa_prefill_launch_count(p):
    return int(lib().csa_prefill_launch_count(ctypes.byref(p)))


def csa_decode_paged_workspace_size(p):
    return int(lib().csa_decode_paged_workspace_size(ctypes.byref(p)))


def csa_decode_paged_launch_count(p):
    return int(lib().csa_decode_paged_launch_count(ctypes.byref(p)))


def csa_decode_paged(p, tensors, ws, ws_bytes=None, stream=None):
    """tensors: dict with the csa_paged_tensors field names (missing -> NULL)."""
    x = _fill(PagedTensors, _PAGED_TENSORS, tensors)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    _check(lib().csa_decode_paged(ctypes.byref(p), ctypes.byref(x), _ptr(ws), ws_bytes,
                                  _stream(stream)))


# ---------------------------------------------------------------- context-parallel decode

def csa_cp_candidates(scores, E_local, idx, count, b, k, entry_offset, cand_scores, cand_idx,
                      stream=None):
    _check(lib().csa_cp_candidates(_ptr(scores), E_local, _ptr(idx), _ptr(count), b, k,
                                   entry_offset, _ptr(cand_scores), _ptr(cand_idx),
                                   _stream(stream)))


def csa_cp_merge_workspace_size(G, b, k):
    return int(lib().csa_cp_merge_workspace_size(G, b, k))


def csa_cp_merge(cand_scores, cand_idx, G, b, k, idx, count, rows_idx, ws, ws_bytes, stream=None):
    _check(lib().csa_cp_merge(_ptr(cand_scores), _ptr(cand_idx), G, b, k, _ptr(idx), _ptr(count),
                              _ptr(rows_idx), _ptr(ws), ws_bytes, _stream(stream)))


def csa_cp_pack_rows(kv_local, E_cap_local, E_local, entry_offset, c, kv_dtype, idx, count, b, k,
                     rows, stream=None):
    _check(lib().csa_cp_pack_rows(_ptr(kv_local), E_cap_local, E_local, entry_offset, c, kv_dtype,
                                  _ptr(idx), _ptr(count), b, k, _ptr(rows), _stream(stream)))
