"""Comparison helpers shared by the parity tests."""

import numpy as np
import torch

from oracle import codecs


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_close(gpu, ref, rtol):
    """Element-wise |gpu - ref| <= rtol * (|ref| + rms(ref)) (the reading of 'relative')."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref[np.isfinite(ref)] ** 2)) if np.any(np.isfinite(ref)) else 0.0
    err = np.abs(gpu - ref)
    bound = rtol * (np.abs(ref) + rms)
    bad = ~(err <= bound)
    same_inf = np.isinf(gpu) & np.isinf(ref) & (np.sign(gpu) == np.sign(ref))
    bad &= ~same_inf
    return (not np.any(bad)), (float(np.max(np.where(np.isfinite(err), err, 0))) if err.size else 0.0), \
        int(np.sum(bad))


def assert_rel_close(gpu, ref, rtol, what=""):
    ok, mx, nbad = rel_close(gpu, ref, rtol)
    assert ok, "%s: %d elements beyond rtol %g (max abs err %g)" % (what, nbad, rtol, mx)


def assert_abs_close(gpu, ref, atol, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.max(np.abs(gpu - ref)) if gpu.size else 0.0
    assert err <= atol, "%s: max abs err %g > %g" % (what, err, atol)


def bf16_ulp(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, ex = np.frexp(np.where(x > 0, x, 1.0))
    return np.ldexp(1.0, np.maximum(ex - 1, -126) - 7)


def topk_band_check(gpu_idx, gpu_cnt, exact_scores, ev, k, rel_band=1e-3):
    """Validate a GPU selection against the oracle's exact (pre-rounding) scores.

    Exact match except for entries whose exact score lies within
    max(rel_band * |tau|, one bf16 ulp of tau) of the k-th largest exact
    score tau.  Also checks count, ordering, range and uniqueness.  Returns the
    number of entries that differ from the oracle's own choice.
    """
    gpu_idx = np.asarray(gpu_idx)
    cnt = int(gpu_cnt)
    assert cnt == min(k, ev), (cnt, k, ev)
    sel = gpu_idx[:cnt]
    assert np.all(gpu_idx[cnt:] == -1)
    assert np.all(np.diff(sel) > 0), "not strictly ascending"
    assert cnt == 0 or (sel[0] >= 0 and sel[-1] < ev), "out of the causal range"
    if ev <= k:
        assert np.array_equal(sel, np.arange(ev))
        return 0
    sc = np.asarray(exact_scores[:ev], dtype=np.float64)
    order = np.lexsort((np.arange(ev), -sc))
    ref = set(order[:k].tolist())
    tau = sc[order[k - 1]]
    band = max(rel_band * abs(tau), float(bf16_ulp(tau)))
    diff = ref.symmetric_difference(set(sel.tolist()))
    for s in diff:
        assert abs(sc[s] - tau) <= band, "entry %d score %r outside the tie band of tau %r" % (
            s, sc[s], tau)
    return len(diff) // 2


def nvfp4_key_scale_index(E_cap, c):
    """Flat byte index, inside one sequence's tiled NVFP4 key-scale area, of (entry, block).

    Tiles of 128 entries; inside a tile, for each 64-element K block, 512 bytes
    ordered [entry % 32][(entry % 128) // 32][block % 4] (the order the block-scaled
    tensor-core MMA reads).  Returns an int array [E_cap][c // 16].
    """
    e = np.arange(E_cap)[:, None]
    blk = np.arange(c // 16)[None, :]
    r = e % 128
    return (e // 128) * (8 * c) + (blk // 4) * 512 + (r % 32) * 16 + (r // 32) * 4 + blk % 4


def nvfp4_scales_to_tiled(rows, E_cap=None):
    """Row-major key scales [..., E, c/16] -> the tiled key-scale layout [..., E_pad, c/16]."""
    rows = np.asarray(rows)
    E, nb = rows.shape[-2], rows.shape[-1]
    E_cap = E_cap or E
    e_pad = (E_cap + 127) // 128 * 128
    idx = nvfp4_key_scale_index(E, nb * 16)
    lead = rows.shape[:-2]
    out = np.zeros(lead + (e_pad * nb,), dtype=rows.dtype)
    flat = rows.reshape(lead + (E * nb,))
    out[..., idx.reshape(-1)] = flat
    return out.reshape(lead + (e_pad, nb))


def nvfp4_scales_from_tiled(tiled, E):
    """Inverse of nvfp4_scales_to_tiled: the first E entries in row-major order."""
    tiled = np.asarray(tiled)
    nb = tiled.shape[-1]
    lead = tiled.shape[:-2]
    flat = tiled.reshape(lead + (-1,))
    idx = nvfp4_key_scale_index(E, nb * 16)
    return flat[..., idx.reshape(-1)].reshape(lead + (E, nb))


class LazyRows:
    """Row access to one sequence of a (large) device tensor, copied to the host in float64 on demand.

    Lets the oracle walk 1M-token inputs without holding them on the host: indexing
    with a slice or an index array returns a numpy float64 array of those rows.
    """

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, key):
        if isinstance(key, np.ndarray):
            key = torch.from_numpy(np.asarray(key, dtype=np.int64)).to(self.t.device)
        return self.t[key].to(torch.float64).cpu().numpy()

    def __len__(self):
        return self.shape[0]
