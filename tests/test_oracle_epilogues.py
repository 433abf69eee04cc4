"""Pins of the oracle's output epilogues: inverse RoPE on the attention output and the
grouped output projection.

Sources: "DeepSeek V4 结构速览", sections "CSA（c4a 路线）" and "HCA（c128a 路线）"
(inverse RoPE on the last 64 output dims); "DeepSeek-V4 技术解读", section 2.1
(分组输出投影: the output projected in g groups).
"""

import math

import numpy as np
import pytest
import scipy.linalg

from oracle import csa, pipeline

from test_oracle_compositions import mutant

RNG = np.random.default_rng(77)


def test_inverse_rope_undoes_rope_at_the_query_position():
    H, d, d_r = 3, 24, 16
    x = RNG.normal(size=(H, d))
    for t in (0, 1, 77, 4095, 1 << 20):
        y = csa.rope_partial(x, np.full(H, t), d_r, 1e4)
        np.testing.assert_allclose(csa.inverse_rope(y, t, d_r, 1e4), x, atol=1e-9)
    # the leading dims never move, t = 0 is the identity
    z = csa.inverse_rope(x, 12345, d_r, 1e4)
    np.testing.assert_array_equal(z[:, :d - d_r], x[:, :d - d_r])
    np.testing.assert_array_equal(csa.inverse_rope(x, 0, d_r, 1e4), x)


def test_inverse_rope_closed_form_pair_rotation():
    # pair j = 0 has frequency 1: (1, 0) at position t goes to (cos t, -sin t)
    d, d_r = 8, 4
    x = np.zeros((1, d)); x[0, d - d_r] = 1.0
    y = csa.inverse_rope(x, 3, d_r, 1e4)
    np.testing.assert_allclose(y[0, d - d_r:d - d_r + 2], [math.cos(3), -math.sin(3)], atol=1e-15)
    # pair j = 1 rotates at theta^(-2/4) = 1e-2: (0, 1) goes to (sin(0.05), cos(0.05)) at t = 5
    x = np.zeros((1, d)); x[0, d - d_r + 3] = 1.0
    y = csa.inverse_rope(x, 5, d_r, 1e4)
    np.testing.assert_allclose(y[0, d - d_r + 2:], [math.sin(0.05), math.cos(0.05)], atol=1e-15)


def test_inverse_rope_makes_a_single_row_output_relative():
    """One attended row v rotated at its anchor p: the output's rotary part is v rotated by
    p - t (the attention weight multiplies it)."""
    H, d, d_r = 2, 16, 8
    v = RNG.normal(size=(1, d))
    p, t = 40, 57
    row = csa.rope_partial(v, [p], d_r, 1e4)
    q = RNG.normal(size=(H, d))
    sink = np.array([-30.0, -30.0])                 # negligible: the weight of the row is ~1
    o, _ = csa.attend(q, row, sink, 0.1)
    rel = csa.rope_partial(v, [p - t], d_r, 1e4)[0]
    np.testing.assert_allclose(csa.inverse_rope(o, t, d_r, 1e4), np.tile(rel, (H, 1)), atol=1e-9)


def test_grouped_projection_one_group_is_a_plain_matmul():
    T, H, d, d_g = 5, 4, 6, 7
    o = RNG.normal(size=(T, H, d))
    W = RNG.normal(size=(1, d_g, H * d))
    np.testing.assert_allclose(csa.grouped_out_proj(o, W), o.reshape(T, H * d) @ W[0].T,
                               rtol=1e-13)


def test_grouped_projection_is_a_block_diagonal_projection():
    T, H, d, g, d_g = 4, 8, 5, 4, 3
    o = RNG.normal(size=(T, H, d))
    W = RNG.normal(size=(g, d_g, (H // g) * d))
    dense = scipy.linalg.block_diag(*W)             # [g d_g][H d]
    np.testing.assert_allclose(csa.grouped_out_proj(o, W), o.reshape(T, H * d) @ dense.T,
                               rtol=1e-12, atol=1e-12)
    # group i's outputs depend on its own heads only
    o2 = o.copy()
    o2[:, 2:4] += 1.0                               # heads 2, 3 = group 1
    diff = np.abs(csa.grouped_out_proj(o2, W) - csa.grouped_out_proj(o, W)).reshape(T, g, d_g)
    assert np.all(diff[:, 1] > 0) and np.all(diff[:, [0, 2, 3]] == 0)


@pytest.mark.parametrize("fn,old,new", [
    (csa.inverse_rope, "-float(t)", "float(t)"),                              # forward, not inverse
    (csa.grouped_out_proj, "grouped = o.reshape(T, g, K)",
     "grouped = o.reshape(T, K, g).transpose(0, 2, 1)"),                      # heads interleaved
])
def test_epilogue_pins_reject_planted_mistakes(fn, old, new):
    bad = mutant(fn, old, new)
    name = fn.__name__
    orig = getattr(csa, name)
    with pytest.raises(Exception):
        try:
            setattr(csa, name, bad)
            test_inverse_rope_undoes_rope_at_the_query_position()
            test_inverse_rope_closed_form_pair_rotation()
            test_grouped_projection_is_a_block_diagonal_projection()
        finally:
            setattr(csa, name, orig)


def test_decode_composition_applies_inverse_rope_last():
    from test_oracle_compositions import CSA_G, _csa_inputs
    main, index, v, u = _csa_inputs()
    rng = np.random.default_rng(4)
    kw = dict(L=CSA_G["L"], m=CSA_G["m"], d_rope=4, theta=1e4, eps=1e-6, k=3, n_w=CSA_G["n_w"],
              scale=0.3, kv_dtype="f32", idx_dtype="fp8")
    q, qI, w, sink = rng.normal(size=(2, 8)), rng.normal(size=(1, 8)), np.array([0.5]), np.zeros(2)
    a = pipeline.csa_decode_seq(main, index, q, qI, w, sink, **kw)
    b = pipeline.csa_decode_seq(main, index, q, qI, w, sink, inv_rope=True, **kw)
    np.testing.assert_allclose(b["out_f64"], csa.inverse_rope(a["out_f64"], CSA_G["L"] - 1, 4, 1e4),
                               rtol=1e-13)
    np.testing.assert_array_equal(a["idx"], b["idx"])
