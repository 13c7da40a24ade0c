"""Pins of the oracle's 4-bit weight functions (quantize_int4, pack_int4,
dequantize_int4) against hand-derived values (tests/golden/int4_packing.txt)
and the properties the rule fixes, plus planted mistakes that must fail them.

The pages name 4-bit post-training quantization of an MoE's weights
("Mixture of Experts (MoE)", inferensys.com, inference-optimization
glossary) without a scheme; the scheme is the library's own, stated in
include/moe.h and oracle/moe_oracle.py.
"""
import numpy as np
import pytest

import oracle.moe_oracle as M
from tests._golden import load

G = load("int4_packing.txt")
rng = np.random.default_rng(23)


def test_packing_matches_the_hand_derived_word():
    q = np.tile(np.array(G["codes_k0_to_k7"], np.int64), (128, 32))  # 128 rows of 256 elements
    words = M.pack_int4(q)
    assert words.shape == (128 * 256 // 8,) and (words == G["word"]).all()
    back = M.dequantize_int4(words, np.ones(128 * 2), 128, 256)
    assert back[0, :8].tolist() == G["codes_k0_to_k7"] and (back == q).all()


def test_tiles_hold_128_rows_by_64_elements_row_after_row():
    """Storage order: tile (row // 128, k // 64), then the tile's row, then the
    word; the word of (row 129, elements 64..71) is the first word of row 1 of
    tile (1, 1)."""
    rows, K = 256, 256
    q = np.full((rows, K), -8, np.int64)
    q[129, 64:72] = G["codes_k0_to_k7"]
    words = M.pack_int4(q)
    nz = np.nonzero(words)[0]
    assert nz.tolist() == [((1 * (K // 64) + 1) * 128 + 1) * 8 + 0] and words[nz[0]] == G["word"]
    s = np.arange(rows * 2, dtype=np.float64).reshape(rows, 2)
    st = M.tile_scales(s)
    assert st[(1 * 2 + 1) * 128 + 1] == s[129, 1]


def test_quantization_matches_the_hand_derived_group():
    w = np.zeros((1, 128), np.float32)
    w[0, :4] = G["w_values"]
    q, s = M.quantize_int4(w)
    assert s[0, 0] == G["scale"] and q[0, :4].tolist() == G["q_values"]
    w2 = np.zeros((1, 128), np.float32)
    w2[0, 17] = -G["group_max_2"]
    q2, s2 = M.quantize_int4(w2)
    assert s2[0, 0] == G["scale_2"] and q2[0, 17] == -7


def test_round_trip_bound_scale_bits_and_code_range():
    W = (rng.normal(size=(128, 512)) * np.exp(rng.uniform(-8, 4, size=(128, 1)))).astype(np.float32)
    W[3, 128:256] = 0
    q, s = M.quantize_int4(W)
    assert q.min() >= -7 and q.max() <= 7
    assert (s.view(np.uint32) & 0x7FFFF == 0).all()
    amax = np.abs(W.reshape(128, 4, 128)).max(axis=2)
    assert (s >= amax / 7).all() and (s <= amax / 7 * (1 + 2 ** -4) + 1e-45).all()
    assert s[3, 1] == 0 and (q[3, 128:256] == 0).all()
    Wd = M.dequantize_int4(M.pack_int4(q), M.tile_scales(s), 128, 512)
    assert (np.abs(Wd - W) <= 0.5 * np.repeat(s, 128, axis=1).astype(np.float64) + 1e-45).all()
    # every dequantized value is exact in bfloat16 (at most 8 significant bits)
    mant = (Wd.astype(np.float32).view(np.uint32) & 0xFFFF)
    assert (mant == 0).all()
    assert np.array_equal(Wd.astype(np.float32).astype(np.float64), Wd)


def test_values_on_the_grid_round_trip_exactly():
    s = np.float32(0.046875)  # 1.1b x 2^-5: 2 significant bits
    q = rng.integers(-7, 8, size=(128, 256))
    q[:, ::128] = 7  # each group's largest magnitude is 7 s, so its scale is s again
    W = (q * s).astype(np.float32)
    q2, s2 = M.quantize_int4(W)
    assert (s2 == s).all() and np.array_equal(q2, q)


# ---------------------------------------------------------------- planted mistakes
def _pack_natural_order(q):
    q = np.asarray(q, np.int64)
    rows, K = q.shape
    u = (q + 8).reshape(rows, K // 8, 8).astype(np.uint64)
    w = np.zeros((rows, K // 8), np.uint64)
    for i in range(8):
        w |= u[:, :, i] << (4 * i)
    tiles = w.reshape(rows // 128, 128, K // 64, 8).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(tiles).astype(np.uint32).reshape(-1)


_pack = M.pack_int4


def _pack_row_major(q):
    """Words in plain row order instead of 128 x 64 tiles."""
    rows, K = np.shape(q)
    t = _pack(q).reshape(rows // 128, K // 64, 128, 8).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(t).reshape(-1)


def _scale_rounded_to_nearest(W):
    W = np.asarray(W, np.float32)
    rows, K = W.shape
    g = W.reshape(rows, K // 128, 128)
    s = (np.abs(g).max(axis=2) / np.float32(7)).astype(np.float32)
    u = s.view(np.uint32).astype(np.uint64)
    u = ((u + (1 << 18)) >> 19) << 19
    s = u.astype(np.uint32).view(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(s[:, :, None] > 0, np.rint(g / s[:, :, None]), 0)
    return np.clip(r, -8, 7).astype(np.int8).reshape(rows, K), s


_quantize = M.quantize_int4


def _codes_truncated(W):
    q, s = _quantize(W)
    W = np.asarray(W, np.float32).reshape(q.shape[0], -1, 128)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(s[:, :, None] > 0, np.trunc(W / s[:, :, None]), 0)
    return t.astype(np.int8).reshape(q.shape), s


@pytest.mark.parametrize("name,attr,fn", [("natural nibble order", "pack_int4", _pack_natural_order),
                                          ("words in row order, not tiles", "pack_int4", _pack_row_major),
                                          ("scale rounded to nearest", "quantize_int4", _scale_rounded_to_nearest),
                                          ("codes truncated", "quantize_int4", _codes_truncated)])
def test_planted_mistake_fails_a_pin(name, attr, fn, monkeypatch):
    monkeypatch.setattr(M, attr, fn)
    failed = 0
    for pin in (test_packing_matches_the_hand_derived_word, test_tiles_hold_128_rows_by_64_elements_row_after_row,
                test_quantization_matches_the_hand_derived_group, test_round_trip_bound_scale_bits_and_code_range,
                test_values_on_the_grid_round_trip_exactly):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1, name
