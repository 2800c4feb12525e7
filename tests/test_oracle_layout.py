"""Pins of the oracle's shard-packed layouts against element-by-element loops."""
import numpy as np
import pytest

from oracle import layout

RNG = np.random.default_rng(7)


def _bits(shape):
    return RNG.integers(0, 2 ** 16, size=shape, dtype=np.uint16)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_shard_cols_element_map_and_round_trip(t):
    w = _bits((5, 8 * t))
    p = layout.shard_cols(w, t)
    ct = w.shape[1] // t
    for i in range(t):
        for r in range(5):
            for c in range(ct):
                assert p[i, r, c] == w[r, i * ct + c]
    np.testing.assert_array_equal(layout.unshard_cols(p), w)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_shard_rows_is_byte_identical(t):
    w = _bits((8 * t, 6))
    p = layout.shard_rows(w, t)
    assert p.tobytes() == w.tobytes()
    np.testing.assert_array_equal(layout.unshard_rows(p), w)


@pytest.mark.parametrize("t,heads,dh", [(1, 2, 4), (2, 4, 2), (4, 8, 2), (8, 8, 3)])
def test_shard_qkv_puts_each_head_on_its_shard(t, heads, dh):
    D = heads * dh
    w = _bits((3, 3 * D))
    p = layout.shard_qkv(w, t)
    ht = heads // t
    for h in range(heads):
        i, hl = divmod(h, ht)
        for j in range(3):          # q, k, v sections
            for d in range(dh):
                src = j * D + h * dh + d
                dst = j * ht * dh + hl * dh + d
                np.testing.assert_array_equal(p[i][:, dst], w[:, src])
    np.testing.assert_array_equal(layout.unshard_qkv(p), w)


def test_bad_divisibility_raises():
    with pytest.raises(ValueError):
        layout.shard_cols(np.zeros((2, 6)), 4)
    with pytest.raises(ValueError):
        layout.shard_rows(np.zeros((6, 2)), 4)
    with pytest.raises(ValueError):
        layout.shard_qkv(np.zeros((2, 9)), 2)
