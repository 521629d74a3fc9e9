"""Pins for the oracle's float-latent helpers (build_indexes, quantize,
dequantize): hand-worked values and an independent formulation of the row
rule, no GPU."""
import numpy as np
import pytest

import oracle as O
import workloads as WL

TABLE = np.array([0.11, 0.2, 0.5, 1.0], dtype=np.float32)


def test_build_indexes_hand_values():
    # the row of s is the first table entry >= max(s, bound); the last row
    # when no entry but the last is; NaN counts as the bound
    s = np.array([0.05, 0.11, 0.15, 0.2, 0.21, 0.5, 0.7, 1.0, 5.0, np.nan], np.float32)
    assert O.build_indexes(s, TABLE, 0.11).tolist() == [0, 0, 1, 1, 2, 2, 3, 3, 3, 0]
    # a bound above the first entries moves small scales up
    assert O.build_indexes(np.float32([0.05, 0.3]), TABLE, 0.4).tolist() == [2, 2]


def test_build_indexes_matches_a_binary_search():
    """Against numpy's searchsorted over the first K - 1 entries (left side:
    the first entry >= s), on the 64-row scale table, exact table values and
    values just beside them included."""
    t = WL.log_spaced_scales(WL.SCALE_MIN, WL.SCALE_MAX_Y, WL.N_ROWS_Y).astype(np.float32)
    rng = np.random.Generator(np.random.PCG64(77))
    s = np.concatenate([
        np.exp(rng.uniform(np.log(0.01), np.log(1000.0), 20000)).astype(np.float32), t,
        np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf)),
        np.float32([0.0, -1.0, np.inf])])
    want = np.searchsorted(t[:-1], np.maximum(s, np.float32(WL.SCALE_MIN)), side="left")
    assert np.array_equal(O.build_indexes(s, t, WL.SCALE_MIN), want.astype(np.int32))


def test_quantize_ties_to_even_in_float32():
    y = np.float32([2.5, 3.5, -2.5, -0.5, 0.5, 1.5, 0.49999997, -7.25])
    assert O.quantize(y).tolist() == [2, 4, -2, 0, 0, 2, 0, -7]
    # y - mean is taken in float32: 1e8 - 0.5 rounds back to 1e8 first
    assert O.quantize(np.float32([1e8]), np.float32([0.5])).tolist() == [100000000]
    assert O.quantize(np.float32([10.0]), np.float32([0.5])).tolist() == [10]   # 9.5 -> 10
    assert O.quantize(np.float32([10.0]), np.float32([1.5])).tolist() == [8]    # 8.5 -> 8


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan, 2.0 ** 31, -2.0 ** 31 - 256])
def test_quantize_range_errors(bad):
    with pytest.raises(O.OracleError):
        O.quantize(np.float32([0.0, bad]))


def test_quantize_int32_edges():
    assert O.quantize(np.float32([-2.0 ** 31])).tolist() == [-2 ** 31]
    assert O.quantize(np.float32([2.0 ** 31 - 128])).tolist() == [2 ** 31 - 128]


def test_dequantize_is_float32_addition():
    sym = np.array([3, -2, 100000000], np.int32)
    mean = np.float32([0.1, 0.25, 0.5])
    got = O.dequantize(sym, mean)
    assert got.dtype == np.float32
    assert got.tolist() == [np.float32(3) + np.float32(0.1), np.float32(-1.75),
                            np.float32(100000000.0)]
