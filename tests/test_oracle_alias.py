"""Pins the oracle's alias coder ("torch_ans 0.3.0", Usage, Alias Coding;
Performance Tuning: the bucket count must be a power of two and push reads a
remap table over the whole 2^precision range): a hand-worked table and
stream, the table's defining properties on random rows, the reduction to the
plain coder on a uniform row, brute-force round trip and injectivity, and
large rows in both formats."""
import itertools

import numpy as np
import pytest

import oracle as O
import workloads as WL

from test_oracle_pins import _row_from


def test_hand_worked_table(golden):
    g = golden("alias_e1_table.txt")
    d, a, b, remap = O.alias_build([int(v) for v in g["cdf"]], int(g["precision"][0]))
    assert d.tolist() == [int(v) for v in g["d"]]
    assert a.tolist() == [int(v) for v in g["a"]]
    assert b.tolist() == [int(v) for v in g["base"]]
    assert remap.tolist() == [int(v) for v in g["remap"]]


def test_hand_worked_stream(golden):
    g = golden("alias_e2_stream.txt")
    cdf, lengths, offsets = _row_from(g)
    p = int(g["precision"][0])
    sym = np.array([int(v) for v in g["symbols"]], dtype=np.int64)
    rows = np.zeros(sym.size, dtype=np.int32)
    want = bytes(int(x, 16) for x in g["bytes"])
    got = O.encode_stream(sym, rows, cdf, lengths, offsets, W=1, fmt="rans32_16", precision=p,
                          alias=True)
    assert got.tobytes() == want
    plain = O.encode_stream(sym, rows, cdf, lengths, offsets, W=1, fmt="rans32_16", precision=p)
    assert plain.tobytes() != want
    back = O.decode_stream(np.frombuffer(want, np.uint8), rows, cdf, lengths, offsets, W=1,
                           fmt="rans32_16", precision=p, alias=True)
    assert back.tolist() == sym.tolist()


def _random_row(rng, n, prec):
    """A strictly increasing row of n + 1 entries from 0 to 2^prec."""
    M = 1 << prec
    cut = np.sort(rng.choice(np.arange(1, M), size=n - 1, replace=False))
    return np.concatenate([[0], cut, [M]]).astype(np.int32)


@pytest.mark.parametrize("n,prec", [(1, 4), (2, 4), (4, 4), (16, 8), (256, 15), (256, 16),
                                    (1024, 12)])
def test_table_properties(n, prec):
    """Every slot holds at most two symbols, its own first; each symbol gets
    exactly its frequency's positions; the remap lists every position once
    and is the inverse of reading a position through its slot."""
    rng = np.random.Generator(np.random.PCG64(n * 31 + prec))
    M, B = 1 << prec, (1 << prec) // n
    for _ in range(5):
        cdf = _random_row(rng, n, prec)
        f = np.diff(cdf)
        d, a, base, remap = O.alias_build(cdf, prec)
        assert ((0 <= d) & (d <= B)).all()
        assert (a[d == B] == np.arange(n)[d == B]).all()
        owned = d.astype(np.int64).copy()
        for j in range(n):
            owned[a[j]] += B - d[j]
        assert owned.tolist() == f.tolist()
        assert sorted(remap.tolist()) == list(range(M))
        for c in range(0, M, max(1, M // 4096)):
            j, o = divmod(c, B)
            if o < d[j]:
                s, r = j, o
            else:
                s, r = int(a[j]), int(base[j]) + o - int(d[j])
            assert r < f[s] and remap[cdf[s] + r] == c


@pytest.mark.parametrize("fmt,prec", [("rans64", 16), ("rans32_16", 15), ("rans32_16", 8)])
def test_uniform_row_reduces_to_plain_coder(fmt, prec):
    """Every frequency equal to the slot width: no aliases, the remap is the
    identity, and the alias stream is the plain stream."""
    n = 64
    cdf = (np.arange(n + 1) * ((1 << prec) // n)).astype(np.int32)[None, :]
    d, a, _, remap = O.alias_build(cdf[0], prec)
    assert (d == (1 << prec) // n).all() and remap.tolist() == list(range(1 << prec))
    lengths, offsets = np.array([n + 1], np.int32), np.array([-20], np.int32)
    rng = np.random.Generator(np.random.PCG64(4))
    for W in (1, 4):
        sym = rng.integers(-30, 60, size=500)           # escapes included
        rows = np.zeros(sym.size, np.int32)
        al = O.encode_stream(sym, rows, cdf, lengths, offsets, W=W, fmt=fmt, precision=prec,
                             alias=True)
        pl = O.encode_stream(sym, rows, cdf, lengths, offsets, W=W, fmt=fmt, precision=prec)
        assert al.tobytes() == pl.tobytes()


@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_brute_force_round_trip_and_injectivity(W):
    cdf = np.array([[0, 7, 8, 13, 16]], np.int32)
    lengths, offsets = np.array([5], np.int32), np.array([-1], np.int32)
    for n in range(0, 5):
        seen = {}
        for seq in itertools.product(range(-3, 4), repeat=n):
            rows = np.zeros(n, np.int32)
            b = O.encode_stream(np.array(seq, np.int64), rows, cdf, lengths, offsets, W=W,
                                fmt="rans32_16", precision=4, alias=True)
            key = b.tobytes()
            assert key not in seen, (seq, seen.get(key))
            seen[key] = seq
            back = O.decode_stream(b, rows, cdf, lengths, offsets, W=W, fmt="rans32_16",
                                   precision=4, alias=True)
            assert tuple(back) == seq


@pytest.mark.parametrize("fmt,prec", [("rans64", 16), ("rans32_16", 15)])
def test_large_rows_round_trip(fmt, prec):
    """The rans32_16 benchmark shape's 256 rows of 257 entries (255 symbols
    and the escape: 256 buckets), with escapes, in both formats."""
    w = WL.r16_rows(n_streams=4, per_stream=3000)
    c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"], precision=prec)
    o = np.asarray(w["offsets"], np.int32)
    sym = w["symbols"][:3000].astype(np.int64)
    sym[::97] = 300 + np.arange(sym[::97].size)           # above the range: bypass
    rows = w["indexes"][:3000]
    for W in (1, 8):
        b = O.encode_stream(sym, rows, c, l, o, W=W, fmt=fmt, precision=prec, alias=True)
        back = O.decode_stream(b, rows, c, l, o, W=W, fmt=fmt, precision=prec, alias=True)
        assert back.tolist() == sym.tolist()
        plain = O.encode_stream(sym, rows, c, l, o, W=W, fmt=fmt, precision=prec)
        assert abs(b.size - plain.size) <= 8 * W + 16      # same information, same size


def test_alias_needs_power_of_two_buckets_and_few_states():
    t = WL.tiny(seed=1, n=64)
    c, l, o = O.build_cdfs_from_scales(t["scales"], t["tail_mass"])
    with pytest.raises(O.OracleError):          # Gaussian rows: 2c + 2 buckets
        O.encode_stream(t["symbols"], t["indexes"], c, l, o, W=1, alias=True)
    cdf = np.array([[0, 7, 8, 13, 16]], np.int32)
    with pytest.raises(O.OracleError):          # no 32-way alias coder
        O.encode_stream([0], [0], cdf, [5], [0], W=32, fmt="rans32_16", precision=4,
                        alias=True)
    with pytest.raises(O.OracleError):
        O.alias_build([0, 5, 10, 16], 4)        # 3 buckets
