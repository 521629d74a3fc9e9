"""Pins the oracle's rans32_16 coder ("torch_ans 0.3.0", Usage, variants
table: 32-bit state, 16-bit words, frequencies of at most 15 bits) to values
fixed outside it: hand-worked streams, a closed form for a uniform row, the
quantiser at precision 15 against an independent restatement and a
hand-worked row, brute force (round trip and injectivity), the reduction of
an interleaved stream to a single state, and the information-content size."""
import itertools
import math

import numpy as np
import pytest

import oracle as O
import workloads as WL

from test_oracle_pins import _row_from

R16 = "rans32_16"
E_ROW15 = (np.array([[0, 8192, 24576, 32767, 32768]], dtype=np.int32),
           np.array([5], dtype=np.int32), np.array([-1], dtype=np.int32))


@pytest.mark.parametrize("name", ["r16_e1_two_symbols.txt", "r16_e2_escape_positive.txt",
                                  "r16_e3_renorm_words.txt", "r16_e6_escape_negative.txt"])
def test_hand_worked_streams(golden, name):
    g = golden(name)
    cdf, lengths, offsets = _row_from(g)
    p = int(g["precision"][0])
    sym = np.array([int(v) for v in g["symbols"]], dtype=np.int64)
    rows = np.zeros(sym.size, dtype=np.int32)
    want = bytes(int(b, 16) for b in g["bytes"])
    W = int(g["W"][0])
    got = O.encode_stream(sym, rows, cdf, lengths, offsets, W=W, fmt=R16, precision=p)
    assert got.tobytes() == want
    back = O.decode_stream(np.frombuffer(want, dtype=np.uint8), rows, cdf, lengths, offsets,
                           W=W, fmt=R16, precision=p)
    assert back.tolist() == sym.tolist()


def test_quantiser_hand_worked_at_precision_15(golden):
    g = golden("r16_e4_quantiser.txt")
    pmf = np.array([float(v) for v in g["pmf"]], dtype=np.float32)
    want = [int(v) for v in g["cdf"]]
    assert O.pmf_to_cdf(pmf, precision=int(g["precision"][0])).tolist() == want


def quantise_by_sorted_drain(pmf32, total):
    """Independent restatement of pmf -> quantised CDF summing to ``total``
    (the steal step drains the narrowest buckets wider than 1 in (width,
    index) order, each down to 1 before the next)."""
    p = np.asarray(pmf32, dtype=np.float32).astype(np.float64)
    f = np.floor(p * float(total) + 0.5).astype(np.int64)
    c = np.concatenate([[0], np.cumsum(f)])
    T = int(c[-1])
    c = np.array([(total * int(v)) // T for v in c], dtype=np.int64)
    w = np.diff(c)
    zeros = np.nonzero(w == 0)[0]
    need = zeros.size
    for width, j in sorted((int(w[j]), j) for j in range(w.size) if w[j] > 1):
        if need == 0:
            break
        take = min(width - 1, need)
        w[j] -= take
        need -= take
    assert need == 0
    w[zeros] = 1
    return np.concatenate([[0], np.cumsum(w)]).astype(np.int32)


@pytest.mark.parametrize("prec", [15, 12, 9])
def test_quantiser_matches_independent_restatement(prec):
    rng = np.random.Generator(np.random.PCG64(70 + prec))
    for trial in range(150):
        n = int(rng.integers(2, min(600, (1 << prec) // 2)))
        kind = trial % 3
        if kind == 0:
            p = rng.random(n) ** 8
        elif kind == 1:
            x = np.arange(n) - n / 2
            p = np.exp(-0.5 * (x / rng.uniform(0.3, n / 4)) ** 2)
        else:
            p = rng.random(n)
            p[rng.random(n) < 0.5] = 0.0
            p[0] = 1.0
        p = (p / p.sum()).astype(np.float32)
        want = quantise_by_sorted_drain(p, 1 << prec)
        assert O.pmf_to_cdf(p, precision=prec).tolist() == want.tolist()


def test_gaussian_rows_at_precision_15():
    """Rows of the 64-entry scale table at precision 15 are the independent
    quantiser applied to the same float pmfs as the 16-bit rows."""
    scales = WL.log_spaced_scales(0.11, 256.0, 64)
    c16, l16, o16 = O.build_cdfs_from_scales(scales, 1e-9)
    c15, l15, o15 = O.build_cdfs_from_scales(scales, 1e-9, precision=15)
    assert l15.tolist() == l16.tolist() and o15.tolist() == o16.tolist()
    for r in range(64):
        row = c15[r, :l15[r]].astype(np.int64)
        assert row[0] == 0 and row[-1] == 32768 and (np.diff(row) >= 1).all()
    # the precision-15 pmfs are those of the 16-bit build: recover them from
    # the oracle's own float construction and re-quantise independently
    import scipy.stats
    for r, s in enumerate(scales.astype(np.float64)):
        c = -int(o15[r])
        d = np.abs(np.arange(2 * c + 1) - c).astype(np.float64)
        pmf = scipy.stats.norm.cdf((0.5 - d) / s) - scipy.stats.norm.cdf((-0.5 - d) / s)
        tail = 2.0 * scipy.stats.norm.cdf((-0.5 - c) / s)
        p32 = np.concatenate([pmf, [tail]]).astype(np.float32)
        assert c15[r, :l15[r]].tolist() == quantise_by_sorted_drain(p32, 32768).tolist(), r


def _le16(words):
    return b"".join(int(w).to_bytes(2, "little") for w in words)


def uniform_byte_row_stream(u):
    """Closed form for a precision-8 row of 256 buckets of width 1, offset 0.

    With freq = 1 a symbol op is x -> x 2^8 + u (an 8-bit digit appended
    below the state) and a word leaves whenever x >= 2^24, so the digits are
    packed two per 16-bit word (the earlier symbol in the low byte) behind a
    state that holds one or two digits under the initial state's leading bit
    2^16."""
    n = len(u)
    if n == 0:
        return _le16([0, 1])
    if n % 2 == 0:
        head, rest = [u[0], 1], u[1:]
    else:
        head = [((u[1] << 8) | u[0]) if n > 1 else u[0], 0x100]
        rest = u[2:]
    words = [(rest[i + 1] << 8) | rest[i] for i in range(0, len(rest) - 1, 2)]
    if len(rest) % 2:
        words.append(rest[-1])
    return _le16(head + words)


def test_uniform_row_matches_packing():
    cdf = np.arange(257, dtype=np.int32)[None, :]
    lengths = np.array([257], dtype=np.int32)
    offsets = np.array([0], dtype=np.int32)
    rng = np.random.Generator(np.random.PCG64(12))
    for n in list(range(0, 12)) + [31, 32, 33, 100, 101]:
        u = [int(v) for v in rng.integers(0, 255, size=n)]   # 255 is the escape
        got = O.encode_stream(np.array(u, np.int64), np.zeros(n, np.int32), cdf, lengths,
                              offsets, W=1, fmt=R16, precision=8)
        assert got.tobytes() == uniform_byte_row_stream(u), n
        back = O.decode_stream(got, np.zeros(n, np.int32), cdf, lengths, offsets, W=1,
                               fmt=R16, precision=8)
        assert back.tolist() == u


def test_interleaved_single_symbol_reduces_to_single_state():
    """A W-state stream holding one symbol is lane 0's single-state stream
    with the idle lanes' initial state (2^16) inserted after its state."""
    cdf, lengths, offsets = E_ROW15
    idle = bytes([0, 0, 1, 0])
    for W in (2, 4, 8, 32):
        for s in [-7, -3, -1, 0, 1, 2, 11, 1 << 20]:
            rows = np.zeros(1, dtype=np.int32)
            b1 = O.encode_stream([s], rows, cdf, lengths, offsets, W=1, fmt=R16).tobytes()
            bw = O.encode_stream([s], rows, cdf, lengths, offsets, W=W, fmt=R16).tobytes()
            assert bw[:4] == b1[:4]
            assert bw[4:4 * W] == idle * (W - 1)
            assert bw[4 * W:] == b1[4:]


def test_empty_stream_is_initial_state():
    cdf = np.array([[0, 16384, 32768]], dtype=np.int32)
    one = np.array([3], dtype=np.int32)
    zero = np.array([0], dtype=np.int32)
    for W in (1, 4, 32):
        b = O.encode_stream(np.zeros(0, np.int64), np.zeros(0, np.int32), cdf, one, zero, W=W,
                            fmt=R16)
        assert b.tobytes() == bytes([0, 0, 1, 0]) * W


@pytest.mark.parametrize("W", [1, 4, 32])
def test_brute_force_round_trip_and_injectivity(W):
    cdf, lengths, offsets = E_ROW15
    for n in range(0, 5):
        seen = {}
        for seq in itertools.product(range(-3, 4), repeat=n):
            rows = np.zeros(n, np.int32)
            b = O.encode_stream(np.array(seq, np.int64), rows, cdf, lengths, offsets, W=W,
                                fmt=R16)
            key = b.tobytes()
            assert key not in seen, (seq, seen.get(key))
            seen[key] = seq
            assert len(key) % 2 == 0
            assert tuple(O.decode_stream(b, rows, cdf, lengths, offsets, W=W, fmt=R16)) == seq


def test_size_tracks_information_content():
    """Bytes = (information bits + the flushed state) / 8 up to the finite-
    state coding loss: each op's state lands within a factor (1 + freq / x)
    of the exact x 2^p / freq, and x stays above 2^16 / freq times the
    frequency after renormalisation, so for the workload below the loss is a
    small fraction of the information."""
    t = WL.tiny(seed=5)
    cdfs, lengths, offsets = O.build_cdfs_from_scales(t["scales"], t["tail_mass"], precision=15)
    for W in (1, 32):
        for n in [0, 1, 7, 33, 500, 4096]:
            sym = t["symbols"][:n].astype(np.int64)
            rows = t["indexes"][:n]
            bits = 0.0
            for s, r in zip(sym.tolist(), rows.tolist()):
                maxv = int(lengths[r]) - 2
                v = s - int(offsets[r])
                raw = 0
                if v < 0:
                    raw, v = -2 * v - 1, maxv
                elif v >= maxv:
                    raw, v = 2 * (v - maxv), maxv
                bits += 15 - math.log2(int(cdfs[r, v + 1]) - int(cdfs[r, v]))
                if v == maxv:
                    nb = 0
                    while raw >> (4 * nb):
                        nb += 1
                    bits += 4 * (nb // 15 + 1 + nb)
            b = O.encode_stream(sym, rows, cdfs, lengths, offsets, W=W, fmt=R16, precision=15)
            lo, hi = 2 * W, 4 * W
            slack = 0.01 * bits / 8
            assert bits / 8 + lo - slack - 2 <= b.size <= bits / 8 + hi + slack, (W, n, b.size)


def test_decoder_reports_corruption():
    t = WL.tiny(seed=2)
    cdfs, lengths, offsets = O.build_cdfs_from_scales(t["scales"], t["tail_mass"], precision=15)
    sym = t["symbols"][:300].astype(np.int64)
    rows = t["indexes"][:300]
    for W in (1, 4, 32):
        b = O.encode_stream(sym, rows, cdfs, lengths, offsets, W=W, fmt=R16)
        assert O.decode_stream(b, rows, cdfs, lengths, offsets, W=W, fmt=R16).tolist() == \
            sym.tolist()
        for bad in (b[:-2], np.concatenate([b, np.zeros(2, np.uint8)])):
            with pytest.raises(O.OracleError) as e:
                O.decode_stream(bad, rows, cdfs, lengths, offsets, W=W, fmt=R16)
            assert e.value.status == O.ERR_CORRUPT
    with pytest.raises(O.OracleError) as e:   # 16-bit frequencies are out of range
        O.encode_stream(sym, rows, cdfs, lengths, offsets, W=1, fmt=R16, precision=16)
    assert e.value.status == O.ERR_ARG
    with pytest.raises(O.OracleError):        # 3 interleaved states is not a variant
        O.encode_stream(sym, rows, cdfs, lengths, offsets, W=3, fmt=R16)


def test_extreme_escapes_round_trip():
    cdf, lengths, offsets = E_ROW15
    vals = [-(1 << 59), (1 << 58) + 12345, -(1 << 40), 1 << 45, 2**31 - 1, -2**31,
            2**59 - 7, -(2**59) + 3]
    for W in (1, 32):
        rows = np.zeros(len(vals), np.int32)
        b = O.encode_stream(np.array(vals, np.int64), rows, cdf, lengths, offsets, W=W, fmt=R16)
        assert O.decode_stream(b, rows, cdf, lengths, offsets, W=W, fmt=R16).tolist() == vals
