"""Pins the CPU oracle to values fixed outside itself: hand-worked streams,
the page's table size, library routines (scipy's inverse normal and normal
CDF) and an independent restatement of the quantiser's steal step."""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats

import oracle as O
import workloads as WL


def _row_from(g):
    cdf = np.array([[int(v) for v in g["cdf"]]], dtype=np.int32)
    lengths = np.array([cdf.shape[1]], dtype=np.int32)
    offsets = np.array([int(g["offset"][0])], dtype=np.int32)
    return cdf, lengths, offsets


@pytest.mark.parametrize("name", ["e1_two_symbols.txt", "e2_escape_positive.txt",
                                  "e3_renorm_word.txt", "e6_escape_negative.txt",
                                  "e7_two_pieces.txt", "e8_bypass_word.txt",
                                  "e9_two_lanes.txt"])
def test_hand_worked_streams(golden, name):
    g = golden(name)
    cdf, lengths, offsets = _row_from(g)
    sym = np.array([int(v) for v in g["symbols"]], dtype=np.int64)
    rows = np.zeros(sym.size, dtype=np.int32)
    want = bytes(int(b, 16) for b in g["bytes"])
    got = O.encode_stream(sym, rows, cdf, lengths, offsets, W=int(g["W"][0]))
    assert got.tobytes() == want
    back = O.decode_stream(np.frombuffer(want, dtype=np.uint8), rows, cdf, lengths, offsets,
                           W=int(g["W"][0]))
    assert back.tolist() == sym.tolist()


def test_quantiser_hand_worked(golden):
    g = golden("e4_quantiser.txt")
    pmf = np.array([float(v) for v in g["pmf"]], dtype=np.float32)
    want = [int(v) for v in g["cdf"]]
    assert O.pmf_to_cdf(pmf).tolist() == want


def test_interleaved_single_symbol_reduces_to_single_state(golden):
    """A 32-lane stream holding one symbol is lane 0's single-state stream
    with the 31 idle lanes' initial state (2^31) inserted after its state."""
    cdf, lengths, offsets = _row_from(golden("e1_two_symbols.txt"))
    idle = bytes([0, 0, 0, 0x80, 0, 0, 0, 0])
    for s in [-7, -3, -1, 0, 1, 2, 11, 1 << 20]:
        rows = np.zeros(1, dtype=np.int32)
        b1 = O.encode_stream([s], rows, cdf, lengths, offsets, W=1).tobytes()
        b32 = O.encode_stream([s], rows, cdf, lengths, offsets, W=32).tobytes()
        assert b32[:8] == b1[:8]
        assert b32[8:256] == idle * 31
        assert b32[256:] == b1[8:]


@pytest.mark.parametrize("W", [2, 4, 8])
def test_few_state_interleave_reduces_to_single_state(golden, W):
    """The same reduction for 2, 4 and 8 interleaved states ("torch_ans
    0.3.0", Usage, variants table: rans64 interleaves 1, 2, 4 or 8 states)."""
    cdf, lengths, offsets = _row_from(golden("e1_two_symbols.txt"))
    idle = bytes([0, 0, 0, 0x80, 0, 0, 0, 0])
    for s in [-7, -1, 0, 2, 11, 1 << 20]:
        rows = np.zeros(1, dtype=np.int32)
        b1 = O.encode_stream([s], rows, cdf, lengths, offsets, W=1).tobytes()
        bw = O.encode_stream([s], rows, cdf, lengths, offsets, W=W).tobytes()
        assert bw[:8] == b1[:8]
        assert bw[8:8 * W] == idle * (W - 1)
        assert bw[8 * W:] == b1[8:]


def test_interleaved_lanes_are_independent_single_state_streams(golden):
    """With symbols that never renormalise, W interleaved states hold W
    single-state codings of the every-W-th subsequences: lane l's state is
    the single-state stream of symbols l, l + W, ... (E1's row, symbols in
    its coded range, few enough per lane that no word leaves)."""
    cdf, lengths, offsets = _row_from(golden("e1_two_symbols.txt"))
    rng = np.random.Generator(np.random.PCG64(17))
    for W in (2, 4, 8, 32):
        n = 2 * W
        sym = rng.integers(-1, 2, size=n)
        rows = np.zeros(n, dtype=np.int32)
        bw = O.encode_stream(sym, rows, cdf, lengths, offsets, W=W).tobytes()
        assert len(bw) == 8 * W                 # no word left any lane
        for l in range(W):
            b1 = O.encode_stream(sym[l::W], rows[l::W], cdf, lengths, offsets, W=1).tobytes()
            assert len(b1) == 8 and bw[8 * l:8 * l + 8] == b1


def test_empty_stream_is_initial_state():
    cdf = np.array([[0, 32768, 65536]], dtype=np.int32)
    one = np.array([3], dtype=np.int32)
    zero = np.array([0], dtype=np.int32)
    b = O.encode_stream(np.zeros(0, np.int64), np.zeros(0, np.int32), cdf, one, zero, W=1)
    assert b.tobytes() == bytes([0, 0, 0, 0x80, 0, 0, 0, 0])
    b = O.encode_stream(np.zeros(0, np.int64), np.zeros(0, np.int32), cdf, one, zero, W=32)
    assert b.tobytes() == bytes([0, 0, 0, 0x80, 0, 0, 0, 0]) * 32


def test_scale_table_size(golden):
    g = golden("k1_scale_table.txt")
    scales = WL.log_spaced_scales(0.11, 256.0, 64)
    cdfs, lengths, offsets = O.build_cdfs_from_scales(scales, 1e-9)
    assert cdfs.shape == (int(g["rows"][0]), int(g["lmax"][0]))
    assert cdfs.size == int(g["padded_entries"][0])
    assert int(lengths.sum()) == int(g["ragged_entries"][0])
    # the same count from a library inverse normal, not from the oracle
    m = -scipy.special.ndtri(5e-10)
    centers = np.ceil(scales.astype(np.float64) * m).astype(np.int64)
    assert (lengths == 2 * centers + 3).all()
    assert (offsets == -centers).all()
    tiny = WL.log_spaced_scales(0.11, 8.0, 8)
    _, tl, _ = O.build_cdfs_from_scales(tiny, 1e-9)
    assert tl.tolist() == [int(v) for v in g["tiny_lengths"]]


def test_multiplier_matches_library_inverse_normal():
    for t in [1e-9, 1e-6, 1e-3, 0.1]:
        want = -scipy.special.ndtri(t / 2)
        assert abs(O.gaussian_multiplier(t) - want) <= 1e-13 * want


def quantise_by_sorted_drain(pmf32):
    """Independent restatement of pmf -> quantised CDF.

    Rounding and rescaling are written out directly; the steal step uses the
    fact that each empty bucket takes one unit from the narrowest bucket wider
    than 1 (first on ties), and that bucket stays the narrowest until it is
    down to 1 -- so the Z units taken come from buckets in (width, index)
    order, each drained to width 1 before the next is touched."""
    p = np.asarray(pmf32, dtype=np.float32).astype(np.float64)
    f = np.floor(p * 65536.0 + 0.5).astype(np.int64)          # half away from 0
    c = np.concatenate([[0], np.cumsum(f)])
    T = int(c[-1])
    c = np.array([(65536 * int(v)) // T for v in c], dtype=np.int64)
    w = np.diff(c)
    zeros = np.nonzero(w == 0)[0]
    need = zeros.size
    order = sorted((int(w[j]), j) for j in range(w.size) if w[j] > 1)
    for width, j in order:
        if need == 0:
            break
        take = min(width - 1, need)
        w[j] -= take
        need -= take
    assert need == 0
    w[zeros] = 1
    return np.concatenate([[0], np.cumsum(w)]).astype(np.int32)


def test_quantiser_matches_independent_restatement():
    rng = np.random.Generator(np.random.PCG64(7))
    for trial in range(300):
        n = int(rng.integers(2, 600))
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
        assert O.pmf_to_cdf(p).tolist() == quantise_by_sorted_drain(p).tolist()


def test_gaussian_rows_match_library_normal_cdf():
    scales = WL.log_spaced_scales(0.11, 256.0, 64)
    cdfs, lengths, offsets = O.build_cdfs_from_scales(scales, 1e-9)
    for r, s in enumerate(scales.astype(np.float64)):
        c = -int(offsets[r])
        d = np.abs(np.arange(2 * c + 1) - c).astype(np.float64)
        pmf = scipy.stats.norm.cdf((0.5 - d) / s) - scipy.stats.norm.cdf((-0.5 - d) / s)
        tail = 2.0 * scipy.stats.norm.cdf((-0.5 - c) / s)
        p32 = np.concatenate([pmf, [tail]]).astype(np.float32)
        want = quantise_by_sorted_drain(p32)
        assert cdfs[r, :lengths[r]].tolist() == want.tolist(), r


def test_identity_on_already_quantised_pmf():
    rng = np.random.Generator(np.random.PCG64(3))
    for _ in range(50):
        n = int(rng.integers(2, 300))
        cut = np.sort(rng.choice(np.arange(1, 65536), size=n - 1, replace=False))
        widths = np.diff(np.concatenate([[0], cut, [65536]]))
        p = (widths / 65536.0).astype(np.float32)
        assert O.pmf_to_cdf(p).tolist() == np.concatenate([[0], np.cumsum(widths)]).tolist()


def _check_rows(cdfs, lengths, alphabet):
    for r in range(cdfs.shape[0]):
        row = cdfs[r, :lengths[r]].astype(np.int64)
        assert row[0] == 0 and row[-1] == 65536
        assert (np.diff(row) >= 1).all()
        assert lengths[r] == alphabet[r] + 2


def test_table_invariants_on_all_workloads():
    t = WL.tiny()
    c, l, o = O.build_cdfs_from_scales(t["scales"], t["tail_mass"])
    _check_rows(c, l, 2 * (-o) + 1)
    c, l, o = O.build_cdfs_from_scales(WL.log_spaced_scales(0.11, 256.0, 64), 1e-9)
    _check_rows(c, l, 2 * (-o) + 1)
    z = WL.z_latent()
    c, l = O.build_cdfs_from_pmfs(z["pmfs"], z["pmf_lengths"], z["tail"])
    _check_rows(c, l, z["pmf_lengths"])
    sw = WL.sweep(log2_n=16)
    c, l = O.build_cdfs_from_pmfs(sw["pmfs"], sw["pmf_lengths"], sw["tail"])
    _check_rows(c, l, sw["pmf_lengths"])
    assert (l == 258).all()     # 256 symbols + the escape bucket


def test_quantiser_errors():
    with pytest.raises(O.OracleError):
        O.pmf_to_cdf(np.zeros(4, np.float32))           # total 0
    full = np.full(65537, 1.0 / 65536.0, dtype=np.float32)
    full[-1] = 0.0                                      # 65536 unit buckets + 1 empty:
    with pytest.raises(O.OracleError):                  # nothing wider than 1 to steal from
        O.pmf_to_cdf(full)
    assert math.isfinite(O.gaussian_multiplier(1e-9))
