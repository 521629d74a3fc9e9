"""Pins the CPU oracle through properties the mathematics fixes: a closed
form for a uniform row, brute force over tiny inputs (round trip and
injectivity), the information-content size bound, decoder end state and
error reporting, and the stream layout of each chunking."""
import itertools
import math

import numpy as np
import pytest

import oracle as O
import workloads as WL

E_ROW = (np.array([[0, 16384, 49152, 65535, 65536]], dtype=np.int32),
         np.array([5], dtype=np.int32), np.array([-1], dtype=np.int32))


def _le32(words):
    return b"".join(int(w).to_bytes(4, "little") for w in words)


def uniform_unit_row_stream(u):
    """Closed form for a row of 65,536 buckets of width 1 and offset 0.

    With freq = 1 a symbol op is x -> x*2^16 + u (a 16-bit digit appended
    below the state) and a word leaves whenever x >= 2^47, so the stream is a
    plain packing of the digits two per word (the earlier symbol in the low
    half), with the initial state's leading bit 2^31 at the top.  Decoding
    order: u0 first."""
    n = len(u)
    if n == 0:
        return _le32([0x80000000, 0])
    if n % 2 == 0:
        head = [0x80000000 | u[0], 0]
        rest = u[1:]
    else:
        head = [u[0] if n == 1 else (u[1] << 16) | u[0], 0x8000]
        rest = u[2:] if n > 1 else []
    words = [(rest[i + 1] << 16) | rest[i] for i in range(0, len(rest) - 1, 2)]
    if len(rest) % 2:
        words.append(rest[-1])
    return _le32(head + words)


def test_uniform_row_matches_packing():
    cdf = np.arange(65537, dtype=np.int32)[None, :]
    lengths = np.array([65537], dtype=np.int32)
    offsets = np.array([0], dtype=np.int32)
    rng = np.random.Generator(np.random.PCG64(11))
    for n in list(range(0, 12)) + [31, 32, 33, 100, 101]:
        u = [int(v) for v in rng.integers(0, 65535, size=n)]   # 65535 is the escape
        got = O.encode_stream(np.array(u, np.int64), np.zeros(n, np.int32), cdf, lengths,
                              offsets, W=1)
        assert got.tobytes() == uniform_unit_row_stream(u), n
        back = O.decode_stream(got, np.zeros(n, np.int32), cdf, lengths, offsets, W=1)
        assert back.tolist() == u


@pytest.mark.parametrize("W", [1, 4, 32])
def test_brute_force_round_trip_and_injectivity(W):
    cdf, lengths, offsets = E_ROW
    for n in range(0, 5):
        seen = {}
        for seq in itertools.product(range(-3, 4), repeat=n):
            rows = np.zeros(n, np.int32)
            b = O.encode_stream(np.array(seq, np.int64), rows, cdf, lengths, offsets, W=W)
            key = b.tobytes()
            assert key not in seen, (seq, seen.get(key))
            seen[key] = seq
            assert len(key) % 4 == 0
            assert tuple(O.decode_stream(b, rows, cdf, lengths, offsets, W=W)) == seq


def _information_bits(sym, rows, cdfs, lengths, offsets):
    """Sum of -log2(freq/2^16) over symbol ops plus 4 bits per bypass op,
    counted from the op rules (value mapping and piece counting)."""
    bits = 0.0
    nops = 0
    for s, r in zip(sym.tolist(), rows.tolist()):
        Lr = int(lengths[r])
        maxv = Lr - 2
        v = s - int(offsets[r])
        raw = 0
        if v < 0:
            raw, v = -2 * v - 1, maxv
        elif v >= maxv:
            raw, v = 2 * (v - maxv), maxv
        f = int(cdfs[r, v + 1]) - int(cdfs[r, v])
        bits += 16 - math.log2(f)
        nops += 1
        if v == maxv:
            nb = 0
            while raw >> (4 * nb):
                nb += 1
            pieces = nb // 15 + 1 + nb
            bits += 4 * pieces
            nops += pieces
    return bits, nops


@pytest.mark.parametrize("W", [1, 8, 32])
def test_size_within_bound_of_information_content(W):
    t = WL.tiny(seed=5)
    cdfs, lengths, offsets = O.build_cdfs_from_scales(t["scales"], t["tail_mass"])
    rng = np.random.Generator(np.random.PCG64(9))
    for n in [0, 1, 7, 33, 500, 4096]:
        sym = t["symbols"][:n].astype(np.int64)
        rows = t["indexes"][:n]
        if n == 500:
            sym = rng.integers(-3, 4, size=n)
        I, nops = _information_bits(sym, rows, cdfs, lengths, offsets)
        eps = 2e-4 * nops / 8
        b = O.encode_stream(sym, rows, cdfs, lengths, offsets, W=W)
        lo, hi = 4 * W, 8 * W
        assert I / 8 + lo - eps < b.size <= I / 8 + hi + eps, (n, b.size, I / 8)


def test_decoder_reports_corruption():
    t = WL.tiny(seed=2)
    cdfs, lengths, offsets = O.build_cdfs_from_scales(t["scales"], t["tail_mass"])
    sym = t["symbols"][:300].astype(np.int64)
    rows = t["indexes"][:300]
    for W in (1, 32):
        b = O.encode_stream(sym, rows, cdfs, lengths, offsets, W=W)
        with pytest.raises(O.OracleError) as e:
            O.decode_stream(b[:-4], rows, cdfs, lengths, offsets, W=W)
        assert e.value.status == O.ERR_CORRUPT
        with pytest.raises(O.OracleError) as e:
            O.decode_stream(np.concatenate([b, np.zeros(4, np.uint8)]), rows, cdfs, lengths,
                            offsets, W=W)
        assert e.value.status == O.ERR_CORRUPT
        bad = rows.copy()
        bad[5] = 99
        with pytest.raises(O.OracleError) as e:
            O.decode_stream(b, bad, cdfs, lengths, offsets, W=W)
        assert e.value.status == O.ERR_INDEX
        with pytest.raises(O.OracleError) as e:
            O.encode_stream(sym, bad, cdfs, lengths, offsets, W=W)
        assert e.value.status == O.ERR_INDEX


def test_zero_width_bucket_is_an_error():
    cdf = np.array([[0, 100, 100, 65536]], dtype=np.int32)
    with pytest.raises(O.OracleError) as e:
        O.encode_stream(np.array([1], np.int64), np.zeros(1, np.int32), cdf,
                        np.array([4], np.int32), np.array([0], np.int32), W=1)
    assert e.value.status == O.ERR_ZERO_FREQ


def test_extreme_escapes_round_trip():
    """int64 values far outside the row: raw values of up to 60 bits need a
    count of 15 pieces or more, sent as two count pieces."""
    cdf, lengths, offsets = E_ROW
    vals = [-(1 << 59), (1 << 58) + 12345, -(1 << 40), 1 << 45, 2**31 - 1, -2**31,
            2**59 - 7, -(2**59) + 3]
    for W in (1, 32):
        rows = np.zeros(len(vals), np.int32)
        b = O.encode_stream(np.array(vals, np.int64), rows, cdf, lengths, offsets, W=W)
        assert O.decode_stream(b, rows, cdf, lengths, offsets, W=W).tolist() == vals
    with pytest.raises(O.OracleError) as e:
        O.encode_stream(np.array([1 << 61], np.int64), np.zeros(1, np.int32), cdf, lengths,
                        offsets, W=1)
    assert e.value.status == O.ERR_RANGE


def test_contiguous_chunking_partitions():
    for n, S in [(0, 3), (10, 3), (65280, 32), (1566720, 24), (5, 8)]:
        pos = O.stream_positions(n, dict(kind="contig", n_streams=S))
        assert len(pos) == S
        allp = np.concatenate(pos) if pos else np.zeros(0)
        assert allp.tolist() == list(range(n))
        per = -(-n // S)
        assert all(p.size <= per for p in pos)


def test_tiled_chunking_layout():
    shape = (2, 6, 5, 7)
    pos = O.stream_positions(int(np.prod(shape)), dict(kind="tiled", shape=shape, cg=4,
                                                        th=3, tw=4))
    # 2 images x 2 channel groups x 2 tile rows x 2 tile cols
    assert len(pos) == 16
    assert np.sort(np.concatenate(pos)).tolist() == list(range(int(np.prod(shape))))
    b, c, h, w = np.unravel_index(pos[0], shape)
    assert (b == 0).all() and c.tolist()[:12] == [0] * 12 and h[:4].tolist() == [0] * 4
    assert w[:5].tolist() == [0, 1, 2, 3, 0]
    # last stream: image 1, channels 4..5, rows 3..4, cols 4..6
    b, c, h, w = np.unravel_index(pos[-1], shape)
    assert pos[-1].size == 2 * 2 * 3
    assert set(c.tolist()) == {4, 5} and set(h.tolist()) == {3, 4} and set(w.tolist()) == {4, 5, 6}
    # the full-size batch: 16 * 48 * 4 streams of 16384 / 14336 / 1024 / 896
    n = 16 * 192 * 68 * 120
    sizes = [p.size for p in O.stream_positions(
        n, dict(kind="tiled", shape=(16, 192, 68, 120), cg=4, th=64, tw=64))]
    assert len(sizes) == 3072 and sorted(set(sizes)) == [896, 1024, 14336, 16384]


@pytest.mark.parametrize("which", ["tiny", "z", "y1", "y32", "batch", "sweep"])
def test_container_round_trip(which):
    if which == "tiny":
        w = WL.tiny()
        c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"])
    elif which == "z":
        w = WL.z_latent()
        c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"])
        o = w["offsets"]
    elif which in ("y1", "y32"):
        w = WL.y_latent(W=1 if which == "y1" else 32)
        c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"])
    elif which == "batch":
        w = WL.y_batch(n_images=1, th=32, tw=48)
        c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"])
    else:
        w = WL.sweep(log2_n=18, n_streams=13)
        c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"])
        o = w["offsets"]
    sym = np.asarray(w["symbols"]).reshape(-1)
    data, offs = O.encode_with_indexes(sym, w["indexes"], c, l, o, w["chunking"], W=w["W"],
                                       index_block=w["index_block"])
    assert offs[0] == 0 and offs[-1] == data.size and (np.diff(offs.astype(np.int64)) % 4 == 0).all()
    back = O.decode_with_indexes(data, offs, w["indexes"], c, l, o, w["chunking"], sym.size,
                                 W=w["W"], index_block=w["index_block"], dtype=sym.dtype)
    assert (back == sym).all()
