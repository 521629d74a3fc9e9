"""GPU parity for the rans32_16 format ("torch_ans 0.3.0", Usage, variants
table: 32-bit state, 16-bit words, frequencies of at most 15 bits):
librans_b200 through its C ABI against the CPU oracle, byte for byte, on the
same seeded inputs; tables built at precision 15 and below identical to the
oracle's."""
import numpy as np
import pytest
import torch

import oracle as O
import rans_entropy_coding_b200 as rb
import workloads as WL
from harness import (gpu_encode_decode, gpu_rows, oracle_encode, oracle_tables,
                     tables_from_numpy)

pytestmark = pytest.mark.gpu

R16 = "rans32_16"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from rans_entropy_coding_b200 import build
    build.build()
    rb.lib()
    torch.cuda.set_device(0)


def _r16(w, W=None, precision=15):
    w = dict(w)
    w["fmt"] = R16
    w["precision"] = precision
    if W is not None:
        w["W"] = W
    return w


def _check_streams(w):
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o, precision=w["precision"])
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode(w, c, l, o)
    assert offs.tolist() == woffs.tolist()
    assert data.size == want.size
    if not np.array_equal(data, want):
        bad = np.nonzero(data != want)[0][0]
        s = int(np.searchsorted(woffs, bad, side="right")) - 1
        raise AssertionError("stream %d differs at byte %d" % (s, bad - int(woffs[s])))
    assert np.array_equal(dec, np.asarray(w["symbols"]).reshape(-1))
    return data, offs


@pytest.mark.parametrize("which,precision", [("tiny", 15), ("y64", 15), ("z", 15),
                                             ("sweep", 15), ("tiny", 12), ("sweep", 9)])
def test_tables_at_precision_match_oracle(which, precision):
    w = {"tiny": WL.tiny(), "y64": WL.y_latent(), "z": WL.z_latent(),
         "sweep": WL.sweep(log2_n=16)}[which]
    w = _r16(w, precision=precision)
    c, l, o = oracle_tables(w)
    gc, gl, go = gpu_rows(w)
    torch.cuda.synchronize()
    gc, gl, go = gc.cpu().numpy(), gl.cpu().numpy(), go.cpu().numpy()
    assert gl.tolist() == l.tolist()
    assert go.tolist() == o.tolist()
    for r in range(len(l)):
        assert gc[r, :l[r]].tolist() == c[r, :l[r]].tolist(), r
        assert c[r, l[r] - 1] == 1 << precision


@pytest.mark.parametrize("W", [1, 2, 4, 8, 32])
def test_tiny_with_escapes(W):
    """4,096 symbols over 8 rows, 1% far outside the rows (bypass pieces of
    up to 8 nibbles) and the int32 extremes."""
    _check_streams(_r16(WL.tiny(seed=3), W=W))


@pytest.mark.parametrize("precision", [15, 13, 12])
def test_contiguous_streams_at_several_precisions(precision):
    w = _r16(WL.many_rows(n=1 << 16, n_rows=16, n_streams=37), precision=precision)
    _check_streams(w)


@pytest.mark.parametrize("W", [1, 2, 8])
def test_z_latent(W):
    _check_streams(_r16(WL.z_latent(), W=W))


def test_y_tiles_two_images():
    """Two images of the batch, 64 x 64 tiles of 4 channels (edge tiles
    partial), one warp per stream."""
    _check_streams(_r16(WL.y_batch(n_images=2)))


def test_uint8_sweep_with_index_blocks():
    w = _r16(WL.sweep(log2_n=20, n_streams=64))
    _check_streams(w)


@pytest.mark.parametrize("W", [1, 4, 32])
def test_large_tables_staged_as_starts(W):
    """The benchmark shape's 256 rows of 257 entries at precision 15: row
    metadata and starts in shared memory, a row search per lookup."""
    w = _r16(WL.r16_rows(n_streams=96, per_stream=1000), W=W)
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o, precision=15)
    assert tables.c.enc_in_smem == 2 and tables.c.dec_in_smem == 2
    _check_streams(w)


def test_streams_of_every_length_phase():
    """Contiguous streams of 1 to 70 symbols (partial first groups of every
    size) and empty streams."""
    rng = np.random.Generator(np.random.PCG64(31))
    lens = list(range(0, 71)) + [0, 0, 129]
    starts = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(starts[-1])
    t = WL.tiny(seed=8, n=n)
    w = _r16(dict(t, chunking=dict(kind="explicit", starts=starts), W=32))
    _check_streams(w)
    w1 = dict(w, W=1)
    _check_streams(w1)
    del rng


def test_stream_lengths_are_even_and_states_flush_to_2_16():
    w = _r16(WL.tiny(seed=4, n=64), W=32)
    data, offs = _check_streams(w)
    assert all(int(b) % 2 == 0 for b in offs)


def test_format_and_precision_must_agree():
    w = WL.tiny(seed=5, n=256)
    c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"], precision=15)
    t15 = tables_from_numpy(c, l, o, precision=15)
    c16, l16, o16 = O.build_cdfs_from_scales(w["scales"], w["tail_mass"])
    t16 = tables_from_numpy(c16, l16, o16)
    sym = torch.from_numpy(w["symbols"]).cuda()
    idx = torch.from_numpy(w["indexes"]).cuda()
    for tab, fmt in ((t15, "rans64"), (t16, R16)):
        ch = rb.Chunking.contig(1, 1, fmt=fmt)
        ws = rb.Workspaces(ch, sym.numel())
        st = rb.rans_encode_with_indexes(sym, idx, sym.numel(), tab, ch, ws.out, ws.offsets,
                                         ws.enc)
        assert st == rb.ERR_ARG
    # rows of precision 15 do not validate as precision-16 tables
    with pytest.raises(rb.RansError):
        tables_from_numpy(c, l, o, precision=16)


def test_truncated_stream_is_corrupt():
    w = _r16(WL.tiny(seed=6, n=2048), W=32)
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o, precision=15)
    data, offs = oracle_encode(w, c, l, o)
    ch = rb.Chunking.contig(1, 32, fmt=R16)
    idx = torch.from_numpy(w["indexes"]).cuda()
    short = torch.from_numpy(data[:-2].copy()).cuda()
    so = torch.tensor([0, data.size - 2], dtype=torch.int64).cuda()
    out = torch.empty(2048, dtype=torch.int32, device="cuda")
    wsd = rb.aligned_empty(256)
    rb.check(rb.rans_decode_with_indexes(short, so, idx, 2048, tables, ch, out, wsd))
    assert rb.rans_get_status(wsd) == rb.ERR_CORRUPT
    # the intact stream decodes
    full = torch.from_numpy(data.copy()).cuda()
    so = torch.tensor([0, data.size], dtype=torch.int64).cuda()
    rb.check(rb.rans_decode_with_indexes(full, so, idx, 2048, tables, ch, out, wsd))
    assert rb.rans_get_status(wsd) == rb.OK
    assert np.array_equal(out.cpu().numpy(), w["symbols"])


def test_table_refresh_at_precision_15():
    """Tables rebuilt in place from new precision-15 rows code like freshly
    prepared ones."""
    scales = WL.log_spaced_scales(WL.SCALE_MIN, WL.SCALE_MAX_Y, 64)
    gs = torch.from_numpy(scales).cuda()
    cdfs, lengths, offsets = rb.Tables.build_from_scales(gs, 1e-9, precision=15)
    tables = rb.Tables(cdfs, lengths, offsets, precision=15)
    rb.check(rb.rans_build_cdfs_from_scales(gs, 1e-9, cdfs, lengths, offsets, precision=15))
    rb.check(rb.rans_tables_refresh(cdfs, lengths, offsets, tables))
    rb.check(rb.rans_get_status(tables.blob))
    w = _r16(WL.y_batch(n_images=1))
    c, l, o = oracle_tables(w)
    assert np.array_equal(cdfs.cpu().numpy()[:, :c.shape[1]], c)
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode(w, c, l, o)
    assert offs.tolist() == woffs.tolist()
    assert np.array_equal(data, want)
    assert np.array_equal(dec, np.asarray(w["symbols"]).reshape(-1))


@pytest.mark.parametrize("fmt,W", [("rans64", 1), ("rans64", 4), ("rans64", 32),
                                   ("rans32_16", 8), ("rans32_16", 32)])
def test_rows_of_two_and_three_entries(fmt, W):
    """Rows with only the escape bucket, one symbol of width 2^p - 1 or of
    width 1 beside the escape, and two halves; symbols in and far out of
    each row's range."""
    prec = 16 if fmt == "rans64" else 15
    M = 1 << prec
    c = np.array([[0, M, 0], [0, M - 1, M], [0, 1, M], [0, M // 2, M]], np.int32)
    l = np.array([2, 3, 3, 3], np.int32)
    o = np.array([0, -1, 5, 100], np.int32)
    rng = np.random.Generator(np.random.PCG64(41))
    n = 5000
    idx = rng.integers(0, 4, size=n).astype(np.int32)
    sym = (o[idx] + rng.integers(-2, 3, size=n)).astype(np.int64)
    sym[::37] = rng.integers(-2**31, 2**31 - 1, size=sym[::37].size)
    w = dict(symbols=sym.astype(np.int32), indexes=idx, W=W, index_block=1, fmt=fmt,
             precision=prec, chunking=dict(kind="contig", n_streams=7))
    tables = tables_from_numpy(c, l, o, precision=prec)
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode(w, c, l, o)
    assert offs.tolist() == woffs.tolist() and np.array_equal(data, want)
    assert np.array_equal(dec, w["symbols"])
