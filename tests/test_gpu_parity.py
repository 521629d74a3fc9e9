"""GPU parity: librans_b200 (through its C ABI) against the CPU oracle.

Integer work, so the bar is exact: CDF tables identical, every stream's bytes
and the offsets identical, decoded symbols identical, on the same seeded
inputs."""
import numpy as np
import pytest
import torch

import oracle as O
import rans_entropy_coding_b200 as rb
import workloads as WL
from harness import (chunking_of, gpu_encode_decode, gpu_rows, oracle_encode, oracle_tables,
                     precision_of, tables_from_numpy)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from rans_entropy_coding_b200 import build
    build.build()
    rb.lib()
    torch.cuda.set_device(0)


def _edge_tiny(W=1, seed=0, dtype=np.int32):
    """The tiny workload plus each row's range edges (centre, centre + 1 --
    the escape with raw value 0 -- and -centre - 1)."""
    w = WL.tiny(seed=seed)
    w["W"] = W
    c, l, o = oracle_tables(w)
    sym = w["symbols"].astype(np.int64)
    rng = np.random.Generator(np.random.PCG64(99))
    for r in range(len(l)):
        cen = -int(o[r])
        for v in (cen, cen + 1, -cen - 1, -cen, 0):
            pos = int(rng.integers(3, sym.size))
            sym[pos] = v
            w["indexes"][pos] = r
    if dtype == np.int16:
        sym = np.clip(sym, -32768, 32767)
    w["symbols"] = sym.astype(dtype)
    return w


def _check_streams(w, exact_tables=True):
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o, precision=precision_of(w))
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode(w, c, l, o)
    assert offs.tolist() == woffs.tolist()
    assert data.size == want.size
    if not np.array_equal(data, want):
        bad = np.nonzero(data != want)[0][0]
        s = int(np.searchsorted(woffs, bad, side="right")) - 1
        raise AssertionError("stream %d differs at byte %d" % (s, bad - int(woffs[s])))
    sym = np.asarray(w["symbols"]).reshape(-1)
    assert np.array_equal(dec, sym)
    return data, offs


# ------------------------------------------------------------- division --
def test_division_is_exact_for_every_frequency():
    f = np.arange(1, 65537, dtype=np.uint64)
    rng = np.random.Generator(np.random.PCG64(5))
    xs = [np.full_like(f, 1 << 31), (f << np.uint64(47)) - np.uint64(1),
          (f << np.uint64(47)) - f, (f << np.uint64(47)) - f - np.uint64(1),
          (f << np.uint64(31)) + np.uint64(12345),
          np.uint64(1 << 31) + (rng.random(f.size) * ((f << np.uint64(47)) - np.uint64(1 << 31))
                                .astype(np.float64)).astype(np.uint64)]
    for x in xs:
        x = np.minimum(x, (f << np.uint64(47)) - np.uint64(1))
        xt = torch.from_numpy(x.astype(np.int64)).cuda()
        ft = torch.from_numpy(f.astype(np.int32)).cuda()
        q = torch.empty_like(xt)
        r = torch.empty_like(ft)
        rb.check(rb.rans_debug_divide(xt, ft, q, r))
        torch.cuda.synchronize()
        assert np.array_equal(q.cpu().numpy().astype(np.uint64), x // f)
        assert np.array_equal(r.cpu().numpy().astype(np.uint64), x % f)


# --------------------------------------------------------------- tables --
@pytest.mark.parametrize("which", ["tiny", "y64", "z", "sweep"])
def test_tables_match_oracle(which):
    w = {"tiny": WL.tiny(), "y64": WL.y_latent(), "z": WL.z_latent(),
         "sweep": WL.sweep(log2_n=16)}[which]
    c, l, o = oracle_tables(w)
    gc, gl, go = gpu_rows(w)
    torch.cuda.synchronize()
    gc, gl, go = gc.cpu().numpy(), gl.cpu().numpy(), go.cpu().numpy()
    assert gl.tolist() == l.tolist()
    assert go.tolist() == o.tolist()
    for r in range(len(l)):
        assert gc[r, :l[r]].tolist() == c[r, :l[r]].tolist(), r


def test_random_pmf_tables_match_oracle():
    rng = np.random.Generator(np.random.PCG64(21))
    K, S = 40, 700
    pmfs = np.zeros((K, S), np.float32)
    lens = rng.integers(1, S, size=K).astype(np.int32)
    tails = np.zeros(K, np.float32)
    for k in range(K):
        n = lens[k]
        kind = k % 4
        if kind == 0:
            p = rng.random(n) ** 10
        elif kind == 1:
            x = np.arange(n) - n / 2
            p = np.exp(-0.5 * (x / rng.uniform(0.2, n / 3)) ** 2)
        elif kind == 2:
            p = rng.random(n)
            p[rng.random(n) < 0.7] = 0
            p[0] = 1
        else:
            p = 1.0 / (np.arange(n) + 1.0) ** 2.5
        p = p / p.sum()
        pmfs[k, :n] = (p * 0.999).astype(np.float32)
        tails[k] = np.float32(0.001 if kind != 3 else 0.0)
    w = dict(pmfs=pmfs, pmf_lengths=lens, tail=tails, offsets=np.zeros(K, np.int32))
    c, l, _ = oracle_tables(w)
    gc, gl, _ = gpu_rows(w)
    gc, gl = gc.cpu().numpy(), gl.cpu().numpy()
    assert gl.tolist() == l.tolist()
    for r in range(K):
        assert gc[r, :l[r]].tolist() == c[r, :l[r]].tolist(), r


def test_bad_rows_are_reported():
    pm = torch.tensor([[0.5, -0.1, 0.6], [0.0, 0.0, 0.0], [np.nan, 0.5, 0.5]],
                      dtype=torch.float32, device="cuda")
    cdfs, lens = rb.Tables.build_from_pmfs(pm, torch.tensor([3, 3, 3], dtype=torch.int32,
                                                            device="cuda"),
                                           torch.zeros(3, device="cuda"))
    assert (lens.cpu() < 0).all()
    sc = torch.tensor([1.0, -1.0], device="cuda")
    lens = torch.empty(2, dtype=torch.int32, device="cuda")
    offs = torch.empty(2, dtype=torch.int32, device="cuda")
    rb.check(rb.rans_gaussian_lengths(sc, 1e-9, lens, offs))
    assert lens[0].item() > 0 and lens[1].item() < 0
    # a non-increasing row is rejected by prepare
    c = torch.tensor([[0, 100, 100, 65536]], dtype=torch.int32, device="cuda")
    with pytest.raises(rb.RansError) as e:
        rb.Tables(c, torch.tensor([4], dtype=torch.int32, device="cuda"),
                  torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert e.value.status == rb.ERR_TABLE


# -------------------------------------------------------------- streams --
@pytest.mark.parametrize("W", [1, 2, 4, 8, 32])
def test_tiny_with_range_edges(W):
    _check_streams(_edge_tiny(W))


def test_tiny_int16_symbols():
    _check_streams(_edge_tiny(32, seed=3, dtype=np.int16))
    _check_streams(_edge_tiny(1, seed=4, dtype=np.int16))


@pytest.mark.parametrize("W", [1, 2, 4, 8, 32])
def test_z_latent(W):
    w = WL.z_latent()
    w["W"] = W
    _check_streams(w)


@pytest.mark.parametrize("W", [1, 32])
def test_y_latent(W):
    _check_streams(WL.y_latent(W=W))


def test_batch_two_images_tiled():
    _check_streams(WL.y_batch(n_images=2))


@pytest.mark.parametrize("W", [1, 2, 4, 8, 32])
def test_batch_small_ragged_tiles(W):
    """Tiles narrower than a warp and a channel group that does not divide C."""
    w = WL.y_batch(n_images=1, cg=5, th=7, tw=11)
    w["W"] = W
    _check_streams(w)


@pytest.mark.parametrize("per", [4, 8, 36, 64, 68, 100, 132, 160, 292, 644])
def test_contiguous_streams_of_every_block_phase(per):
    """Streams of per symbols (a multiple of 4, so the encoder copies its
    inputs in 16-byte blocks of 4 groups): stream lengths of 1 to 21 groups
    put the partial last block in every phase; the last stream is shorter."""
    S = 5
    n = S * per - (4 if per > 4 else 0)
    w = WL.tiny(seed=per, n=n)
    w["W"] = 32
    w["chunking"] = dict(kind="contig", n_streams=S)
    _check_streams(w)


def test_tiled_with_index_blocks():
    w = WL.y_batch(n_images=1, cg=4, th=16, tw=48)
    n = np.asarray(w["symbols"]).size
    rng = np.random.Generator(np.random.PCG64(8))
    w["index_block"] = 64
    w["indexes"] = rng.integers(0, 64, size=n // 64).astype(np.int32)
    _check_streams(w)


def test_sweep_uint8_blocks():
    _check_streams(WL.sweep(log2_n=20, n_streams=32))


@pytest.mark.parametrize("block", [256, 1])
@pytest.mark.parametrize("dtype", [np.uint8, np.int16, np.int32])
def test_chunked_contiguous_streams(dtype, block):
    """Contiguous streams of whole 256-symbol chunks with one row per 256
    symbols or one per symbol (the chunked coders): uint8, int16 and int32
    symbols on rows shorter than the alphabet, and far values, so that
    chunks with escapes are coded again on the escape path."""
    w = WL.sweep(log2_n=16, n_streams=8, block=block)
    w["pmf_lengths"] = np.full(16, 200, dtype=np.int32)
    sym = np.asarray(w["symbols"]).astype(dtype)
    if dtype != np.uint8:
        rng = np.random.Generator(np.random.PCG64(5))
        far = rng.choice(sym.size, sym.size // 200, replace=False)
        big = 30000 if dtype == np.int16 else 1 << 30
        sym[far] = rng.integers(-big, big, far.size).astype(dtype)
    w["symbols"] = sym
    _check_streams(w)


@pytest.mark.parametrize("W", [2, 4, 8])
def test_few_state_interleaves(W):
    """2, 4 and 8 interleaved states per stream, one thread per stream:
    int16 symbols, uint8 symbols with index blocks, tables read from global
    memory (256 rows) and tables staged as starts (256 rows of 257)."""
    _check_streams(_edge_tiny(W, seed=9, dtype=np.int16))
    sw = WL.sweep(log2_n=16, n_streams=8)
    sw["W"] = W
    _check_streams(sw)
    mr = WL.many_rows(n=1 << 15, W=W)
    _check_streams(mr)
    big = dict(WL.r16_rows(n_streams=24, per_stream=777), fmt="rans64", precision=16, W=W)
    _check_streams(big)


def test_sweep_uint8_single_state():
    w = WL.sweep(log2_n=16, n_streams=8)
    w["W"] = 1
    _check_streams(w)


@pytest.mark.parametrize("W", [1, 2, 4, 8, 32])
def test_explicit_chunking_with_empty_streams(W):
    w = WL.tiny(seed=6)
    w["W"] = W
    n = w["symbols"].size
    starts = [0, 0, 5, 5, 37, 100, 100, 1500, n, n]
    w["chunking"] = dict(kind="explicit", starts=starts)
    _check_streams(w)


@pytest.mark.parametrize("W", [1, 2, 4, 8, 32])
def test_more_streams_than_symbols(W):
    w = WL.tiny(seed=7, n=45)
    w["W"] = W
    w["chunking"] = dict(kind="contig", n_streams=64)
    _check_streams(w)


def test_all_escape_row():
    cdf = np.array([[0, 65536] + [0] * 3], dtype=np.int32)
    rng = np.random.Generator(np.random.PCG64(12))
    sym = rng.integers(-2**31, 2**31 - 1, size=3000, dtype=np.int64).astype(np.int32)
    sym[:5] = [0, -1, 1, np.iinfo(np.int32).min, np.iinfo(np.int32).max]
    for W in (1, 32):
        w = dict(symbols=sym, indexes=np.zeros(3000, np.int32),
                 chunking=dict(kind="contig", n_streams=3), W=W, index_block=1)
        c, l, o = cdf, np.array([2], np.int32), np.array([0], np.int32)
        tables = tables_from_numpy(c, l, o)
        data, offs, dec, _, _ = gpu_encode_decode(w, tables)
        want, woffs = oracle_encode(w, c, l, o)
        assert offs.tolist() == woffs.tolist() and np.array_equal(data, want)
        assert np.array_equal(dec, sym)


def test_empty_input():
    w = WL.tiny(n=0)
    for W in (1, 32):
        w["W"] = W
        data, offs = _check_streams(w)
        assert data.size == 8 * W


def test_gpu_built_tables_code_like_oracle_tables():
    w = WL.y_latent(W=32)
    gpu_tables = rb.Tables(*gpu_rows(w))
    data, offs, dec, _, _ = gpu_encode_decode(w, gpu_tables)
    c, l, o = oracle_tables(w)
    want, woffs = oracle_encode(w, c, l, o)
    assert np.array_equal(data, want) and offs.tolist() == woffs.tolist()


# --------------------------------------------------------------- errors --
def _coded(w):
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o)
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    return tables, data, offs


def _decode_status(w, tables, data, offs, indexes=None):
    ch = chunking_of(w)
    idx = torch.from_numpy(np.asarray(w["indexes"] if indexes is None else indexes,
                                      np.int32)).cuda()
    d = torch.from_numpy(data).cuda()
    o = torch.from_numpy(offs.astype(np.int64)).cuda()
    n = np.asarray(w["symbols"]).size
    out = torch.empty(n, dtype=torch.int32, device="cuda")
    ws = rb.aligned_empty(256)
    rb.check(rb.rans_decode_with_indexes(d, o, idx, n, tables, ch, out, ws))
    return rb.rans_get_status(ws)


@pytest.mark.parametrize("W", [1, 32])
def test_decoder_reports_corrupt_streams(W):
    w = WL.y_latent(W=W)
    tables, data, offs = _coded(w)
    assert _decode_status(w, tables, data, offs) == rb.OK
    # a word dropped from the end of stream 3
    o2 = offs.copy()
    o2[4:] -= 4
    d2 = np.concatenate([data[:int(offs[4]) - 4], data[int(offs[4]):]])
    assert _decode_status(w, tables, d2, o2) == rb.ERR_CORRUPT
    # a flipped byte inside stream 5's words
    d3 = data.copy()
    d3[int(offs[5]) + 300] ^= 0x5A
    assert _decode_status(w, tables, d3, offs) == rb.ERR_CORRUPT
    # offsets running past the buffer
    o4 = offs.copy()
    o4[-1] += 64
    assert _decode_status(w, tables, data, o4) == rb.ERR_CORRUPT
    # an index out of range
    bad = np.asarray(w["indexes"]).copy()
    bad[777] = 1000
    assert _decode_status(w, tables, data, offs, bad) == rb.ERR_INDEX


@pytest.mark.parametrize("kind", ["tile", "chunk"])
def test_staged_coders_report_errors(kind):
    """The tile-staged coders (tiled streams) and the chunked coders
    (contiguous streams of whole 256-symbol chunks) record a row index out of
    range (encoder and decoder) and corrupt streams, like the general ones."""
    if kind == "tile":
        w = WL.y_batch(n_images=1)
        w["W"] = 32
    else:
        w = WL.sweep(log2_n=16, n_streams=8, block=256)
        w["symbols"] = np.asarray(w["symbols"]).astype(np.int32)
    tables, data, offs = _coded(w)
    assert _decode_status(w, tables, data, offs) == rb.OK
    o2 = offs.copy()
    o2[4:] -= 4
    d2 = np.concatenate([data[:int(offs[4]) - 4], data[int(offs[4]):]])
    assert _decode_status(w, tables, d2, o2) == rb.ERR_CORRUPT
    d3 = data.copy()
    d3[int(offs[5]) + 300] ^= 0x5A
    assert _decode_status(w, tables, d3, offs) == rb.ERR_CORRUPT
    bad = np.asarray(w["indexes"]).copy()
    bad[min(777, bad.size - 1)] = 1000
    assert _decode_status(w, tables, data, offs, bad) == rb.ERR_INDEX
    sym = torch.from_numpy(np.ascontiguousarray(w["symbols"]).reshape(-1)).cuda()
    _, _, ws = rb.encode_with_indexes(sym, torch.from_numpy(bad.astype(np.int32)).cuda(), tables,
                                      chunking_of(w))
    assert rb.rans_get_status(ws.enc) == rb.ERR_INDEX


def test_encoder_reports_bad_index_and_capacity():
    w = WL.y_latent(W=32)
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o)
    sym = torch.from_numpy(np.asarray(w["symbols"]).reshape(-1)).cuda()
    idx = torch.from_numpy(np.asarray(w["indexes"], np.int32)).cuda()
    ch = chunking_of(w)
    ws = rb.Workspaces(ch, sym.numel())
    bad = idx.clone()
    bad[12345] = -3
    rb.check(rb.rans_encode_with_indexes(sym, bad, sym.numel(), tables, ch, ws.out, ws.offsets,
                                         ws.enc))
    assert rb.rans_get_status(ws.enc) == rb.ERR_INDEX
    small = ws.out[:1000]
    rb.check(rb.rans_encode_with_indexes(sym, idx, sym.numel(), tables, ch, small, ws.offsets,
                                         ws.enc))
    assert rb.rans_get_status(ws.enc) == rb.ERR_CAPACITY
    # a workspace that is too small is refused on the host
    st = rb.rans_encode_with_indexes(sym, idx, sym.numel(), tables, ch, ws.out, ws.offsets,
                                     ws.enc[:1 << 20])
    assert st == rb.ERR_CAPACITY


def _header(tables):
    """The blob header's words (an internal layout: word 16 counts the bitmap
    words the last slot fill handed out, word 17 flags slots that search,
    words 18-20 are a slot fill's own counters, zero between launches)."""
    return tables.blob[:256].view(torch.int32).cpu().numpy()


def test_refreshes_publish_and_clear_build_words():
    """Slot-filling launches count their bitmap words and search flag in build
    words (header words 18, 19; word 20 counts finished blocks) that the last
    block publishes in words 16 and 17 and clears, with no reset between
    launches: repeated refreshes, fused or from rows, report the count of a
    fresh prepare and leave the build words at zero, and the tables still
    code like the oracle."""
    w = WL.y_latent(W=32)
    scales = np.asarray(w["scales"], np.float32)
    tail = w["tail_mass"]
    c, l, o = O.build_cdfs_from_scales(scales, tail)
    tables = tables_from_numpy(c, l, o)
    h0 = _header(tables)
    assert h0[16] > 0 and h0[17] == 0 and not h0[18:21].any()
    K, Lmax = c.shape
    dcd = torch.zeros((K, Lmax), dtype=torch.int32, device="cuda")
    dl = torch.zeros(K, dtype=torch.int32, device="cuda")
    do = torch.zeros(K, dtype=torch.int32, device="cuda")
    dsc = torch.from_numpy(scales).cuda()
    for k in range(6):
        if k % 2 == 0:
            rb.check(rb.rans_tables_refresh_from_scales(dsc, tail, dcd, dl, do, tables))
        else:
            rb.check(rb.rans_tables_refresh(dcd, dl, do, tables))
        h = _header(tables)
        assert rb.rans_get_status(tables.blob) == rb.OK
        assert h[16] == h0[16] and h[17] == 0 and not h[18:21].any(), (k, h[16:21])
    assert np.array_equal(dcd.cpu().numpy(), c)
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode(w, c, l, o)
    assert offs.tolist() == woffs.tolist() and np.array_equal(data, want)
    assert np.array_equal(dec, np.asarray(w["symbols"]).reshape(-1))


def test_refresh_multiplier_cache_follows_the_tail():
    """The fused refresh keeps the Gaussian multiplier of its tail in the
    table header and reuses it only for the same tail: refreshes of one
    table set with alternating tail masses give the oracle's rows, lengths
    and offsets for each tail."""
    w = WL.y_latent(W=32)
    scales = np.asarray(w["scales"], np.float32)
    t0 = w["tail_mass"]
    c, l, o = O.build_cdfs_from_scales(scales, t0)
    tables = tables_from_numpy(c, l, o)
    K, Lmax = c.shape
    dcd = torch.zeros((K, Lmax), dtype=torch.int32, device="cuda")
    dl = torch.zeros(K, dtype=torch.int32, device="cuda")
    do = torch.zeros(K, dtype=torch.int32, device="cuda")
    dsc = torch.from_numpy(scales).cuda()
    for tail in (t0, 1e-6, 1e-6, 1e-4, t0, t0):
        # (a tail other than t0 changes the row lengths: the table set
        # refuses the layout, the rows are still written)
        rb.check(rb.rans_tables_refresh_from_scales(dsc, tail, dcd, dl, do, tables))
        c2, l2, o2 = O.build_cdfs_from_scales(scales, tail)
        gc, gl, go = dcd.cpu().numpy(), dl.cpu().numpy(), do.cpu().numpy()
        assert gl.tolist() == l2.tolist() and go.tolist() == o2.tolist(), tail
        for r in range(K):
            assert gc[r, :l2[r]].tolist() == c2[r, :l2[r]].tolist(), (tail, r)


@pytest.mark.parametrize("W", [1, 32])
def test_slots_without_bitmap_room_search(W):
    """Prepared in a blob with no room for boundary bitmaps, the slots that
    hold three or more boundaries fall back to a search: same symbols."""
    w = WL.y_latent()
    w["W"] = W
    c, l, o = oracle_tables(w)
    full = tables_from_numpy(c, l, o)
    h = _header(full)
    assert h[16] > 0 and h[17] == 0 and full.c.dec_in_smem == 1
    spare = full.c.slot_bytes - 4 * full.c.n_slots
    assert spare >= 4 * h[16]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    tight = rb.Tables(dev(c), dev(l), dev(o), blob_bytes=full.c.blob_bytes - spare)
    assert tight.c.slot_bytes == 4 * tight.c.n_slots
    assert _header(tight)[17] == 1
    data, offs, dec, _, _ = gpu_encode_decode(w, tight)
    want, woffs = oracle_encode(w, c, l, o)
    assert offs.tolist() == woffs.tolist() and np.array_equal(data, want)
    assert np.array_equal(dec, np.asarray(w["symbols"]).reshape(-1))
    # a refresh from the same rows keeps the fallback and the results
    rb.check(rb.rans_tables_refresh(dev(c), dev(l), dev(o), tight))
    assert rb.rans_get_status(tight.blob) == rb.OK and _header(tight)[17] == 1
    _, _, dec2, _, _ = gpu_encode_decode(w, tight)
    assert np.array_equal(dec2, np.asarray(w["symbols"]).reshape(-1))


@pytest.mark.parametrize("W", [1, 32])
def test_tables_too_large_for_shared_memory(W):
    """256 Gaussian rows (0.4 MB of bucket words): both coders read the tables
    from global memory."""
    w = WL.many_rows(W=W)
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o)
    assert tables.c.enc_in_smem == 0 and tables.c.dec_in_smem == 0
    _check_streams(w)


@pytest.mark.parametrize("W", [1, 32])
def test_large_tables_staged_as_starts(W):
    """256 pmf rows of 257 entries (the rans32_16 benchmark shape at the
    64-bit format): too large for bucket words or lookup slots in shared
    memory, so both coders stage the row metadata and 16-bit starts and the
    decoder searches each row."""
    w = WL.r16_rows(n_streams=96, per_stream=1000)
    w = dict(w, fmt="rans64", precision=16, W=W)
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o)
    assert tables.c.enc_in_smem == 2 and tables.c.dec_in_smem == 2
    _check_streams(w)


def test_table_refresh_matches_fresh_prepare():
    """A prepared table set refreshed from new rows of the same lengths codes
    exactly like one prepared from those rows."""
    w = WL.z_latent()
    w["W"] = 32
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o)
    # the same pmf shapes flattened a little: same lengths, other quantised rows
    w2 = dict(w)
    pm = np.asarray(w["pmfs"], np.float64)
    lens = np.asarray(w["pmf_lengths"])
    flat = np.zeros_like(pm)
    for r in range(pm.shape[0]):
        flat[r, :lens[r]] = 1.0 / lens[r]
    w2["pmfs"] = (0.97 * pm + 0.03 * flat).astype(np.float32)
    w2["offsets"] = (np.asarray(w["offsets"]) - 1).astype(np.int32)
    w2["symbols"] = (np.asarray(w["symbols"]) - 1).astype(np.int32)
    c2, l2, o2 = oracle_tables(w2)
    assert np.array_equal(l2, l) and not np.array_equal(c2, c)
    dc2 = torch.from_numpy(np.ascontiguousarray(c2)).cuda()
    dl2 = torch.from_numpy(l2).cuda()
    do2 = torch.from_numpy(o2).cuda()
    rb.check(rb.rans_tables_refresh(dc2, dl2, do2, tables))
    assert rb.rans_get_status(tables.blob) == rb.OK
    data, offs, dec, _, _ = gpu_encode_decode(w2, tables)
    want, woffs = oracle_encode(w2, c2, l2, o2)
    assert offs.tolist() == woffs.tolist() and np.array_equal(data, want)
    assert np.array_equal(dec, np.asarray(w2["symbols"]).reshape(-1))
    # a row of another length is refused on the device
    bad_l = dl2.clone()
    bad_l[3] += 2
    rb.check(rb.rans_tables_refresh(dc2, bad_l, do2, tables))
    assert rb.rans_get_status(tables.blob) == rb.ERR_TABLE


# -------------------------------------------------------- float latents --
def _float_case(W=32, with_means=True, n_images=1, **kw):
    w = WL.y_float(n_images=n_images, W=W, with_means=with_means, **kw)
    c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"])
    rows = O.build_indexes(w["fscales"], w["scales"], w["scale_bound"]).reshape(-1)
    sym = O.quantize(w["y"], w["means"]).reshape(-1)
    wi = dict(w, symbols=sym, indexes=rows)
    return w, wi, (c, l, o)


@pytest.mark.parametrize("K", [1, 2, 64, 65, 66, 300])
def test_build_indexes_matches_oracle(K):
    """Tables of 1 to 300 entries (the 6-step search up to 65 entries, the
    16-step one above), exact table values, values beside them, out of
    range, NaN."""
    t = WL.log_spaced_scales(WL.SCALE_MIN, WL.SCALE_MAX_Y, K).astype(np.float32) if K > 1 \
        else np.float32([WL.SCALE_MIN])
    rng = np.random.Generator(np.random.PCG64(31))
    s = np.concatenate([np.exp(rng.uniform(np.log(1e-3), np.log(1e4), 100000)), t,
                        np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf)),
                        [0.0, -1.0, np.inf, np.nan]]).astype(np.float32)
    got = torch.empty(s.size, dtype=torch.int32, device="cuda")
    rb.check(rb.rans_build_indexes(torch.from_numpy(s).cuda(), torch.from_numpy(t).cuda(),
                                   WL.SCALE_MIN, got))
    assert np.array_equal(got.cpu().numpy(), O.build_indexes(s, t, WL.SCALE_MIN))


@pytest.mark.parametrize("kind", ["dense", "repeated", "wide"])
def test_build_indexes_unusual_tables(kind):
    """Tables the key-count lookup must hand back to the search (a repeated
    entry) or index at fine or coarse key widths (64 entries within 0.1%, or
    spread over 2^-100 .. 2^100): rows equal the oracle's."""
    rng = np.random.Generator(np.random.PCG64(32))
    if kind == "dense":
        t = np.float32(1.0) + np.arange(64, dtype=np.float32) * np.float32(1.6e-5)
    elif kind == "repeated":
        t = WL.log_spaced_scales(WL.SCALE_MIN, WL.SCALE_MAX_Y, 64).astype(np.float32)
        t[20] = t[21]
    else:
        t = np.exp2(np.linspace(-100, 100, 64)).astype(np.float32)
    lo, hi = float(t.min()) / 2, float(t.max()) * 2
    s = np.concatenate([np.exp(rng.uniform(np.log(lo), np.log(hi), 50000)), t,
                        np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf)),
                        [0.0, -1.0, np.inf, np.nan]]).astype(np.float32)
    got = torch.empty(s.size, dtype=torch.int32, device="cuda")
    bound = float(t.min()) / 4
    rb.check(rb.rans_build_indexes(torch.from_numpy(s).cuda(), torch.from_numpy(t).cuda(),
                                   bound, got))
    assert np.array_equal(got.cpu().numpy(), O.build_indexes(s, t, bound))


@pytest.mark.parametrize("W,with_means,n_rows", [(32, True, 64), (32, False, 64), (1, True, 64),
                                                (32, True, 256), (32, True, 128)])
def test_encode_from_scales_matches_oracle(W, with_means, n_rows):
    """Float latents in: the streams equal the oracle's encode of
    build_indexes(scales) and rint(y - mean); decoding gives back
    float32(symbol) + mean exactly."""
    kw = {} if W == 32 else dict(th=17, tw=30)
    # 256 rows: a 16-step table search, and tables read from global memory
    w, wi, (c, l, o) = _float_case(W=W, with_means=with_means, n_rows=n_rows, **kw)
    want, woffs = oracle_encode(wi, c, l, o)
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    tables = tables_from_numpy(c, l, o)
    ch = chunking_of(w)
    table = dev(np.asarray(w["scales"], np.float32))
    out, offs, ws = rb.encode_from_scales(dev(w["y"]), dev(w["fscales"]), table,
                                          w["scale_bound"], tables, ch, means=dev(w["means"]))
    assert rb.rans_get_status(ws.enc) == rb.OK
    total = int(offs[-1].item())
    assert offs.cpu().numpy().astype(np.uint64).tolist() == woffs.tolist()
    assert np.array_equal(out[:total].cpu().numpy(), want)
    vals, wsd = rb.decode_to_values(out[:total], offs, dev(w["fscales"]), table,
                                    w["scale_bound"], tables, ch, means=dev(w["means"]))
    assert rb.rans_get_status(wsd) == rb.OK
    ref = O.dequantize(wi["symbols"], None if w["means"] is None else w["means"].reshape(-1))
    assert np.array_equal(vals.cpu().numpy(), ref)


@pytest.mark.parametrize("with_means", [True, False])
def test_float_tiles_with_far_values(with_means):
    """Float latents on the tile-staged coders (64- and 56-wide tiles): 0.1%
    of the values pushed far outside their rows, so chunks with escapes are
    coded and decoded again on the escape path; streams and values equal the
    oracle's."""
    w = WL.y_float(n_images=2, W=32, with_means=with_means)
    rng = np.random.Generator(np.random.PCG64(77))
    y = np.array(w["y"], copy=True).reshape(-1)
    far = rng.choice(y.size, y.size // 1000, replace=False)
    y[far] += rng.choice(np.float32([-1, 1]), far.size) * rng.uniform(3e3, 3e6, far.size).astype(np.float32)
    w["y"] = y.reshape(w["y"].shape)
    c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"])
    rows = O.build_indexes(w["fscales"], w["scales"], w["scale_bound"]).reshape(-1)
    sym = O.quantize(w["y"], w["means"]).reshape(-1)
    wi = dict(w, symbols=sym, indexes=rows)
    want, woffs = oracle_encode(wi, c, l, o)
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    tables = tables_from_numpy(c, l, o)
    assert tables.c.enc_in_smem == 1 and tables.c.dec_in_smem == 1
    ch = chunking_of(w)
    table = dev(np.asarray(w["scales"], np.float32))
    out, offs, ws = rb.encode_from_scales(dev(w["y"]), dev(w["fscales"]), table,
                                          w["scale_bound"], tables, ch, means=dev(w["means"]))
    assert rb.rans_get_status(ws.enc) == rb.OK
    total = int(offs[-1].item())
    assert offs.cpu().numpy().astype(np.uint64).tolist() == woffs.tolist()
    assert np.array_equal(out[:total].cpu().numpy(), want)
    vals, wsd = rb.decode_to_values(out[:total], offs, dev(w["fscales"]), table,
                                    w["scale_bound"], tables, ch, means=dev(w["means"]))
    assert rb.rans_get_status(wsd) == rb.OK
    ref = O.dequantize(sym, None if w["means"] is None else w["means"].reshape(-1))
    assert np.array_equal(vals.cpu().numpy(), ref)


def test_encode_from_scales_reports_values_out_of_range():
    w, wi, (c, l, o) = _float_case(W=32)
    y = np.array(w["y"], copy=True).reshape(-1)
    y[12345] = np.inf
    tables = tables_from_numpy(c, l, o)
    ch = chunking_of(w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    out, offs, ws = rb.encode_from_scales(dev(y), dev(w["fscales"]),
                                          dev(np.asarray(w["scales"], np.float32)),
                                          w["scale_bound"], tables, ch, means=dev(w["means"]))
    assert rb.rans_get_status(ws.enc) == rb.ERR_RANGE


def test_float_latents_take_the_64_bit_format_only():
    """The float-latent entry points code the 64-bit format at W = 1 or 32;
    rans32_16 or alias chunkings, and 2/4/8 interleaves, are refused."""
    w, wi, (c, l, o) = _float_case(W=32)
    tables = tables_from_numpy(c, l, o)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    y, sc, tab = dev(w["y"]), dev(w["fscales"]), dev(np.asarray(w["scales"], np.float32))
    n = y.numel()
    shape = w["chunking"]["shape"]
    for ch in (rb.Chunking.tiled(shape, 4, 64, 64, 32, fmt="rans32_16"),
               rb.Chunking.tiled(shape, 4, 64, 64, 4, alias=True),
               rb.Chunking.tiled(shape, 4, 64, 64, 4)):
        ws = rb.Workspaces(ch, n)
        st = rb.rans_encode_from_scales(y, None, sc, n, tab, w["scale_bound"], tables, ch,
                                        ws.out, ws.offsets, ws.enc)
        assert st == rb.ERR_ARG
        st = rb.rans_decode_to_values(ws.out, ws.offsets, sc, None, n, tab, w["scale_bound"],
                                      tables, ch, torch.empty(n, device="cuda"), ws.dec)
        assert st == rb.ERR_ARG


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    """The table staging's bounded mbarrier wait, run on a barrier nothing
    completes, records RANS_ERR_TIMEOUT and returns; the next coding call on
    the same context works."""
    import time
    ws = rb.aligned_empty(256)
    t = time.time()
    rb.check(rb.rans_debug_wait_timeout(ws, 2000))
    assert rb.rans_get_status(ws) == rb.ERR_TIMEOUT
    assert time.time() - t < 30
    assert rb.rans_debug_wait_timeout(ws, 0) == rb.ERR_ARG
    _check_streams(_edge_tiny(32, seed=11))


@pytest.mark.parametrize("shape,cg,th,tw,fmt", [
    ((1, 192, 68, 120), 4, 64, 64, "rans32_16"),   # the batch tiles in the 16-bit word format
    ((2, 10, 12, 48), 3, 8, 16, "rans64"),         # narrowest tiles, a partial channel group
    ((1, 6, 20, 96), 2, 4, 40, "rans64"),          # last column 16 wide, 4-row tiles
    ((1, 4, 64, 256), 4, 64, 64, "rans64"),        # every tile full
])
def test_tile_staged_decoder_shapes(shape, cg, th, tw, fmt):
    """Tiled streams whose rows are whole 16-byte units (the decoder stages
    them 4 rows at a time): several tile shapes, both coder formats, and the
    tiny workload's far escapes spread over the tensor."""
    n = int(np.prod(shape))
    w = WL.y_batch(n_images=1, cg=cg, th=th, tw=tw)
    rng = np.random.Generator(np.random.PCG64(41))
    sym = np.asarray(w["symbols"]).reshape(-1)[:n].copy() if n <= np.asarray(
        w["symbols"]).size else np.resize(np.asarray(w["symbols"]).reshape(-1), n)
    idx = np.resize(np.asarray(w["indexes"]), n).astype(np.int32)
    far = rng.random(n) < 0.002
    sym = np.where(far, rng.integers(-2**31, 2**31 - 1, size=n, dtype=np.int64), sym)
    w = dict(w, symbols=sym.astype(np.int32).reshape(shape), indexes=idx,
             chunking=dict(kind="tiled", shape=shape, cg=cg, th=th, tw=tw), W=32, fmt=fmt,
             precision=16 if fmt == "rans64" else 15)
    _check_streams(w)


def test_fused_gaussian_refresh_matches_oracle_rows():
    """rans_tables_refresh_from_scales: the Gaussian rows, lengths and offsets
    of a nudged scale table equal the oracle's, and the refreshed table set
    codes exactly like the oracle on those rows; a scale whose row changes
    length is refused on the device."""
    w = WL.y_latent(W=32)
    scales = np.asarray(w["scales"], np.float32)
    tail = w["tail_mass"]
    c, l, o = O.build_cdfs_from_scales(scales, tail)
    tables = tables_from_numpy(c, l, o)
    # every scale nudged up where its row keeps its length
    s2 = (scales * np.float32(1.0005)).astype(np.float32)
    c2, l2, o2 = O.build_cdfs_from_scales(s2, tail)
    keep = l2 != l
    s2[keep] = scales[keep]
    c2, l2, o2 = O.build_cdfs_from_scales(s2, tail)
    assert np.array_equal(l2, l) and not np.array_equal(c2, c)
    K, Lmax = c.shape
    dcd = torch.full((K, Lmax), -7, dtype=torch.int32, device="cuda")
    dl = torch.zeros(K, dtype=torch.int32, device="cuda")
    do = torch.zeros(K, dtype=torch.int32, device="cuda")
    rb.check(rb.rans_tables_refresh_from_scales(torch.from_numpy(s2).cuda(), tail, dcd, dl, do,
                                                tables))
    assert rb.rans_get_status(tables.blob) == rb.OK
    assert np.array_equal(dcd.cpu().numpy(), c2)
    assert np.array_equal(dl.cpu().numpy(), l2) and np.array_equal(do.cpu().numpy(), o2)
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode(w, c2, l2, o2)
    assert offs.tolist() == woffs.tolist() and np.array_equal(data, want)
    assert np.array_equal(dec, np.asarray(w["symbols"]).reshape(-1))
    # a row whose length changes
    s3 = s2.copy()
    s3[5] *= np.float32(2.0)
    rb.check(rb.rans_tables_refresh_from_scales(torch.from_numpy(s3).cuda(), tail, dcd, dl, do,
                                                tables))
    assert rb.rans_get_status(tables.blob) == rb.ERR_TABLE
