"""GPU parity for alias-coded streams ("torch_ans 0.3.0", Usage, Alias
Coding; Performance Tuning: bucket counts that are powers of two, 1/2/4/8
interleaved states): librans_b200 through its C ABI against the oracle, byte
for byte, in both formats."""
import numpy as np
import pytest
import torch

import oracle as O
import rans_entropy_coding_b200 as rb
import workloads as WL
from harness import gpu_encode_decode, oracle_encode, oracle_tables, tables_from_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from rans_entropy_coding_b200 import build
    build.build()
    rb.lib()
    torch.cuda.set_device(0)


def _check(w):
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o, precision=w["precision"]).prepare_alias()
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode(w, c, l, o)
    assert offs.tolist() == woffs.tolist()
    if not np.array_equal(data, want):
        bad = np.nonzero(data != want)[0][0]
        s = int(np.searchsorted(woffs, bad, side="right")) - 1
        raise AssertionError("stream %d differs at byte %d" % (s, bad - int(woffs[s])))
    assert np.array_equal(dec, np.asarray(w["symbols"]).reshape(-1))
    return tables


def _rows(fmt, W, n_streams=40, per_stream=1500, escapes=True):
    w = WL.r16_rows(n_streams=n_streams, per_stream=per_stream)
    w = dict(w, fmt=fmt, precision=16 if fmt == "rans64" else 15, W=W, alias=True)
    if escapes:
        sym = w["symbols"].copy()
        sym[::131] = 255 + np.arange(sym[::131].size) % 5000    # at and above the range
        sym[7::293] = -1 - np.arange(sym[7::293].size)           # below it
        w["symbols"] = sym
    return w


@pytest.mark.parametrize("fmt", ["rans32_16", "rans64"])
@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_alias_streams_match_oracle(fmt, W):
    """256 rows of 256 buckets (255 symbols and the escape), escapes on both
    sides of the range."""
    _check(_rows(fmt, W))


def test_alias_tables_match_oracle_slots():
    """The device-built remap of every row is the oracle's."""
    w = _rows("rans32_16", 4, n_streams=4, per_stream=64)
    c, l, o = oracle_tables(w)
    tables = tables_from_numpy(c, l, o, precision=15).prepare_alias()
    remap = tables.alias[tables.c.alias_remap_offset:].view(torch.int16).cpu().numpy()
    remap = remap.astype(np.int64) & 0xffff
    for r in (0, 1, 77, 255):
        want = O.alias_build(c[r, :l[r]], 15)[3]
        assert remap[r << 15:(r + 1) << 15].tolist() == want.tolist(), r


def test_alias_hand_worked_row(golden):
    """The hand-worked row and stream of the oracle's pins (precision 4)."""
    g = golden("alias_e2_stream.txt")
    cdf = np.array([[int(v) for v in g["cdf"]]], np.int32)
    w = dict(symbols=np.array([2, 0, 1, 2, 2, 0, 3, 9, -4], np.int32),
             indexes=np.zeros(9, np.int32), chunking=dict(kind="contig", n_streams=1), W=1,
             index_block=1, fmt="rans32_16", precision=4, alias=True,
             pmfs=None)
    c, l, o = cdf, np.array([5], np.int32), np.array([0], np.int32)
    tables = tables_from_numpy(c, l, o, precision=4).prepare_alias()
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want = O.encode_stream(w["symbols"], w["indexes"], c, l, o, W=1, fmt="rans32_16",
                           precision=4, alias=True)
    assert data.tobytes() == want.tobytes()
    assert dec.tolist() == w["symbols"].tolist()
    two = O.encode_stream([2, 0], [0, 0], c, l, o, W=1, fmt="rans32_16", precision=4,
                          alias=True)
    assert two.tobytes() == bytes(int(x, 16) for x in g["bytes"])


def test_alias_argument_errors():
    w = _rows("rans32_16", 4, n_streams=2, per_stream=100, escapes=False)
    c, l, o = oracle_tables(w)
    plain = tables_from_numpy(c, l, o, precision=15)
    sym = torch.from_numpy(w["symbols"]).cuda()
    idx = torch.from_numpy(w["indexes"]).cuda()
    ch = rb.Chunking.contig(2, 4, fmt="rans32_16", alias=True)
    ws = rb.Workspaces(ch, sym.numel())
    # no alias tables prepared
    assert rb.rans_encode_with_indexes(sym, idx, sym.numel(), plain, ch, ws.out, ws.offsets,
                                       ws.enc) == rb.ERR_ARG
    # no 32-way alias coder
    assert rb.rans_num_streams(rb.Chunking.contig(2, 32, fmt="rans32_16", alias=True),
                               10) == rb.ERR_ARG
    # Gaussian rows: bucket counts are not powers of two
    t = WL.tiny(seed=2, n=64)
    gc, gl, go = O.build_cdfs_from_scales(t["scales"], t["tail_mass"])
    with pytest.raises(rb.RansError):
        tables_from_numpy(gc, gl, go).prepare_alias()
