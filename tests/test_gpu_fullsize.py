"""Byte-exact parity at the configurations' stated sizes, in the launch
configuration the benchmark times: every stream of the 16-image 1080p latent
batch (25,067,520 int32 symbols, 3,072 tiled streams, 32 states per stream)
and of the 2^28-symbol uint8 sweep (8,192 streams, one row index per 4,096
symbols) is coded on the GPU from GPU-built rows and compared byte for byte,
with its offsets, against the oracle's encode of the same arrays on the
oracle's rows; decoding must give back every symbol.  The oracle codes one
stream per call over the host's threads."""
import numpy as np
import pytest
import torch

import rans_entropy_coding_b200 as rb
import workloads as WL
from harness import gpu_encode_decode, gpu_rows, oracle_encode_parallel, oracle_tables

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from rans_entropy_coding_b200 import build
    build.build()
    rb.lib()
    torch.cuda.set_device(0)


def _full_size(w):
    c, l, o = oracle_tables(w)
    gc, gl, go = gpu_rows(w)
    # the rows the benchmark builds on the GPU are the oracle's rows
    assert gl.cpu().numpy().tolist() == l.tolist()
    assert go.cpu().numpy().tolist() == o.tolist()
    gcn = gc.cpu().numpy()
    for r in range(len(l)):
        assert np.array_equal(gcn[r, :l[r]], c[r, :l[r]]), r
    tables = rb.Tables(gc, gl, go, precision=16)
    data, offs, dec, _, _ = gpu_encode_decode(w, tables)
    want, woffs = oracle_encode_parallel(w, c, l, o)
    assert offs.size == woffs.size
    if not np.array_equal(offs, woffs):
        s = int(np.nonzero(offs != woffs)[0][0])
        raise AssertionError("offsets differ first at entry %d" % s)
    assert data.size == want.size
    if not np.array_equal(data, want):
        bad = int(np.nonzero(data != want)[0][0])
        s = int(np.searchsorted(woffs, bad, side="right")) - 1
        raise AssertionError("stream %d differs at byte %d" % (s, bad - int(woffs[s])))
    assert np.array_equal(dec, np.asarray(w["symbols"]).reshape(-1))


def test_batch16_all_streams():
    w = WL.y_batch(n_images=16)
    assert np.asarray(w["symbols"]).size == 25_067_520
    _full_size(w)


def test_sweep_2e28_all_streams():
    w = WL.sweep(log2_n=28)
    assert np.asarray(w["symbols"]).size == 1 << 28
    assert w["chunking"]["n_streams"] == 8192 and w["index_block"] == 4096
    _full_size(w)
