"""The allocation-free encode entry point (for callers that cannot allocate
device memory themselves) gives exactly the output of the regular entry
point, on two calls in a row, through the C ABI.  Collected last so that a
run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import rans_entropy_coding_b200 as rb
import workloads as WL

pytestmark = pytest.mark.gpu


def test_noalloc_encode_matches_regular_encode():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from rans_entropy_coding_b200 import build
    build.build()
    torch.cuda.set_device(0)
    w = WL.y_batch(n_images=1)                      # 1,566,720 symbols, 192 streams
    sym = torch.from_numpy(np.asarray(w["symbols"]).reshape(-1)).cuda()
    idx = torch.from_numpy(w["indexes"]).cuda()
    tables = rb.Tables.from_scales(torch.from_numpy(w["scales"]).cuda())
    ch = rb.Chunking.from_spec(w["chunking"], 32)
    out, offs, ws = rb.encode_with_indexes(sym, idx, tables, ch)
    assert rb.rans_get_status(ws.enc) == rb.OK
    total = int(offs[-1].item())
    want_bytes = out[:total].clone()
    want_offs = offs.clone()
    for _ in range(2):
        out2 = torch.zeros(rb.rans_max_compressed_bytes(ch, sym.numel()), dtype=torch.uint8,
                           device="cuda")
        offs2 = torch.zeros_like(offs)
        rb.check(rb.rans_encode_with_indexes_noalloc(sym, idx, sym.numel(), tables, ch, out2,
                                                     offs2), "noalloc encode")
        torch.cuda.synchronize()
        assert torch.equal(offs2, want_offs)
        assert torch.equal(out2[:total], want_bytes)
    # device errors are marked in the outputs (stream_offsets[S] = UINT64_MAX,
    # -1 read as int64); the next good call, which starts from a cleared
    # status word in the shared array, gives the regular result again
    bad = idx.clone()
    bad[4321] = 64                                  # rows are 0..63
    small = torch.zeros(total // 2, dtype=torch.uint8, device="cuda")
    for case in ("index", "capacity"):
        offs3 = torch.zeros_like(offs)
        if case == "index":
            st = rb.rans_encode_with_indexes_noalloc(sym, bad, sym.numel(), tables, ch, out2,
                                                     offs3)
        else:
            st = rb.rans_encode_with_indexes_noalloc(sym, idx, sym.numel(), tables, ch, small,
                                                     offs3)
        rb.check(st, "noalloc encode (%s error)" % case)
        torch.cuda.synchronize()
        assert int(offs3[-1].item()) == -1, case
        out4 = torch.zeros_like(out2)
        offs4 = torch.zeros_like(offs)
        rb.check(rb.rans_encode_with_indexes_noalloc(sym, idx, sym.numel(), tables, ch, out4,
                                                     offs4), "noalloc encode after an error")
        torch.cuda.synchronize()
        assert torch.equal(offs4, want_offs), case
        assert torch.equal(out4[:total], want_bytes), case
    # past the fixed workspace size: refused with a clear error, nothing launched
    big = rb.Chunking.contig(1, 32)
    st = rb.lib().rans_encode_with_indexes_noalloc(None, 0, None, 1 << 30, tables.c, big.c, None,
                                                   0, None, None)
    assert st == rb.ERR_CAPACITY
