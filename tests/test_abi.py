"""The C-ABI library loads without a GPU, exports exactly the functions
include/rans_b200.h declares, and answers its host-only queries."""
import ctypes
import os
import re
import subprocess

import pytest

import rans_entropy_coding_b200 as rb
from rans_entropy_coding_b200 import build as rbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("rans_b200.h", "rans_b200_debug.h")]


def declared_functions():
    names = set()
    for path in HEADERS:
        src = re.sub(r"/\*.*?\*/", "", open(path).read(), flags=re.S)
        names |= set(re.findall(r"\b(rans_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return rb.lib()


def test_exports_match_header(lib):
    decl = declared_functions()
    assert len(decl) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", rb.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(set(m for m in re.findall(r"\bT (rans_\w+)", out)))
    assert exported == decl
    for name in decl:
        assert getattr(lib, name) is not None
    assert sorted(n for n, _, _ in rb.SIGNATURES) == decl


def test_status_strings_and_version(lib):
    assert lib.rans_version() >= 100
    for code in range(0, -10, -1):
        assert lib.rans_status_string(code)
    assert lib.rans_status_string(-6).decode().startswith("stream")


def test_stream_counts_and_workspace_sizes(lib):
    ch = rb.Chunking.tiled((16, 192, 68, 120), 4, 64, 64, interleave=32)
    n = 16 * 192 * 68 * 120
    assert rb.rans_num_streams(ch, n) == 3072
    ws = rb.rans_encode_workspace_bytes(ch, n)
    # 3072 slots of 8*16384 + 16*32 + 16 bytes, plus the header and lengths
    assert ws >= 3072 * (8 * 16384 + 528)
    assert rb.rans_decode_workspace_bytes(ch, n) == 256
    assert rb.rans_num_streams(ch, n - 1) == rb.ERR_ARG          # shape mismatch
    c = rb.Chunking.contig(24, interleave=1)
    assert rb.rans_num_streams(c, 1566720) == 24
    assert rb.rans_max_compressed_bytes(c, 1566720) == 8 * 1566720 + 24 * 32
    for W in (2, 4, 8):
        assert rb.rans_num_streams(rb.Chunking.contig(24, interleave=W), 10) == 24
    bad = rb.Chunking.contig(24, interleave=3)
    assert rb.rans_num_streams(bad, 10) == rb.ERR_ARG
    bad = rb.Chunking.contig(24, interleave=16)
    assert rb.rans_num_streams(bad, 10) == rb.ERR_ARG
    nb = rb.Chunking.contig(4, interleave=32, index_block=3000)
    assert rb.rans_num_streams(nb, 10) == rb.ERR_ARG             # not a power of two
    assert rb.rans_num_streams(rb.Chunking.contig(8192, 32, 4096), 1 << 28) == 8192


def test_tables_bound(lib):
    assert rb.rans_tables_bytes(64, 3133) > 256 + 64 * 16 + 4 * 64 * 3132
    assert rb.rans_tables_bytes(0, 10) == 0


def test_cuda_calls_fail_cleanly_without_device(lib):
    """Entry points that need a device return an error code, never crash."""
    t = rb.rans_tables()
    st = lib.rans_encode_with_indexes(None, 0, None, 0, ctypes.byref(t), None, None, 0, None,
                                      None, 0, None)
    assert st == rb.ERR_ARG


def test_workspace_sizes_do_not_truncate(lib):
    """A single stream of 2^30 symbols needs more than 8 GiB of scratch; the
    size must not wrap at 32 bits."""
    big = rb.Chunking.contig(1, 32)
    assert rb.rans_encode_workspace_bytes(big, 1 << 30) >= 8 << 30
    assert rb.rans_max_compressed_bytes(big, 1 << 30) >= 8 << 30
    # the allocation-free encoder refuses it before touching the device
    st = lib.rans_encode_with_indexes_noalloc(None, 0, None, 1 << 30, rb.rans_tables(), big.c,
                                              None, 0, None, None)
    assert st == rb.ERR_CAPACITY
