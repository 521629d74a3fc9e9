"""The correctness oracle: a plain, slow, single-threaded CPU restatement of
indexed 64-bit rANS coding (C core in rans_oracle.c, stream layout here in
numpy).

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
bench's ``cpu_baseline`` / ``--impl reference`` legs may import this package.
It shares no code with ``rans_entropy_coding_b200`` and never imports it.

Sources (page title, then section):
  * "kompressor" README -- Why: the symbol array is cut into independent
    chunks with no cross-chunk dependency (the rayon parallelism); Getting
    Started: "chunks=24".
  * "torch_ans 0.3.0" -- Low-level API (cdfs, cdfs_sizes, offsets, one index
    per symbol); rans_stream_to_byte_strings (streams serialised as byte
    strings).

Readings where the pages are silent:
  * contiguous chunking: stream k covers [k*ceil(N/S), min((k+1)*ceil(N/S), N));
  * tiled chunking of an NCHW tensor: streams ordered (b, channel group,
    tile row, tile column); symbols inside a stream in (channel, row, column)
    order; edge tiles are partial;
  * one index per ``index_block`` consecutive elements of the flattened
    tensor: element p uses indexes[p // index_block];
  * the container is the streams' bytes concatenated, with uint64 offsets
    (S + 1 entries, offsets[0] = 0).

Parity status: every function here is pinned (tests/test_oracle_*.py).
Byte-exactness against CompressAI itself is unpinned: no CompressAI output is
available to compare against.
"""
import ctypes
import os

import numpy as np

from . import build as _build

OK = 0
ERR_ARG = -1
ERR_INDEX = -2
ERR_ZERO_FREQ = -3
ERR_RANGE = -4
ERR_CAPACITY = -5
ERR_CORRUPT = -6

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L.orc_pmf_to_cdf.argtypes = [P, ctypes.c_int, P]
        L.orc_pmf_to_cdf.restype = ctypes.c_int
        L.orc_pmf_to_cdf_prec.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
        L.orc_pmf_to_cdf_prec.restype = ctypes.c_int
        L.orc_build_cdfs_from_scales_prec.argtypes = [P, ctypes.c_int, f64, ctypes.c_int, P,
                                                      ctypes.c_int, P, P]
        L.orc_build_cdfs_from_scales_prec.restype = ctypes.c_int
        L.orc_build_cdfs_from_pmfs_prec.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P,
                                                    ctypes.c_int, P, ctypes.c_int, P]
        L.orc_build_cdfs_from_pmfs_prec.restype = ctypes.c_int
        L.orc_encode_stream16.argtypes = [P, P, i64, P, ctypes.c_int, ctypes.c_int, P, P,
                                          ctypes.c_int, ctypes.c_int, P, i64]
        L.orc_encode_stream16.restype = i64
        L.orc_decode_stream16.argtypes = [P, i64, P, i64, P, ctypes.c_int, ctypes.c_int, P, P,
                                          ctypes.c_int, ctypes.c_int, P]
        L.orc_decode_stream16.restype = ctypes.c_int
        L.orc_alias_build.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P, P]
        L.orc_alias_build.restype = ctypes.c_int
        L.orc_encode_stream_alias.argtypes = [P, P, i64, P, ctypes.c_int, ctypes.c_int, P, P,
                                              ctypes.c_int, ctypes.c_int, P, i64]
        L.orc_encode_stream_alias.restype = i64
        L.orc_decode_stream_alias.argtypes = [P, i64, P, i64, P, ctypes.c_int, ctypes.c_int, P,
                                              P, ctypes.c_int, ctypes.c_int, P]
        L.orc_decode_stream_alias.restype = ctypes.c_int
        L.orc_gaussian_multiplier.argtypes = [f64]
        L.orc_gaussian_multiplier.restype = f64
        L.orc_gaussian_center.argtypes = [ctypes.c_float, f64, P]
        L.orc_gaussian_center.restype = ctypes.c_int
        L.orc_build_cdfs_from_scales.argtypes = [P, ctypes.c_int, f64, P, ctypes.c_int, P, P]
        L.orc_build_cdfs_from_scales.restype = ctypes.c_int
        L.orc_build_cdfs_from_pmfs.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P,
                                               ctypes.c_int, P]
        L.orc_build_cdfs_from_pmfs.restype = ctypes.c_int
        L.orc_encode_stream.argtypes = [P, P, i64, P, ctypes.c_int, ctypes.c_int, P, P,
                                        ctypes.c_int, P, i64]
        L.orc_encode_stream.restype = i64
        L.orc_decode_stream.argtypes = [P, i64, P, i64, P, ctypes.c_int, ctypes.c_int, P, P,
                                        ctypes.c_int, P]
        L.orc_decode_stream.restype = ctypes.c_int
        del i32
        _lib = L
    return _lib


class OracleError(RuntimeError):
    def __init__(self, status, what=""):
        super().__init__("oracle status %d %s" % (status, what))
        self.status = status


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


# ------------------------------------------------------------------ tables --
def pmf_to_cdf(pmf, precision=16):
    """pmf (tail mass last) -> quantised cdf row of len(pmf) + 1 entries,
    summing to 2^precision."""
    p = np.ascontiguousarray(pmf, dtype=np.float32)
    out = np.zeros(p.size + 1, dtype=np.int32)
    if precision == 16:
        st = lib().orc_pmf_to_cdf(_ptr(p), p.size, _ptr(out))
    else:
        st = lib().orc_pmf_to_cdf_prec(_ptr(p), p.size, precision, _ptr(out))
    if st:
        raise OracleError(st, "pmf_to_cdf")
    return out


def gaussian_multiplier(tail_mass=1e-9):
    return lib().orc_gaussian_multiplier(tail_mass)


def gaussian_center(scale, tail_mass=1e-9):
    c = np.zeros(1, dtype=np.int32)
    st = lib().orc_gaussian_center(ctypes.c_float(scale), tail_mass, _ptr(c))
    if st:
        raise OracleError(st, "gaussian_center")
    return int(c[0])


def build_cdfs_from_scales(scales, tail_mass=1e-9, Lmax=None, precision=16):
    """Gaussian rows -> (cdfs[K, Lmax] int32, lengths[K], offsets[K]); rows sum
    to 2^precision."""
    s = np.ascontiguousarray(scales, dtype=np.float32)
    K = s.size
    if Lmax is None:
        Lmax = max(2 * gaussian_center(float(v), tail_mass) + 3 for v in s)
    cdfs = np.zeros((K, Lmax), dtype=np.int32)
    lengths = np.zeros(K, dtype=np.int32)
    offsets = np.zeros(K, dtype=np.int32)
    st = lib().orc_build_cdfs_from_scales_prec(_ptr(s), K, tail_mass, precision, _ptr(cdfs),
                                               Lmax, _ptr(lengths), _ptr(offsets))
    if st:
        raise OracleError(st, "build_cdfs_from_scales")
    return cdfs, lengths, offsets


def build_cdfs_from_pmfs(pmfs, pmf_lengths, tail_mass, Lmax=None, precision=16):
    """pmf rows -> (cdfs[K, Lmax] int32, lengths[K]); rows sum to 2^precision."""
    p = np.ascontiguousarray(pmfs, dtype=np.float32)
    K, S = p.shape
    pl = np.ascontiguousarray(pmf_lengths, dtype=np.int32)
    tm = np.ascontiguousarray(tail_mass, dtype=np.float32)
    if Lmax is None:
        Lmax = int(pl.max()) + 2
    cdfs = np.zeros((K, Lmax), dtype=np.int32)
    lengths = np.zeros(K, dtype=np.int32)
    st = lib().orc_build_cdfs_from_pmfs_prec(_ptr(p), K, S, _ptr(pl), _ptr(tm), precision,
                                             _ptr(cdfs), Lmax, _ptr(lengths))
    if st:
        raise OracleError(st, "build_cdfs_from_pmfs")
    return cdfs, lengths


# ----------------------------------------------------------------- streams --
# Coder formats ("torch_ans 0.3.0", Usage, variants table): "rans64" has a
# 64-bit state, 32-bit words and rows summing to 2^16; "rans32_16" a 32-bit
# state, 16-bit words and rows summing to 2^precision, precision <= 15.
FORMATS = ("rans64", "rans32_16")


def _precision(fmt, precision):
    return precision if precision is not None else (16 if fmt == "rans64" else 15)


def alias_build(cdf_row, precision):
    """Alias table of one row (its cdf entries, bucket count a power of two):
    (d, a, base, remap) as int32 arrays."""
    c = np.ascontiguousarray(cdf_row, dtype=np.int32)
    n = c.size - 1
    d, a, b = (np.zeros(max(n, 1), np.int32) for _ in range(3))
    remap = np.zeros(1 << precision, np.int32)
    st = lib().orc_alias_build(_ptr(c), c.size, precision, _ptr(d), _ptr(a), _ptr(b),
                               _ptr(remap))
    if st:
        raise OracleError(st, "alias_build")
    return d[:n], a[:n], b[:n], remap


def encode_stream(symbols, rows, cdfs, lengths, offsets, W=1, fmt="rans64", precision=None,
                  alias=False):
    """Codes one stream; returns its bytes as a uint8 array.  alias: the
    alias-coded variant (bucket counts powers of two; W = 1, 2, 4 or 8)."""
    s = np.ascontiguousarray(symbols, dtype=np.int64)
    r = np.ascontiguousarray(rows, dtype=np.int32)
    c = np.ascontiguousarray(cdfs, dtype=np.int32)
    ln = np.ascontiguousarray(lengths, dtype=np.int32)
    of = np.ascontiguousarray(offsets, dtype=np.int32)
    K, Lmax = c.shape
    cap = 8 * W + 16 + 8 * s.size + 64
    out = np.zeros(cap, dtype=np.uint8)
    if alias:
        if fmt not in FORMATS:
            raise ValueError("unknown format %r" % fmt)
        n = lib().orc_encode_stream_alias(_ptr(s), _ptr(r), s.size, _ptr(c), K, Lmax, _ptr(ln),
                                          _ptr(of), _precision(fmt, precision), W, _ptr(out),
                                          cap)
    elif fmt == "rans64":
        n = lib().orc_encode_stream(_ptr(s), _ptr(r), s.size, _ptr(c), K, Lmax, _ptr(ln),
                                    _ptr(of), W, _ptr(out), cap)
    elif fmt == "rans32_16":
        n = lib().orc_encode_stream16(_ptr(s), _ptr(r), s.size, _ptr(c), K, Lmax, _ptr(ln),
                                      _ptr(of), 15 if precision is None else precision, W,
                                      _ptr(out), cap)
    else:
        raise ValueError("unknown format %r" % fmt)
    if n < 0:
        raise OracleError(int(n), "encode_stream")
    return out[:n].copy()


def decode_stream(data, rows, cdfs, lengths, offsets, W=1, fmt="rans64", precision=None,
                  alias=False):
    """Decodes len(rows) symbols of one stream; returns int64 symbols."""
    d = np.ascontiguousarray(data, dtype=np.uint8)
    r = np.ascontiguousarray(rows, dtype=np.int32)
    c = np.ascontiguousarray(cdfs, dtype=np.int32)
    ln = np.ascontiguousarray(lengths, dtype=np.int32)
    of = np.ascontiguousarray(offsets, dtype=np.int32)
    K, Lmax = c.shape
    out = np.zeros(r.size, dtype=np.int64)
    if alias:
        if fmt not in FORMATS:
            raise ValueError("unknown format %r" % fmt)
        st = lib().orc_decode_stream_alias(_ptr(d), d.size, _ptr(r), r.size, _ptr(c), K, Lmax,
                                           _ptr(ln), _ptr(of), _precision(fmt, precision), W,
                                           _ptr(out))
    elif fmt == "rans64":
        st = lib().orc_decode_stream(_ptr(d), d.size, _ptr(r), r.size, _ptr(c), K, Lmax,
                                     _ptr(ln), _ptr(of), W, _ptr(out))
    elif fmt == "rans32_16":
        st = lib().orc_decode_stream16(_ptr(d), d.size, _ptr(r), r.size, _ptr(c), K, Lmax,
                                       _ptr(ln), _ptr(of), 15 if precision is None else precision,
                                       W, _ptr(out))
    else:
        raise ValueError("unknown format %r" % fmt)
    if st:
        raise OracleError(st, "decode_stream")
    return out


# ---------------------------------------------------------------- chunking --
def num_streams(n, chunking):
    """Number of streams of a chunking of n elements."""
    kind = chunking["kind"]
    if kind == "contig":
        return int(chunking["n_streams"])
    if kind == "explicit":
        return len(chunking["starts"]) - 1
    if kind == "tiled":
        B, C, H, Wd = (int(v) for v in chunking["shape"])
        cg, th, tw = int(chunking["cg"]), int(chunking["th"]), int(chunking["tw"])
        return B * (-(-C // cg)) * (-(-H // th)) * (-(-Wd // tw))
    raise ValueError("unknown chunking kind %r" % kind)


def stream_position(n, chunking, k):
    """Flat element positions of stream k, in coding order.

    ``chunking`` is a dict: {"kind": "contig", "n_streams": S} |
    {"kind": "explicit", "starts": [S+1 offsets]} |
    {"kind": "tiled", "shape": (B, C, H, W), "cg": g, "th": th, "tw": tw}.
    """
    kind = chunking["kind"]
    if kind == "contig":
        S = int(chunking["n_streams"])
        per = -(-n // S) if S > 0 else 0
        a = min(k * per, n)
        b = min((k + 1) * per, n)
        return np.arange(a, b, dtype=np.int64)
    if kind == "explicit":
        st = np.asarray(chunking["starts"], dtype=np.int64)
        return np.arange(st[k], st[k + 1], dtype=np.int64)
    if kind == "tiled":
        B, C, H, Wd = (int(v) for v in chunking["shape"])
        cg, th, tw = int(chunking["cg"]), int(chunking["th"]), int(chunking["tw"])
        assert B * C * H * Wd == n
        ng, nty, ntx = -(-C // cg), -(-H // th), -(-Wd // tw)
        # streams are numbered (b, channel group, tile row, tile column)
        b, r = divmod(k, ng * nty * ntx)
        g, r = divmod(r, nty * ntx)
        ty, tx = divmod(r, ntx)
        c0, h0, w0 = g * cg, ty * th, tx * tw
        cs = np.arange(c0, min(c0 + cg, C), dtype=np.int64)
        hs = np.arange(h0, min(h0 + th, H), dtype=np.int64)
        ws = np.arange(w0, min(w0 + tw, Wd), dtype=np.int64)
        pos = ((b * C + cs[:, None, None]) * H + hs[None, :, None]) * Wd + ws[None, None, :]
        return pos.reshape(-1)
    raise ValueError("unknown chunking kind %r" % kind)


def stream_positions(n, chunking):
    """Flat element positions of every stream, in coding order (a list with
    one array per stream)."""
    return [stream_position(n, chunking, k) for k in range(num_streams(n, chunking))]


def _rows_for(positions, indexes, index_block):
    return np.asarray(indexes, dtype=np.int32)[positions // index_block]


def encode_with_indexes(symbols, indexes, cdfs, lengths, offsets, chunking, W=1,
                        index_block=1, streams=None, fmt="rans64", precision=None, alias=False):
    """Container encode: returns (bytes uint8[total], offsets uint64[S+1]).

    ``streams`` optionally restricts the work to a subset of stream ids; the
    result then holds those streams only (offsets over the subset)."""
    flat = np.asarray(symbols).reshape(-1)
    pos = stream_positions(flat.size, chunking)
    ids = range(len(pos)) if streams is None else streams
    parts, offs = [], [0]
    for k in ids:
        p = pos[k]
        b = encode_stream(flat[p].astype(np.int64), _rows_for(p, indexes, index_block),
                          cdfs, lengths, offsets, W, fmt, precision, alias)
        parts.append(b)
        offs.append(offs[-1] + b.size)
    data = np.concatenate(parts) if parts else np.zeros(0, dtype=np.uint8)
    return data, np.asarray(offs, dtype=np.uint64)


def decode_with_indexes(data, stream_offsets, indexes, cdfs, lengths, offsets, chunking,
                        n, W=1, index_block=1, dtype=np.int32, fmt="rans64", precision=None,
                        alias=False):
    """Container decode of n elements; returns a flat array of ``dtype``."""
    pos = stream_positions(n, chunking)
    out = np.zeros(n, dtype=np.int64)
    so = np.asarray(stream_offsets, dtype=np.uint64)
    d = np.asarray(data, dtype=np.uint8)
    for k, p in enumerate(pos):
        a, b = int(so[k]), int(so[k + 1])
        out[p] = decode_stream(d[a:b], _rows_for(p, indexes, index_block), cdfs, lengths,
                               offsets, W, fmt, precision, alias)
    return out.astype(dtype)


# --------------------------------------------------- float latents -------
# Readings (the pages name CompressAI's build_indexes and the quantisation of
# a mean-scale model -- symbol = round(y - mean) -- but print neither):
#   * a scale below ``scale_bound`` counts as the bound (a NaN scale too);
#   * the row of a scale s is the first of the K table entries that is >= s,
#     the last row when none of the first K - 1 is: CompressAI starts every
#     index at K - 1 and takes one off for each of the first K - 1 entries
#     that is >= s;
#   * the symbol is y - mean computed in float32, rounded to the nearest
#     integer with ties to even (torch.round); a value that is not finite or
#     falls outside int32 is a range error;
#   * decoding gives back float32(symbol) + mean, in float32.
def build_indexes(scales, scale_table, scale_bound):
    """Row index of every scale (int32 array of the scales' shape)."""
    s = np.asarray(scales, dtype=np.float32)
    s = np.where(np.isnan(s) | (s < np.float32(scale_bound)), np.float32(scale_bound), s)
    t = np.asarray(scale_table, dtype=np.float32)
    K = t.size
    idx = np.full(s.shape, K - 1, dtype=np.int32)
    for i in range(K - 1):
        idx -= (s <= t[i]).astype(np.int32)
    return idx


def quantize(y, means=None):
    """Symbols round(y - mean) (float32, ties to even); raises OracleError
    (ERR_RANGE) for a value that is not finite or not in int32."""
    d = np.asarray(y, dtype=np.float32)
    if means is not None:
        d = d - np.asarray(means, dtype=np.float32)
    r = np.rint(d)
    if not np.all(np.isfinite(r)) or np.any(r < -2147483648.0) or np.any(r >= 2147483648.0):
        raise OracleError(ERR_RANGE, "quantize")
    return r.astype(np.int32)


def dequantize(symbols, means=None):
    """float32(symbol) + mean, in float32."""
    v = np.asarray(symbols).astype(np.float32)
    if means is not None:
        v = v + np.asarray(means, dtype=np.float32)
    return v
