"""ctypes binding of librans_b200 (include/rans_b200.h).

Argument marshalling only: torch tensors supply device memory and the
current CUDA stream; every coding step runs in the library's kernels.  The
functions named ``rans_*`` mirror the C entry points one to one; the helpers
below them (``Chunking``, ``Tables``, ``encode_with_indexes``,
``decode_with_indexes``) only allocate outputs and workspaces with torch and
call those entry points.

There is no fallback: if the shared library is missing or no CUDA device is
present, calls raise.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librans_b200.so")

OK = 0
ERR_ARG = -1
ERR_INDEX = -2
ERR_ZERO_FREQ = -3
ERR_RANGE = -4
ERR_CAPACITY = -5
ERR_CORRUPT = -6
ERR_CUDA = -7
ERR_TABLE = -8
ERR_TIMEOUT = -9

SYM_INT32, SYM_UINT8, SYM_INT16 = 0, 1, 2
CHUNK_CONTIG, CHUNK_EXPLICIT, CHUNK_TILED = 0, 1, 2
# coder formats: 64-bit state / 32-bit words / precision 16, and 32-bit
# state / 16-bit words / precision <= 15
FMT_RANS64, FMT_RANS32_16 = 0, 1
FMT_ALIAS = 0x100  # or'ed into a format: alias-coded streams
_FMT_CODE = {"rans64": FMT_RANS64, "rans32_16": FMT_RANS32_16}

_DTYPE_CODE = {torch.int32: SYM_INT32, torch.uint8: SYM_UINT8, torch.int16: SYM_INT16}


class rans_chunking(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("interleave", ctypes.c_int32),
                ("n_streams", ctypes.c_int64), ("stream_starts", ctypes.c_void_p),
                ("shape", ctypes.c_int64 * 4), ("group", ctypes.c_int64),
                ("tile_h", ctypes.c_int64), ("tile_w", ctypes.c_int64),
                ("index_block", ctypes.c_int64), ("format", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class rans_tables(ctypes.Structure):
    _fields_ = [("blob", ctypes.c_void_p), ("blob_bytes", ctypes.c_uint64),
                ("K", ctypes.c_int32), ("max_buckets", ctypes.c_int32),
                ("n_buckets", ctypes.c_int64), ("n_slots", ctypes.c_int64),
                ("meta_bytes", ctypes.c_uint32), ("bucket_bytes", ctypes.c_uint32),
                ("start_bytes", ctypes.c_uint32), ("slot_bytes", ctypes.c_uint32),
                ("enc_in_smem", ctypes.c_int32),
                ("dec_in_smem", ctypes.c_int32), ("device", ctypes.c_int32),
                ("precision", ctypes.c_int32), ("max_slot_log2", ctypes.c_int32),
                ("alias", ctypes.c_void_p), ("alias_bytes", ctypes.c_uint64),
                ("alias_remap_offset", ctypes.c_uint64)]


# (name, restype, argtypes) for every exported symbol of include/rans_b200.h
_P, _I32, _I64, _U64, _F64, _F32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                   ctypes.c_uint64, ctypes.c_double, ctypes.c_float)
_CHP = ctypes.POINTER(rans_chunking)
_TBP = ctypes.POINTER(rans_tables)
SIGNATURES = [
    ("rans_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("rans_version", ctypes.c_int, []),
    ("rans_gaussian_lengths", ctypes.c_int, [_P, _I32, _F64, _P, _P, _P]),
    ("rans_build_cdfs_from_scales", ctypes.c_int, [_P, _I32, _F64, _I32, _P, _I32, _P, _P, _P]),
    ("rans_build_cdfs_from_pmfs", ctypes.c_int,
     [_P, _I32, _I32, _P, _P, _I32, _P, _I32, _P, _P]),
    ("rans_tables_bytes", _U64, [_I32, _I32]),
    ("rans_tables_prepare", ctypes.c_int, [_P, _I32, _I32, _P, _P, _I32, _P, _U64, _TBP, _P]),
    ("rans_tables_refresh", ctypes.c_int, [_P, _I32, _I32, _P, _P, _TBP, _P]),
    ("rans_tables_refresh_from_scales", ctypes.c_int,
     [_P, _I32, _F64, _P, _I32, _P, _P, _TBP, _P]),
    ("rans_alias_bytes", _U64, [_TBP]),
    ("rans_alias_prepare", ctypes.c_int, [_P, _I32, _I32, _P, _TBP, _P, _U64, _P]),
    ("rans_num_streams", _I64, [_CHP, _I64]),
    ("rans_encode_workspace_bytes", _U64, [_CHP, _I64]),
    ("rans_decode_workspace_bytes", _U64, [_CHP, _I64]),
    ("rans_max_compressed_bytes", _U64, [_CHP, _I64]),
    ("rans_encode_with_indexes", ctypes.c_int,
     [_P, _I32, _P, _I64, _TBP, _CHP, _P, _U64, _P, _P, _U64, _P]),
    ("rans_decode_with_indexes", ctypes.c_int,
     [_P, _U64, _P, _P, _I64, _TBP, _CHP, _P, _I32, _P, _U64, _P]),
    ("rans_encode_with_indexes_noalloc", ctypes.c_int,
     [_P, _I32, _P, _I64, _TBP, _CHP, _P, _U64, _P, _P]),
    ("rans_build_indexes", ctypes.c_int, [_P, _I64, _P, _I32, _F32, _P, _P]),
    ("rans_encode_from_scales", ctypes.c_int,
     [_P, _P, _P, _I64, _P, _I32, _F32, _TBP, _CHP, _P, _U64, _P, _P, _U64, _P]),
    ("rans_decode_to_values", ctypes.c_int,
     [_P, _U64, _P, _P, _P, _I64, _P, _I32, _F32, _TBP, _CHP, _P, _P, _U64, _P]),
    ("rans_get_status", ctypes.c_int, [_P, _P]),
    ("rans_debug_divide", ctypes.c_int, [_P, _P, _I64, _P, _P, _P]),
    ("rans_debug_wait_timeout", ctypes.c_int, [_P, ctypes.c_uint32, _P]),
]

_lib = None


def lib():
    """Loads librans_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("librans_b200.so is missing: run "
                               "`python -m rans_entropy_coding_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class RansError(RuntimeError):
    def __init__(self, status, what=""):
        msg = lib().rans_status_string(int(status)).decode()
        super().__init__("librans_b200 %s: status %d (%s)" % (what, status, msg))
        self.status = int(status)


def check(status, what=""):
    if status != OK:
        raise RansError(status, what)
    return status


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("librans_b200 takes contiguous CUDA tensors")


# --------------------------------------------------------- C entry points --
def rans_gaussian_lengths(scales, tail_mass, cdf_lengths, offsets, stream=None):
    _need_cuda(scales, cdf_lengths, offsets)
    return lib().rans_gaussian_lengths(_ptr(scales), scales.numel(), tail_mass,
                                       _ptr(cdf_lengths), _ptr(offsets), _stream(stream))


def rans_build_cdfs_from_scales(scales, tail_mass, cdfs, cdf_lengths, offsets, stream=None,
                                precision=16):
    _need_cuda(scales, cdfs, cdf_lengths, offsets)
    return lib().rans_build_cdfs_from_scales(_ptr(scales), scales.numel(), tail_mass, precision,
                                             _ptr(cdfs), cdfs.shape[1], _ptr(cdf_lengths),
                                             _ptr(offsets), _stream(stream))


def rans_build_cdfs_from_pmfs(pmfs, pmf_lengths, tail_mass, cdfs, cdf_lengths, stream=None,
                              precision=16):
    _need_cuda(pmfs, pmf_lengths, tail_mass, cdfs, cdf_lengths)
    return lib().rans_build_cdfs_from_pmfs(_ptr(pmfs), pmfs.shape[0], pmfs.shape[1],
                                           _ptr(pmf_lengths), _ptr(tail_mass), precision,
                                           _ptr(cdfs), cdfs.shape[1], _ptr(cdf_lengths),
                                           _stream(stream))


def rans_tables_bytes(K, Lmax):
    return lib().rans_tables_bytes(K, Lmax)


def rans_tables_prepare(cdfs, cdf_lengths, offsets, blob, out, stream=None, precision=16):
    _need_cuda(cdfs, cdf_lengths, offsets, blob)
    return lib().rans_tables_prepare(_ptr(cdfs), cdfs.shape[0], cdfs.shape[1], _ptr(cdf_lengths),
                                     _ptr(offsets), precision, _ptr(blob), blob.numel(),
                                     ctypes.byref(out), _stream(stream))


def rans_tables_refresh(cdfs, cdf_lengths, offsets, tables, stream=None):
    _need_cuda(cdfs, cdf_lengths, offsets)
    return lib().rans_tables_refresh(_ptr(cdfs), cdfs.shape[0], cdfs.shape[1], _ptr(cdf_lengths),
                                     _ptr(offsets), ctypes.byref(tables.c), _stream(stream))


def rans_tables_refresh_from_scales(scales, tail_mass, cdfs, cdf_lengths, offsets, tables,
                                    stream=None):
    _need_cuda(scales, cdfs, cdf_lengths, offsets)
    return lib().rans_tables_refresh_from_scales(_ptr(scales), scales.numel(), tail_mass,
                                                 _ptr(cdfs), cdfs.shape[1], _ptr(cdf_lengths),
                                                 _ptr(offsets), ctypes.byref(tables.c),
                                                 _stream(stream))


def rans_alias_bytes(tables):
    return lib().rans_alias_bytes(ctypes.byref(tables.c))


def rans_alias_prepare(cdfs, cdf_lengths, tables, alias, stream=None):
    _need_cuda(cdfs, cdf_lengths, alias)
    return lib().rans_alias_prepare(_ptr(cdfs), cdfs.shape[0], cdfs.shape[1], _ptr(cdf_lengths),
                                    ctypes.byref(tables.c), _ptr(alias), alias.numel(),
                                    _stream(stream))


def rans_num_streams(chunking, n):
    return lib().rans_num_streams(ctypes.byref(chunking.c), n)


def rans_encode_workspace_bytes(chunking, n):
    return lib().rans_encode_workspace_bytes(ctypes.byref(chunking.c), n)


def rans_decode_workspace_bytes(chunking, n):
    return lib().rans_decode_workspace_bytes(ctypes.byref(chunking.c), n)


def rans_max_compressed_bytes(chunking, n):
    return lib().rans_max_compressed_bytes(ctypes.byref(chunking.c), n)


def rans_encode_with_indexes(symbols, indexes, n, tables, chunking, out, stream_offsets,
                             workspace, stream=None):
    _need_cuda(symbols, indexes, out, stream_offsets, workspace)
    return lib().rans_encode_with_indexes(
        _ptr(symbols), _DTYPE_CODE[symbols.dtype], _ptr(indexes), n, ctypes.byref(tables.c),
        ctypes.byref(chunking.c), _ptr(out), out.numel(), _ptr(stream_offsets), _ptr(workspace),
        workspace.numel(), _stream(stream))


def rans_decode_with_indexes(data, stream_offsets, indexes, n, tables, chunking, symbols_out,
                             workspace, stream=None):
    _need_cuda(data, stream_offsets, indexes, symbols_out, workspace)
    return lib().rans_decode_with_indexes(
        _ptr(data), data.numel(), _ptr(stream_offsets), _ptr(indexes), n,
        ctypes.byref(tables.c), ctypes.byref(chunking.c), _ptr(symbols_out),
        _DTYPE_CODE[symbols_out.dtype], _ptr(workspace), workspace.numel(), _stream(stream))


def rans_encode_with_indexes_noalloc(symbols, indexes, n, tables, chunking, out,
                                     stream_offsets, stream=None):
    _need_cuda(symbols, indexes, out, stream_offsets)
    return lib().rans_encode_with_indexes_noalloc(
        _ptr(symbols), _DTYPE_CODE[symbols.dtype], _ptr(indexes), n, ctypes.byref(tables.c),
        ctypes.byref(chunking.c), _ptr(out), out.numel(), _ptr(stream_offsets), _stream(stream))


def rans_build_indexes(scales, scale_table, scale_bound, indexes, stream=None):
    _need_cuda(scales, scale_table, indexes)
    return lib().rans_build_indexes(_ptr(scales), scales.numel(), _ptr(scale_table),
                                    scale_table.numel(), float(scale_bound), _ptr(indexes),
                                    _stream(stream))


def rans_encode_from_scales(y, means, scales, n, scale_table, scale_bound, tables, chunking,
                            out, stream_offsets, workspace, stream=None):
    _need_cuda(y, means, scales, scale_table, out, stream_offsets, workspace)
    return lib().rans_encode_from_scales(
        _ptr(y), _ptr(means), _ptr(scales), n, _ptr(scale_table), scale_table.numel(),
        float(scale_bound), ctypes.byref(tables.c), ctypes.byref(chunking.c), _ptr(out),
        out.numel(), _ptr(stream_offsets), _ptr(workspace), workspace.numel(), _stream(stream))


def rans_decode_to_values(data, stream_offsets, scales, means, n, scale_table, scale_bound,
                          tables, chunking, values, workspace, stream=None):
    _need_cuda(data, stream_offsets, scales, means, scale_table, values, workspace)
    return lib().rans_decode_to_values(
        _ptr(data), data.numel(), _ptr(stream_offsets), _ptr(scales), _ptr(means), n,
        _ptr(scale_table), scale_table.numel(), float(scale_bound), ctypes.byref(tables.c),
        ctypes.byref(chunking.c), _ptr(values), _ptr(workspace), workspace.numel(),
        _stream(stream))


def rans_get_status(workspace, stream=None):
    return lib().rans_get_status(_ptr(workspace), _stream(stream))


def rans_debug_wait_timeout(workspace, limit, stream=None):
    _need_cuda(workspace)
    return lib().rans_debug_wait_timeout(_ptr(workspace), limit, _stream(stream))


def rans_debug_divide(x, f, q, r, stream=None):
    _need_cuda(x, f, q, r)
    return lib().rans_debug_divide(_ptr(x), _ptr(f), x.numel(), _ptr(q), _ptr(r),
                                   _stream(stream))


# ------------------------------------------------------------- helpers --
class Chunking:
    """A rans_chunking plus the tensors it points to."""

    def __init__(self, c, keep=None):
        self.c = c
        self._keep = keep

    @property
    def interleave(self):
        return self.c.interleave

    @staticmethod
    def _format(fmt, alias):
        return _FMT_CODE[fmt] | (FMT_ALIAS if alias else 0)

    @staticmethod
    def contig(n_streams, interleave=1, index_block=1, fmt="rans64", alias=False):
        c = rans_chunking()
        c.kind, c.interleave, c.n_streams, c.index_block = (CHUNK_CONTIG, interleave, n_streams,
                                                            index_block)
        c.format = Chunking._format(fmt, alias)
        return Chunking(c)

    @staticmethod
    def explicit(starts, interleave=1, index_block=1, fmt="rans64", alias=False):
        """starts: CUDA int64 tensor of S + 1 element offsets."""
        _need_cuda(starts)
        assert starts.dtype == torch.int64
        c = rans_chunking()
        c.kind, c.interleave, c.n_streams, c.index_block = (CHUNK_EXPLICIT, interleave,
                                                            starts.numel() - 1, index_block)
        c.stream_starts = starts.data_ptr()
        c.format = Chunking._format(fmt, alias)
        return Chunking(c, keep=starts)

    @staticmethod
    def tiled(shape, group, tile_h, tile_w, interleave=32, index_block=1, fmt="rans64",
              alias=False):
        c = rans_chunking()
        c.kind, c.interleave, c.index_block = CHUNK_TILED, interleave, index_block
        for i, v in enumerate(shape):
            c.shape[i] = int(v)
        c.group, c.tile_h, c.tile_w = group, tile_h, tile_w
        c.format = Chunking._format(fmt, alias)
        return Chunking(c)

    @staticmethod
    def from_spec(spec, interleave, index_block=1, device="cuda", fmt="rans64", alias=False):
        """From the dict form used by the workloads module."""
        k = spec["kind"]
        if k == "contig":
            return Chunking.contig(spec["n_streams"], interleave, index_block, fmt, alias)
        if k == "tiled":
            return Chunking.tiled(spec["shape"], spec["cg"], spec["th"], spec["tw"], interleave,
                                  index_block, fmt, alias)
        if k == "explicit":
            st = torch.as_tensor(spec["starts"], dtype=torch.int64, device=device)
            return Chunking.explicit(st, interleave, index_block, fmt, alias)
        raise ValueError(k)


class Tables:
    """CDF rows (cdfs, cdf_lengths, offsets) plus the prepared table blob."""

    def __init__(self, cdfs, cdf_lengths, offsets, stream=None, blob_bytes=None, precision=16):
        """blob_bytes: the blob's size (default rans_tables_bytes(K, Lmax)); a
        smaller blob leaves the decoder fewer bitmap words.  precision: the
        rows sum to 2^precision (16 for the rans64 format, <= 15 for
        rans32_16)."""
        self.cdfs, self.cdf_lengths, self.offsets = cdfs, cdf_lengths, offsets
        self.precision = precision
        K, Lmax = cdfs.shape
        nbytes = rans_tables_bytes(K, Lmax) if blob_bytes is None else int(blob_bytes)
        self.blob = torch.empty(nbytes + 256, dtype=torch.uint8, device=cdfs.device)
        off = (-self.blob.data_ptr()) % 256
        self.blob = self.blob[off:off + nbytes]
        self.c = rans_tables()
        check(rans_tables_prepare(cdfs, cdf_lengths, offsets, self.blob, self.c, stream,
                                  precision), "tables_prepare")

    def prepare_alias(self, stream=None):
        """Builds the alias tables (every row's bucket count a power of two)
        for alias-coded streams (Chunking(..., alias=True))."""
        nbytes = rans_alias_bytes(self)
        self.alias = aligned_empty(nbytes, self.cdfs.device)
        check(rans_alias_prepare(self.cdfs, self.cdf_lengths, self, self.alias, stream),
              "alias_prepare")
        return self

    @staticmethod
    def build_from_scales(scales, tail_mass=1e-9, stream=None, precision=16):
        """Gaussian rows for a float32 CUDA scale table; returns
        (cdfs, cdf_lengths, offsets)."""
        K = scales.numel()
        dev = scales.device
        lengths = torch.empty(K, dtype=torch.int32, device=dev)
        offsets = torch.empty(K, dtype=torch.int32, device=dev)
        check(rans_gaussian_lengths(scales, tail_mass, lengths, offsets, stream), "lengths")
        lmin = int(lengths.min().item())
        if lmin < 0:
            raise RansError(lmin, "gaussian_lengths")
        Lmax = int(lengths.max().item())
        cdfs = torch.empty((K, Lmax), dtype=torch.int32, device=dev)
        check(rans_build_cdfs_from_scales(scales, tail_mass, cdfs, lengths, offsets, stream,
                                          precision), "build_cdfs_from_scales")
        return cdfs, lengths, offsets

    @staticmethod
    def build_from_pmfs(pmfs, pmf_lengths, tail_mass, stream=None, precision=16):
        K = pmfs.shape[0]
        Lmax = int(pmf_lengths.max().item()) + 2
        cdfs = torch.empty((K, Lmax), dtype=torch.int32, device=pmfs.device)
        lengths = torch.empty(K, dtype=torch.int32, device=pmfs.device)
        check(rans_build_cdfs_from_pmfs(pmfs, pmf_lengths, tail_mass, cdfs, lengths, stream,
                                        precision), "build_cdfs_from_pmfs")
        return cdfs, lengths

    @staticmethod
    def from_scales(scales, tail_mass=1e-9, stream=None, precision=16):
        return Tables(*Tables.build_from_scales(scales, tail_mass, stream, precision),
                      stream=stream, precision=precision)

    @staticmethod
    def from_pmfs(pmfs, pmf_lengths, tail_mass, offsets, stream=None, precision=16):
        cdfs, lengths = Tables.build_from_pmfs(pmfs, pmf_lengths, tail_mass, stream, precision)
        return Tables(cdfs, lengths, offsets, stream=stream, precision=precision)


def aligned_empty(nbytes, device="cuda"):
    """A 256-byte aligned uint8 CUDA buffer of nbytes."""
    raw = torch.empty(int(nbytes) + 256, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 256
    return raw[off:off + int(nbytes)]


class Workspaces:
    """Reusable encode/decode workspaces and output buffers for one shape."""

    def __init__(self, chunking, n, device="cuda"):
        self.S = rans_num_streams(chunking, n)
        if self.S < 0:
            check(int(self.S), "num_streams")
        self.enc = aligned_empty(rans_encode_workspace_bytes(chunking, n), device)
        self.dec = aligned_empty(max(256, rans_decode_workspace_bytes(chunking, n)), device)
        self.out = torch.empty(rans_max_compressed_bytes(chunking, n), dtype=torch.uint8,
                               device=device)
        self.offsets = torch.empty(self.S + 1, dtype=torch.int64, device=device)


def encode_with_indexes(symbols, indexes, tables, chunking, ws=None, stream=None):
    """Returns (buffer, stream_offsets[S+1] as int64, workspaces); the coded
    bytes are buffer[:stream_offsets[-1]]."""
    n = symbols.numel()
    if ws is None:
        ws = Workspaces(chunking, n, symbols.device)
    check(rans_encode_with_indexes(symbols, indexes, n, tables, chunking, ws.out, ws.offsets,
                                   ws.enc, stream), "encode")
    return ws.out, ws.offsets, ws


def encode_from_scales(y, scales, scale_table, scale_bound, tables, chunking, means=None,
                       ws=None, stream=None):
    """Float latents in: like encode_with_indexes, rows from the scales and
    symbols rint(y - mean) computed inside the coder."""
    n = y.numel()
    if ws is None:
        ws = Workspaces(chunking, n, y.device)
    check(rans_encode_from_scales(y, means, scales, n, scale_table, scale_bound, tables,
                                  chunking, ws.out, ws.offsets, ws.enc, stream), "encode")
    return ws.out, ws.offsets, ws


def decode_to_values(data, stream_offsets, scales, scale_table, scale_bound, tables, chunking,
                     means=None, out=None, ws=None, stream=None):
    """Float values out: float32(symbol) + mean."""
    n = scales.numel()
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=data.device)
    wsd = ws.dec if ws is not None else aligned_empty(256, data.device)
    check(rans_decode_to_values(data, stream_offsets, scales, means, n, scale_table,
                                scale_bound, tables, chunking, out, wsd, stream), "decode")
    return out, wsd


def decode_with_indexes(data, stream_offsets, indexes, tables, chunking, n, dtype=torch.int32,
                        out=None, ws=None, stream=None):
    if out is None:
        out = torch.empty(n, dtype=dtype, device=data.device)
    wsd = ws.dec if ws is not None else aligned_empty(256, data.device)
    check(rans_decode_with_indexes(data, stream_offsets, indexes, n, tables, chunking, out, wsd,
                                   stream), "decode")
    return out, wsd
