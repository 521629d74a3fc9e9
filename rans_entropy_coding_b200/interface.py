"""A coder object over the C ABI, in the shape of the interfaces the pages
describe ("torch_ans 0.3.0", High-level API: a TorchANSInterface chosen by
impl / freq_precision / num_interleaves / alias_sampling, whose
encode_with_indexes and decode_with_indexes take symbols, indexes, cdfs,
cdf sizes and offsets; rans_stream_to_byte_strings and
rans_byte_strings_to_stream move streams to and from Python bytes).

Argument marshalling only: every coding step runs in librans_b200's kernels.
"""
import torch

from . import _lib as L

_SYM = {torch.int32, torch.int16, torch.uint8}


class RansCoder:
    """Rows set once, then any number of encode / decode calls.

    impl: "rans64" (64-bit state, 32-bit words, precision 16) or
    "rans32_16" (32-bit state, 16-bit words, precision <= 15).
    interleave: 1, 2, 4, 8 or 32 states per stream (alias: up to 8).
    """

    def __init__(self, impl="rans64", precision=None, interleave=32, alias=False,
                 device="cuda"):
        if impl not in L._FMT_CODE:
            raise ValueError("impl must be one of %s" % sorted(L._FMT_CODE))
        self.impl = impl
        self.precision = precision if precision is not None else (16 if impl == "rans64" else 15)
        self.interleave = interleave
        self.alias = alias
        self.device = torch.device(device)
        self.tables = None

    # -------------------------------------------------------------- rows --
    def set_scale_table(self, scales, tail_mass=1e-9):
        """Gaussian rows from a float32 scale table (one row per entry)."""
        scales = torch.as_tensor(scales, dtype=torch.float32, device=self.device)
        rows = L.Tables.build_from_scales(scales, tail_mass, precision=self.precision)
        return self._set_rows(*rows)

    def set_pmfs(self, pmfs, pmf_lengths, tail_mass, offsets):
        """Rows from pmfs ([K, S] float32, lengths, tail masses, offsets)."""
        dev = self.device
        pmfs = torch.as_tensor(pmfs, dtype=torch.float32, device=dev).contiguous()
        lens = torch.as_tensor(pmf_lengths, dtype=torch.int32, device=dev)
        tail = torch.as_tensor(tail_mass, dtype=torch.float32, device=dev)
        offs = torch.as_tensor(offsets, dtype=torch.int32, device=dev)
        cdfs, lengths = L.Tables.build_from_pmfs(pmfs, lens, tail, precision=self.precision)
        return self._set_rows(cdfs, lengths, offs)

    def set_cdfs(self, cdfs, cdf_lengths, offsets):
        """Quantised rows given directly (int32 [K, Lmax], summing to
        2^precision)."""
        dev = self.device
        return self._set_rows(torch.as_tensor(cdfs, dtype=torch.int32, device=dev).contiguous(),
                              torch.as_tensor(cdf_lengths, dtype=torch.int32, device=dev),
                              torch.as_tensor(offsets, dtype=torch.int32, device=dev))

    def _set_rows(self, cdfs, lengths, offsets):
        self.tables = L.Tables(cdfs, lengths, offsets, precision=self.precision)
        if self.alias:
            self.tables.prepare_alias()
        return self

    # ----------------------------------------------------------- streams --
    def chunking(self, n, n_streams=None, tiles=None, index_block=1):
        """Contiguous streams (n_streams, default one per 64 Ki symbols) or,
        with tiles=(shape, group, tile_h, tile_w), spatial tiles of an NCHW
        tensor."""
        fmt = dict(fmt=self.impl, alias=self.alias)
        if tiles is not None:
            shape, group, th, tw = tiles
            return L.Chunking.tiled(shape, group, th, tw, self.interleave, index_block, **fmt)
        if n_streams is None:
            n_streams = max(1, -(-n // 65536))
        return L.Chunking.contig(n_streams, self.interleave, index_block, **fmt)

    def encode_with_indexes(self, symbols, indexes, chunking=None, **kw):
        """Returns (data, stream_offsets): the packed streams as a uint8 CUDA
        tensor and S + 1 int64 byte offsets; device errors raise."""
        self._need_tables()
        symbols = symbols.to(self.device).contiguous().reshape(-1)
        if symbols.dtype not in _SYM:
            symbols = symbols.to(torch.int32)
        indexes = torch.as_tensor(indexes, dtype=torch.int32, device=self.device).reshape(-1)
        ch = chunking or self.chunking(symbols.numel(), **kw)
        out, offs, ws = L.encode_with_indexes(symbols, indexes, self.tables, ch)
        L.check(L.rans_get_status(ws.enc), "encode")
        total = int(offs[-1].item())
        return out[:total].clone(), offs.clone()

    def decode_with_indexes(self, data, stream_offsets, indexes, n, chunking=None,
                            dtype=torch.int32, **kw):
        """Symbols (a flat CUDA tensor of n elements of dtype)."""
        self._need_tables()
        data = torch.as_tensor(data, dtype=torch.uint8).to(self.device).contiguous()
        offs = torch.as_tensor(stream_offsets, dtype=torch.int64).to(self.device).contiguous()
        indexes = torch.as_tensor(indexes, dtype=torch.int32, device=self.device).reshape(-1)
        ch = chunking or self.chunking(n, **kw)
        sym, wsd = L.decode_with_indexes(data, offs, indexes, self.tables, ch, n, dtype)
        L.check(L.rans_get_status(wsd), "decode")
        return sym

    def _need_tables(self):
        if self.tables is None:
            raise RuntimeError("set the rows first (set_scale_table, set_pmfs or set_cdfs)")


def to_byte_strings(data, stream_offsets):
    """One Python bytes object per stream."""
    d = data.cpu().numpy().tobytes()
    o = [int(v) for v in stream_offsets.cpu().tolist()]
    return [d[o[k]:o[k + 1]] for k in range(len(o) - 1)]


def from_byte_strings(strings, device="cuda"):
    """(data, stream_offsets) from per-stream byte strings."""
    offs = [0]
    for b in strings:
        offs.append(offs[-1] + len(b))
    data = torch.frombuffer(bytearray(b"".join(strings)), dtype=torch.uint8) if offs[-1] else \
        torch.zeros(0, dtype=torch.uint8)
    return data.to(device), torch.tensor(offs, dtype=torch.int64, device=device)
