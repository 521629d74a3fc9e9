"""Runs one workload through the oracle and through librans_b200 (C ABI) so
tests can compare them.  Both sides code the same seeded arrays; the GPU
side never feeds the oracle.  A workload dict may name a coder format
("fmt": "rans64" | "rans32_16") and the rows' "precision"."""
import numpy as np
import torch

import oracle as O
import rans_entropy_coding_b200 as rb


def fmt_of(w):
    return w.get("fmt", "rans64")


def alias_of(w):
    return bool(w.get("alias", False))


def precision_of(w):
    return w.get("precision", 16 if fmt_of(w) == "rans64" else 15)


def oracle_tables(w):
    p = precision_of(w)
    if "scales" in w:
        c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"], precision=p)
    else:
        c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"], precision=p)
        o = np.asarray(w["offsets"], dtype=np.int32)
    return c, l, o


def gpu_rows(w, dev="cuda"):
    """CDF rows built on the GPU: (cdfs, lengths, offsets) CUDA tensors."""
    p = precision_of(w)
    if "scales" in w:
        return rb.Tables.build_from_scales(torch.from_numpy(np.asarray(w["scales"])).to(dev),
                                           w["tail_mass"], precision=p)
    cdfs, lengths = rb.Tables.build_from_pmfs(
        torch.from_numpy(np.ascontiguousarray(w["pmfs"])).to(dev),
        torch.from_numpy(np.asarray(w["pmf_lengths"], np.int32)).to(dev),
        torch.from_numpy(np.asarray(w["tail"], np.float32)).to(dev), precision=p)
    return cdfs, lengths, torch.from_numpy(np.asarray(w["offsets"], np.int32)).to(dev)


def tables_from_numpy(c, l, o, dev="cuda", precision=16):
    return rb.Tables(torch.from_numpy(np.ascontiguousarray(c)).to(dev),
                     torch.from_numpy(np.ascontiguousarray(l)).to(dev),
                     torch.from_numpy(np.ascontiguousarray(o)).to(dev), precision=precision)


def chunking_of(w, dev="cuda"):
    return rb.Chunking.from_spec(w["chunking"], w["W"], w["index_block"], device=dev,
                                 fmt=fmt_of(w), alias=alias_of(w))


def gpu_encode_decode(w, tables, dev="cuda", expect_ok=True):
    """Returns (bytes, offsets, decoded, enc_status, dec_status) as numpy."""
    sym = torch.from_numpy(np.ascontiguousarray(w["symbols"]).reshape(-1)).to(dev)
    idx = torch.from_numpy(np.ascontiguousarray(w["indexes"], dtype=np.int32)).to(dev)
    ch = chunking_of(w, dev)
    out, offs, ws = rb.encode_with_indexes(sym, idx, tables, ch)
    est = rb.rans_get_status(ws.enc)
    total = int(offs[-1].item()) if offs.numel() else 0
    if expect_ok:
        assert est == rb.OK, rb.RansError(est, "encode")
    data = out[:total] if est == rb.OK else out[:0]
    dec, wsd = rb.decode_with_indexes(data, offs, idx, tables, ch, sym.numel(), sym.dtype, ws=ws)
    dst = rb.rans_get_status(wsd)
    if expect_ok:
        assert dst == rb.OK, rb.RansError(dst, "decode")
    return (data.cpu().numpy(), offs.cpu().numpy().astype(np.uint64), dec.cpu().numpy(), est,
            dst)


def oracle_encode(w, c, l, o, streams=None):
    sym = np.asarray(w["symbols"]).reshape(-1)
    return O.encode_with_indexes(sym, w["indexes"], c, l, o, w["chunking"], W=w["W"],
                                 index_block=w["index_block"], streams=streams, fmt=fmt_of(w),
                                 precision=precision_of(w), alias=alias_of(w))


def oracle_encode_parallel(w, c, l, o, workers=None):
    """The oracle's container encode of every stream of the workload, one
    stream per oracle call spread over host threads (the C oracle runs
    without the GIL); returns (bytes, offsets uint64[S+1]) like
    oracle_encode."""
    import concurrent.futures as cf
    import os
    flat = np.asarray(w["symbols"]).reshape(-1)
    idx = np.asarray(w["indexes"], dtype=np.int32)
    blk = int(w["index_block"])
    S = O.num_streams(flat.size, w["chunking"])

    def one(k):
        p = O.stream_position(flat.size, w["chunking"], k)
        return O.encode_stream(flat[p].astype(np.int64), idx[p // blk], c, l, o, w["W"],
                               fmt_of(w), precision_of(w), alias_of(w))

    with cf.ThreadPoolExecutor(max_workers=workers or os.cpu_count() or 1) as ex:
        parts = list(ex.map(one, range(S)))
    offs = np.zeros(S + 1, dtype=np.uint64)
    offs[1:] = np.cumsum([p.size for p in parts], dtype=np.uint64)
    data = np.concatenate(parts) if parts else np.zeros(0, dtype=np.uint8)
    return data, offs
