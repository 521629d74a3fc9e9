"""The coder object (rans_entropy_coding_b200.interface): byte-string
conversion on the CPU; encode / decode through it on the GPU, against the
oracle's streams."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from rans_entropy_coding_b200 import interface as I


def test_byte_strings_round_trip():
    strings = [b"", b"\x01\x02\x03\x04", b"", b"abcdefgh" * 3]
    data, offs = I.from_byte_strings(strings, device="cpu")
    assert offs.tolist() == [0, 0, 4, 4, 28]
    assert I.to_byte_strings(data, offs) == strings
    data, offs = I.from_byte_strings([], device="cpu")
    assert data.numel() == 0 and offs.tolist() == [0]


def test_unknown_impl_is_refused():
    with pytest.raises(ValueError):
        I.RansCoder(impl="rans32")


@pytest.mark.gpu
@pytest.mark.parametrize("impl,interleave,alias", [("rans64", 32, False), ("rans64", 1, False),
                                                   ("rans32_16", 32, False),
                                                   ("rans32_16", 4, True), ("rans64", 8, True)])
def test_coder_matches_oracle(impl, interleave, alias):
    prec = 16 if impl == "rans64" else 15
    if alias:   # power-of-two bucket counts: the pmf rows of 255 symbols + escape
        w = WL.r16_rows(n_streams=8, per_stream=2000)
        coder = I.RansCoder(impl, interleave=interleave, alias=True)
        coder.set_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"], w["offsets"])
        c, l = O.build_cdfs_from_pmfs(w["pmfs"], w["pmf_lengths"], w["tail"], precision=prec)
        o = np.asarray(w["offsets"], np.int32)
    else:
        w = WL.tiny(seed=21, n=16000)
        coder = I.RansCoder(impl, interleave=interleave).set_scale_table(w["scales"])
        c, l, o = O.build_cdfs_from_scales(w["scales"], w["tail_mass"], precision=prec)
    sym = torch.from_numpy(np.asarray(w["symbols"]).reshape(-1))
    idx = torch.from_numpy(np.asarray(w["indexes"], np.int32))
    n = sym.numel()
    data, offs = coder.encode_with_indexes(sym, idx, n_streams=8)
    want = [O.encode_stream(sym.numpy()[p].astype(np.int64), idx.numpy()[p], c, l, o,
                            W=interleave, fmt=impl, precision=prec, alias=alias).tobytes()
            for p in O.stream_positions(n, dict(kind="contig", n_streams=8))]
    assert I.to_byte_strings(data, offs) == want
    d2, o2 = I.from_byte_strings(want)
    back = coder.decode_with_indexes(d2, o2, idx, n, n_streams=8)
    assert torch.equal(back.cpu(), sym)
