"""Property tests of the oracle over random rows, precisions, symbols,
interleaves, formats and both lookups: every stream decodes to its symbols,
has the format's word size and holds at least the W flushed states."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O


@st.composite
def cases(draw):
    fmt = draw(st.sampled_from(["rans64", "rans32_16"]))
    prec = 16 if fmt == "rans64" else draw(st.integers(min_value=3, max_value=15))
    alias = draw(st.booleans())
    if alias:
        n = 1 << draw(st.integers(min_value=0, max_value=min(6, prec)))
    else:
        n = draw(st.integers(min_value=1, max_value=min(40, 1 << prec)))
    M = 1 << prec
    cuts = sorted(draw(st.lists(st.integers(min_value=1, max_value=M - 1), min_size=n - 1,
                                max_size=n - 1, unique=True)))
    cdf = np.array([0] + cuts + [M], np.int32)
    offset = draw(st.integers(min_value=-50, max_value=50))
    W = draw(st.sampled_from([1, 2, 4, 8] + ([] if alias else [32])))
    syms = draw(st.lists(st.one_of(st.integers(min_value=offset - 3, max_value=offset + n + 3),
                                   st.integers(min_value=-2**31, max_value=2**31 - 1)),
                         max_size=60))
    return fmt, prec, alias, cdf, offset, W, syms


@settings(max_examples=300, deadline=None)
@given(cases())
def test_round_trip_and_layout(case):
    fmt, prec, alias, cdf, offset, W, syms = case
    c = cdf[None, :]
    lengths = np.array([cdf.size], np.int32)
    offsets = np.array([offset], np.int32)
    sym = np.array(syms, np.int64)
    rows = np.zeros(sym.size, np.int32)
    b = O.encode_stream(sym, rows, c, lengths, offsets, W=W, fmt=fmt, precision=prec,
                        alias=alias)
    word = 4 if fmt == "rans64" else 2
    assert b.size % word == 0 and b.size >= 2 * word * W
    back = O.decode_stream(b, rows, c, lengths, offsets, W=W, fmt=fmt, precision=prec,
                           alias=alias)
    assert back.tolist() == sym.tolist()
