"""rans_entropy_coding_b200 -- indexed 64-bit rANS entropy coding on NVIDIA
B200 (sm_100a): the C-ABI library librans_b200 and its thin Python binding.

See include/rans_b200.h for the boundary.  Build the library with
``python -m rans_entropy_coding_b200.build``.
"""
from ._lib import (  # noqa: F401
    CHUNK_CONTIG, CHUNK_EXPLICIT, CHUNK_TILED, ERR_ARG, ERR_CAPACITY, ERR_CORRUPT, ERR_CUDA,
    FMT_ALIAS, FMT_RANS32_16, FMT_RANS64,
    ERR_INDEX, ERR_RANGE, ERR_TABLE, ERR_TIMEOUT, ERR_ZERO_FREQ, LIB_PATH, OK, SIGNATURES,
    SYM_INT16, SYM_INT32, SYM_UINT8, Chunking, RansError, Tables, Workspaces, aligned_empty,
    check, decode_to_values, decode_with_indexes, encode_from_scales, encode_with_indexes, lib,
    rans_alias_bytes, rans_alias_prepare, rans_build_cdfs_from_pmfs, rans_build_indexes, rans_decode_to_values,
    rans_encode_from_scales,
    rans_build_cdfs_from_scales, rans_chunking, rans_debug_divide, rans_debug_wait_timeout, rans_decode_with_indexes,
    rans_decode_workspace_bytes, rans_encode_with_indexes, rans_encode_with_indexes_noalloc,
    rans_encode_workspace_bytes,
    rans_gaussian_lengths, rans_get_status, rans_max_compressed_bytes, rans_num_streams,
    rans_tables, rans_tables_bytes, rans_tables_prepare, rans_tables_refresh,
    rans_tables_refresh_from_scales)
from .interface import RansCoder, from_byte_strings, to_byte_strings  # noqa: F401,E402
