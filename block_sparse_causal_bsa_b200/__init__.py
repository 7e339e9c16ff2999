"""Block-sparse causal attention for NVIDIA B200 (sm_100a).

The compute lives in libbsa.so (C ABI: include/bsa.h); ``binding`` is its
ctypes wrapper, ``synthetic`` the seeded input generators.
"""
from .binding import (  # noqa: F401
    BsaError, SelectConfig, Shape, SelectParams, DecodeShape, DecodeParams, ScoreParams,
    bsa_score, bsa_score_ex, bsa_score_workspace_bytes, bsa_select, bsa_select_workspace_bytes,
    bsa_kv_idx_width, bsa_attend, bsa_attend_vs, bsa_attend_vs_workspace_bytes, bsa_decode,
    bsa_decode_list, bsa_select_noalloc, bsa_selftest_wait, score, select, attend, attend_vs,
    decode, prefill, lib,
)
