"""SPADE executor hot path on B200 (sm_100a): input-adaptive block-sparse
attention of a video-DiT layer behind a C ABI (include/spade.h).

    from input_adaptive_block_b200 import api
    out = api.grouped_attn(q, k, v, schemes, table)

The kernels live in libspade.so (built by `python -m
input_adaptive_block_b200.build`); `api` only marshals tensors and streams.
"""
from . import _lib

__version__ = "0.1.0"


def library_path() -> str:
    return _lib.LIB_PATH
