"""B200-native PagedAttention over a block-table KV cache.

The hot path lives in libtv.so (CUDA kernels for sm_100a behind the C ABI of
include/tv.h); this package is its thin Python binding plus the seeded
synthetic workloads used by the tests and the benchmark.
"""
from ._lib import (TVError, load, tv_kv_append, tv_paged_decode,  # noqa: F401
                   tv_paged_decode_append, tv_paged_decode_split,
                   tv_paged_decode_split_static, tv_paged_prefill,
                   tv_split_merge)

__all__ = ["TVError", "load", "tv_kv_append", "tv_paged_decode",
           "tv_paged_decode_append", "tv_paged_decode_split",
           "tv_split_merge", "tv_paged_prefill",
           "tv_paged_decode_split_static"]
