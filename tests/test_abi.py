"""The C-ABI library loads and exports every symbol include/tv.h declares,
and host-side argument checks reject bad calls before anything is launched.
None of these tests needs a GPU: every call here returns before CUDA."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_376_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(tv_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = _declared()
    assert {"tv_kv_append", "tv_paged_decode", "tv_paged_decode_split",
            "tv_split_merge", "tv_paged_prefill"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(_lib.SIGNATURES), names ^ set(_lib.SIGNATURES)


def test_status_strings(lib):
    assert lib.tv_status_string(0) == b"TV_OK"
    assert lib.tv_status_string(2) == b"TV_ERR_UNSUPPORTED"
    assert lib.tv_version() >= 100


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_unsupported_shapes_are_rejected_before_launch(lib):
    p = _fake()
    # head_dim 128
    assert lib.tv_paged_decode(p, p, p, p, p, 4, p, 1, 32, 8, 128, 16, 10,
                               0.1, None, None) == 2
    # page sizes other than 16 and 32
    for ps in (8, 24, 64):
        assert lib.tv_paged_decode(p, p, p, p, p, 4, p, 1, 32, 8, 64, ps, 10,
                                   0.1, None, None) == 2
    # 12 query heads over 8 KV heads
    assert lib.tv_paged_decode(p, p, p, p, p, 4, p, 1, 12, 8, 64, 16, 10,
                               0.1, None, None) == 2
    # GQA ratio 16
    assert lib.tv_paged_decode(p, p, p, p, p, 4, p, 1, 32, 2, 64, 16, 10,
                               0.1, None, None) == 2
    assert lib.tv_kv_append(p, p, p, 4, p, p, 10, 8, 96, 16, None,
                            None) == 2
    assert lib.tv_split_merge(p, p, p, p, 2, 32, 32, 512, 4, None) == 2
    # prefill takes 1, 2, 4 or 8 query heads per KV head, not 16
    assert lib.tv_paged_prefill(p, p, 8, p, p, p, p, 4, p, 1, 8, 32, 2, 64,
                                16, 10, 0.1, None, 0, None, None) == 2


def test_invalid_arguments_are_rejected_before_launch(lib):
    p = _fake()
    unaligned = _fake(0x10008)
    # null q
    assert lib.tv_paged_decode(p, None, p, p, p, 4, p, 1, 32, 8, 64, 16, 10,
                               0.1, None, None) == 1
    # misaligned pool
    assert lib.tv_paged_decode(p, p, unaligned, p, p, 4, p, 1, 32, 8, 64, 16,
                               10, 0.1, None, None) == 1
    # non-finite scale
    assert lib.tv_paged_decode(p, p, p, p, p, 4, p, 1, 32, 8, 64, 16, 10,
                               float("nan"), None, None) == 1
    # partition not a multiple of the page size
    assert lib.tv_paged_decode_split(p, p, p, p, p, p, 4, p, 1, 32, 8, 64,
                                     16, 10, 0.1, 100, 4, None, None) == 1
    # negative token count
    assert lib.tv_kv_append(p, p, p, -1, p, p, 10, 8, 64, 16, None,
                            None) == 1
    assert lib.tv_split_merge(None, p, p, p, 2, 32, 64, 512, 4, None) == 1
    # prefill workspace too small for 3 sequences x 2 blocks, or misaligned
    assert lib.tv_paged_prefill(p, p, 100, p, p, p, p, 4, p, 3, 100, 32, 8,
                                64, 16, 10, 0.1, p, 16, None, None) == 1
    assert lib.tv_paged_prefill(p, p, 100, p, p, p, p, 4, p, 3, 100, 32, 8,
                                64, 16, 10, 0.1, unaligned, 64, None,
                                None) == 1


def test_prefill_refuses_a_scale_that_is_not_positive(lib):
    """The prefill kernel scales each key tile's maximum raw score; that is
    the maximum of the scaled scores only for scale > 0, so anything else is
    refused instead of silently overflowing the exponentials."""
    p = _fake()
    for scale in (-0.125, 0.0, -0.0, float("-inf")):
        assert lib.tv_paged_prefill(p, p, 8, p, p, p, p, 4, p, 1, 8, 32, 8,
                                    64, 16, 10, scale, None, 0, None,
                                    None) == 1, scale


def test_rope_calls_need_a_table(lib):
    p = _fake()
    unaligned = _fake(0x10008)
    # no table, a misaligned table, an empty table
    for tab, npos in ((None, 8), (unaligned, 8), (p, 0)):
        assert lib.tv_kv_append_rope(p, p, p, p, 4, p, p, 10, 8, 64, 16, tab,
                                     npos, None, None) == 1
        assert lib.tv_paged_decode_append_rope(
            p, p, p, p, p, p, p, 4, p, 1, 32, 8, 64, 16, 10, 0.125, tab, npos,
            None, None) == 1
    # no positions
    assert lib.tv_kv_append_rope(p, p, p, None, 4, p, p, 10, 8, 64, 16, p, 8,
                                 None, None) == 1
    # head_dim 128 is not supported
    assert lib.tv_kv_append_rope(p, p, p, p, 4, p, p, 10, 8, 128, 16, p, 8,
                                 None, None) == 2
    assert lib.tv_kv_append_rope(None, None, None, None, 0, p, p, 10, 8, 64,
                                 16, None, 0, None, None) == 0


def test_pool_state_size_includes_the_growth_marks(lib):
    """TV_POOL_STATE_INTS(np) = 4 + 4 np + TV_POOL_MAX_SEQS (include/tv.h);
    the binding sizes and checks state arrays by the same rule."""
    hdr = open(os.path.join(ROOT, "include", "tv.h")).read()
    assert re.search(r"#define TV_POOL_MAX_SEQS 1024\b", hdr)
    assert _lib.POOL_MAX_SEQS == 1024
    assert _lib.pool_state_ints(10) == 4 + 40 + 1024
    # more sequences than the marks cover are refused before any launch
    p = _fake()
    assert lib.tv_pool_append_slots(p, 10, p, 4, p, None, 1025, None, p, p,
                                    8, 64, 16, None, None) == 2


def test_sizes_beyond_32_bit_positions_are_refused(lib):
    p = _fake()
    big_mb = 1 << 27          # x 16-token pages = 2^31 token positions
    assert lib.tv_paged_decode(p, p, p, p, p, big_mb, p, 1, 32, 8, 64, 16, 10,
                               0.1, None, None) == 2
    assert lib.tv_paged_decode_append(p, p, p, p, p, p, p, big_mb, p, 1, 32,
                                      8, 64, 16, 10, 0.1, None, None) == 2
    assert lib.tv_paged_prefill(p, p, 8, p, p, p, p, big_mb, p, 1, 8, 32, 8,
                                64, 16, 10, 0.1, None, 0, None, None) == 2
    # 65535 sequences x 65535 blocks of 64 rows: more ordering items than an
    # int holds (refused only when the ordering workspace is given)
    assert lib.tv_paged_prefill(p, p, 1 << 30, p, p, p, p, 4, p, 65535,
                                65535 * 64, 32, 8, 64, 16, 10, 0.1, p,
                                1 << 40, None, None) == 2


def test_prefill_workspace_size(lib):
    import ctypes
    n = ctypes.c_size_t(0)
    # 4 bytes per 32-row block of every sequence (the blocks of the largest
    # group size, 8: 256 / 8 rows), rounded up to 16
    assert lib.tv_prefill_workspace_size(3, 100, ctypes.byref(n)) == 0
    assert n.value == 48          # 3 x 4 blocks = 48 bytes
    assert lib.tv_prefill_workspace_size(16, 512, ctypes.byref(n)) == 0
    assert n.value == 1024        # 16 x 16 blocks
    assert lib.tv_prefill_workspace_size(0, 0, ctypes.byref(n)) == 0
    assert n.value == 0
    assert lib.tv_prefill_workspace_size(-1, 8, ctypes.byref(n)) == 1


def test_prefill_workspace_is_checked_for_the_call_group(lib):
    """A call checks the workspace its own group needs: 16 sequences of up
    to 512 rows need 16 x 8 blocks of 64 rows at G = 4 (512 bytes) but
    16 x 16 blocks of 32 rows at G = 8 (1024 bytes)."""
    p = _fake()
    args = lambda hq, hkv, nbytes: (p, p, 8192, p, p, p, p, 64, p, 16, 512, hq,
                                    hkv, 64, 16, 4096, 0.1, p, nbytes, None,
                                    None)
    assert lib.tv_paged_prefill(*args(32, 4, 512)) == 1      # G = 8: too small
    assert lib.tv_paged_prefill(*args(32, 4, 1023)) == 1
    assert lib.tv_paged_prefill(*args(24, 8, 64)) == 2       # G = 3: unsupported


def test_empty_work_is_a_no_op(lib):
    p = _fake()
    assert lib.tv_kv_append(None, None, None, 0, p, p, 10, 8, 64, 16, None,
                            None) == 0
    assert lib.tv_paged_decode(None, None, None, None, None, 4, None, 0, 32,
                               8, 64, 16, 10, 0.1, None, None) == 0
    assert lib.tv_paged_prefill(None, None, 0, None, None, None, None, 4,
                                None, 0, 0, 32, 8, 64, 16, 10, 0.1, None, 0,
                                None, None) == 0


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(_lib.TVError):
        _lib.load(str(tmp_path / "nope.so"))
