"""The C ABI loads, exports every declared symbol, and its host-only calls
behave as documented (no GPU needed)."""

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq():
    from layer_wise_mixed_kvq_b200 import build
    build.build()
    from layer_wise_mixed_kvq_b200 import kvq as _kvq
    return _kvq


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for required in ("kvq_cache_create", "kvq_append", "kvq_decode_attn", "kvq_equiv_bits"):
        assert required in names


def test_library_exports_every_declared_symbol(kvq):
    import ctypes
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert sorted(kvq.EXPORTS) == _declared_symbols()


def test_equiv_bits_printed_maps(kvq):
    llama = [(4, 8) if l in (0, 1, 2, 31) else (4, 2) if l <= 26 else (2, 2) for l in range(32)]
    qwen = [(8, 4) if l <= 3 else (4, 4) if l <= 19 else (4, 2) for l in range(28)]
    assert kvq.kvq_equiv_bits(llama) == 3.25
    assert kvq.kvq_equiv_bits(qwen) == 4.0
    assert kvq.kvq_equiv_bits([(16, 16)] * 8 + [(8, 8)] * 24) == 10.0
    assert kvq.kvq_equiv_bits([(3, 4)]) == -1.0
    assert kvq.kvq_equiv_bits([(16, 8)]) == -1.0


def test_page_bytes(kvq):
    for D in (64, 128):
        for k in (2, 4, 8):
            for v in (2, 4, 8):
                assert kvq.kvq_page_bytes((k, v), D) == 4 * D * (k + v) + 4 * D + 128
        assert kvq.kvq_page_bytes((16, 16), D) == 128 * D
    assert kvq.kvq_page_bytes((4, 4), 96) == 0
    assert kvq.kvq_page_bytes((1, 4), 128) == 0


def test_page_bytes_per_token_keys(kvq):
    # per-token keys: 32 key scale/zero pairs per page instead of D
    for D in (64, 128):
        for k in (2, 4, 8):
            for v in (2, 4, 8):
                assert kvq.kvq_page_bytes((k, v, kvq.KVQ_KEY_PER_TOKEN), D) == 4 * D * (k + v) + 256
    assert kvq.kvq_page_bytes((16, 16, kvq.KVQ_KEY_PER_TOKEN), 128) == 0   # bf16 layers have no key mode
    assert kvq.kvq_page_bytes((4, 4, 2), 128) == 0                         # unknown mode
    assert kvq.kvq_page_bytes((4, 4, 0, 1), 128) == 0                      # fp8 needs 8/8 bits
    assert kvq.kvq_page_bytes((8, 8, 1, 1), 128) == 0                      # fp8 has no key mode
    assert kvq.kvq_page_bytes((8, 8, 0, 2), 128) == 0                      # unknown format
    assert kvq.kvq_equiv_bits([(4, 4, 1), (4, 2, 0)]) == 3.5               # the mode does not change bits
    pc = kvq.kvq_cache_pool_bytes([(4, 4)] * 2, 32, 8, 128, 16, 4097)
    pt = kvq.kvq_cache_pool_bytes([(4, 4, 1)] * 2, 32, 8, 128, 16, 4097)
    assert 0 < pt < pc


def test_fp8_pairs(kvq):
    for D in (64, 128):
        assert kvq.kvq_page_bytes((8, 8, 0, kvq.KVQ_FMT_FP8), D) == 64 * D   # e4m3 elements, no page metadata
    assert kvq.kvq_equiv_bits([(16, 16)] * 8 + [(8, 8, 0, 1)] * 24) == 10.0
    with pytest.raises(kvq.KVQError):
        kvq.kvq_cache_create([(8, 8, 1, 1)], 8, 8, 128, 4, 1024)


def test_pool_bytes_validation(kvq):
    good = kvq.kvq_cache_pool_bytes([(4, 4)] * 2, 32, 8, 128, 16, 4097)
    assert good > 2 * 16 * 8 * 128 * kvq.kvq_page_bytes((4, 4), 128)
    assert good % 256 == 0
    assert kvq.kvq_cache_pool_bytes([(4, 4)], 30, 8, 128, 16, 4097) == 0   # GQA not integral
    assert kvq.kvq_cache_pool_bytes([(4, 4)], 80, 8, 128, 16, 4097) == 0   # G = 10 > 8
    assert kvq.kvq_cache_pool_bytes([(4, 4)], 32, 8, 96, 16, 4097) == 0    # head_dim
    assert kvq.kvq_cache_pool_bytes([(4, 4)], 32, 8, 128, 0, 4097) == 0    # batch
    assert kvq.kvq_cache_pool_bytes([(5, 4)], 32, 8, 128, 16, 4097) == 0   # pair


def test_create_rejects_bad_arguments_before_touching_the_device(kvq):
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_create([(4, 6)], 8, 8, 128, 4, 1024)
    assert e.value.status == kvq.KVQ_EINVAL
    assert "unsupported pair" in str(e.value)
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_create([(4, 4)], 12, 8, 128, 4, 1024)
    assert e.value.status == kvq.KVQ_EINVAL


def test_null_cache_calls_fail_cleanly(kvq):
    import ctypes
    assert kvq.lib.kvq_sync(None) == kvq.KVQ_EINVAL
    assert kvq.lib.kvq_seq_len(None, 0, 0) == -1
    assert kvq.lib.kvq_bytes(None, 0, 1, 1) == -1
    assert kvq.lib.kvq_launch_count(None) == -1
    assert kvq.lib.kvq_decode_attn(None, 0, None, 1, None, None) == kvq.KVQ_EINVAL
    n = (ctypes.c_int32 * 1)(1)
    assert kvq.lib.kvq_append(None, 0, None, None, 0, n, 1, None) == kvq.KVQ_EINVAL
    assert kvq.lib.kvq_decode_step(None, 0, None, None, None, 1, None, None) == kvq.KVQ_EINVAL
    assert kvq.lib.kvq_set_decode_mode(None, -1) == kvq.KVQ_EINVAL
    kvq.kvq_cache_destroy(None)


def test_noalloc_rejects_bad_arguments_before_touching_the_device(kvq):
    """Every argument check of kvq_decode_attn_noalloc returns before any CUDA call
    (this machine may have no GPU), with the status its header comment gives."""
    import ctypes
    f = kvq.lib.kvq_decode_attn_noalloc
    A = 1 << 20  # a 16-byte aligned stand-in address (never dereferenced: every call below fails first)
    good = dict(pair=(4, 4), D=128, hq=32, hkv=8, pages=A, max_pages=128, window=A, seq_len=A, max_len=4096,
                Q=A, batch=16, out=A)

    def call(**kw):
        a = dict(good, **kw)
        return f(kvq._pair(a["pair"]), a["D"], a["hq"], a["hkv"], ctypes.c_void_p(a["pages"]), a["max_pages"],
                 ctypes.c_void_p(a["window"]), ctypes.c_void_p(a["seq_len"]), a["max_len"], ctypes.c_void_p(a["Q"]),
                 a["batch"], ctypes.c_void_p(a["out"]), None)

    E = kvq.KVQ_EINVAL
    assert call(pair=(3, 4)) == E                       # unsupported bits
    assert call(pair=(16, 8)) == E                      # mixed bf16 / int
    assert call(pair=(16, 16, 1)) == E                  # bf16 layer with a key mode
    assert call(pair=(8, 8, 0, 1)) == E                 # fp8 needs per-head scales (a cache)
    assert call(pair=(4, 4, 2)) == E                    # unknown key mode
    assert call(D=96) == E
    assert call(hq=30) == E and call(hq=80) == E and call(hkv=0) == E
    assert call(batch=0) == E and call(batch=1025) == E
    assert call(max_pages=-1) == E and call(max_len=-1) == E
    assert call(max_len=4097 + 32 * 128) == E           # max_seq_len/32 > max_pages
    assert call(max_pages=(1 << 25) + 1, max_len=0) == E
    for name in ("pages", "window", "seq_len", "Q", "out"):
        assert call(**{name: 0}) == E, name
    for name in ("pages", "window", "Q", "out"):
        assert call(**{name: A + 8}) == E, name         # not 16-byte aligned
    assert call(seq_len=A + 2) == E                     # not 4-byte aligned
    # more than 2^31 units: 1024 sequences x 64 heads x (2^25/32... pages + overhead)
    assert call(batch=1024, hq=64, hkv=64, max_pages=1 << 25, max_len=1 << 30) == E
    assert "too many pages" in kvq.lib.kvq_last_error().decode()
    # merge counters alone would fill the 16 MiB array
    assert call(batch=1024, hq=8192, hkv=8192, max_len=0) == kvq.KVQ_ECAPACITY
