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
