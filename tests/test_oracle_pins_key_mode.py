"""Pins of the oracle's per-token key mode against the pages and mathematics.

Per-token asymmetric keys (one scale/zero per key token over the head
dimension) are the second key mode the KVTuner pages compare with the
per-channel (KIVI-like) one: OpenReview rebuttal, section 4 "Per-channel vs.
per-token quantization"; facts page: per-channel asymmetric beats per-token
asymmetric for keys because keys carry channel-wise outliers, and the Pareto
pairs differ between the modes. Nothing here re-calls the oracle's quantizer to
produce an expected value: scales and zeros are parsed from the page bytes with
the documented layout and every code is checked by brute force.
"""

import numpy as np
import pytest
import torch

PT = 1  # per-token key mode
PAIRS = [(2, 2), (4, 2), (4, 4), (8, 4), (4, 8), (8, 8)]


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _bits(x):
    return (_bf16(x).view(np.uint32) >> 16).astype(np.uint16)


def _f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _meta(page, D, kb, vb):
    """Key scales/zeros (32 each, token order) and value scales/zeros of a
    per-token-key page: [K codes][V codes][K s][K z][V s][V z] (fp16)."""
    off = 32 * D * kb // 8 + 32 * D * vb // 8
    m = page[off:off + 256].view(np.uint16)
    return _f16(m[0:32]), _f16(m[32:64]), _f16(m[64:96]), _f16(m[96:128])


def _page_inputs(rng, D, outliers=True):
    K = rng.standard_normal((32, D)).astype(np.float32)
    if outliers:
        K[:, [3, 17]] *= 10
    V = rng.standard_normal((32, D)).astype(np.float32)
    return _bf16(K), _bf16(V)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("pair", PAIRS)
def test_per_token_key_codes_brute_force(oracle, D, pair):
    kb, vb = pair
    qmax = (1 << kb) - 1
    rng = np.random.default_rng(kb * 10 + vb + D)
    for trial in range(3):
        K, V = _page_inputs(rng, D)
        page = oracle.build_page(_bits(K), _bits(V), D, kb, vb, key_mode=PT)
        assert page.size == 32 * D * (kb + vb) // 8 + 256
        ks, kz, _, _ = _meta(page, D, kb, vb)
        codes = oracle.unpack_block(page[:32 * D * kb // 8], D, kb, False).astype(np.int64)
        assert codes.max() <= qmax
        for t in range(32):
            x = K[t].astype(np.float64)
            s, z = ks[t], kz[t]
            # the stored range covers the token: z <= min, z + qmax s >= max
            assert z <= x.min() and z + qmax * s >= x.max() * (1 - 2 ** -20)
            # each code is a nearest level of this token's own (s, z)
            levels = np.arange(qmax + 1) * s + z
            dist = np.abs(x[:, None] - levels[None, :])
            slack = s * qmax * 2.0 ** -21 + np.abs(x) * 2.0 ** -22
            assert np.all(dist[np.arange(D), codes[t]] <= dist.min(1) + slack)
            # the token's extremes take the end codes (grouping is along channels)
            if s >= 2.0 ** -14:
                assert codes[t, np.argmin(x)] == 0 and codes[t, np.argmax(x)] == qmax


@pytest.mark.parametrize("pair", PAIRS)
def test_per_token_key_round_trip_and_values_unchanged(oracle, pair):
    kb, vb = pair
    D = 128
    rng = np.random.default_rng(40 + kb + vb)
    K, V = _page_inputs(rng, D)
    pt = oracle.build_page(_bits(K), _bits(V), D, kb, vb, key_mode=PT)
    pc = oracle.build_page(_bits(K), _bits(V), D, kb, vb)
    Kh, Vh = oracle.dequant_page(pt, D, kb, vb, key_mode=PT)
    ks = _meta(pt, D, kb, vb)[0]
    assert np.all(np.abs(Kh - K) <= (ks / 2)[:, None] * (1 + 2 ** -9) + 1e-6)
    # values do not depend on the key mode: same V code block, same V metadata
    kcb, vcb = 32 * D * kb // 8, 32 * D * vb // 8
    np.testing.assert_array_equal(pt[kcb:kcb + vcb], pc[kcb:kcb + vcb])
    np.testing.assert_array_equal(pt[-128:], pc[-128:])
    np.testing.assert_array_equal(Vh, oracle.dequant_page(pc, D, kb, vb)[1])


def test_per_token_constant_token_exact(oracle):
    D = 64
    rng = np.random.default_rng(3)
    K, V = _page_inputs(rng, D)
    K[5] = 1.5
    K[9] = -0.25
    page = oracle.build_page(_bits(K), _bits(V), D, 4, 4, key_mode=PT)
    ks, kz, _, _ = _meta(page, D, 4, 4)
    Kh = oracle.dequant_page(page, D, 4, 4, key_mode=PT)[0]
    for t, v in ((5, 1.5), (9, -0.25)):
        assert ks[t] == 0.0 and kz[t] == v
        assert np.all(Kh[t] == v)


def test_per_token_byte_accounting(oracle):
    # per token per KV head: codes D (k + v)/8, key (s, z) 4 B, value (s, z) 4 B
    for kb, vb in PAIRS:
        assert oracle.page_bytes(kb, vb, 128, key_mode=PT) == 4 * 128 * (kb + vb) + 256
        assert oracle.layer_bytes(kb, vb, 1000, 8, 128, with_meta=True, key_mode=PT) == \
            1000 * 8 * (128 * (kb + vb) // 8 + 8)
        # codes-only count is the same in both modes (equivalent bits ignore metadata)
        assert oracle.layer_bytes(kb, vb, 1000, 8, 128, key_mode=PT) == oracle.layer_bytes(kb, vb, 1000, 8, 128)
    # a bf16 layer has no key mode
    assert oracle.page_bytes(16, 16, 128, key_mode=PT) == oracle.page_bytes(16, 16, 128)


@pytest.mark.parametrize("bits", [2, 4])
def test_per_channel_beats_per_token_on_channel_outliers(oracle, bits):
    # facts page / OpenReview section 4: keys carry channel-wise outliers, so
    # per-channel asymmetric keys reconstruct them better than per-token ones.
    rng = np.random.default_rng(100 + bits)
    D, pages = 128, 16
    err = {0: 0.0, PT: 0.0}
    for _ in range(pages):
        K, V = _page_inputs(rng, D)
        for mode in err:
            page = oracle.build_page(_bits(K), _bits(V), D, bits, 4, key_mode=mode)
            Kh = oracle.dequant_page(page, D, bits, 4, key_mode=mode)[0]
            err[mode] += float(((Kh - K) ** 2).sum())
    assert err[0] < 0.5 * err[PT], err


def _kv(rng, n, H, D):
    K = rng.standard_normal((n, H, D)).astype(np.float32)
    K[:, :, 3] *= 10
    V = rng.standard_normal((n, H, D)).astype(np.float32)
    return _bf16(K), _bf16(V)


@pytest.mark.parametrize("pair", [(8, 4), (2, 2), (4, 8)])
def test_per_token_window_chunking_invariance(oracle, pair):
    rng = np.random.default_rng(5)
    H, D, T = 2, 64, 97
    K, V = _kv(rng, T, H, D)
    whole = oracle.OracleLayer(*pair, 1, H, D, key_mode=PT)
    whole.append(K, V, [T])
    ones = oracle.OracleLayer(*pair, 1, H, D, key_mode=PT)
    for i in range(T):
        ones.append(K[i:i + 1], V[i:i + 1], [1])
    a, b = whole.export(), ones.export()
    np.testing.assert_array_equal(a, b)
    pb = oracle.page_bytes(*pair, D, key_mode=PT)
    assert a.size == H * ((T // 32) * pb + 2 * (T % 32) * D * 2)
    # keys of a per-token page are quantized token by token: the first page of
    # a per-token layer equals a page built from the same 32 tokens alone
    first = oracle.build_page(_bits(K[:32, 0]), _bits(V[:32, 0]), D, *pair, key_mode=PT)
    np.testing.assert_array_equal(a[:pb], first)


def _dequant_numpy(oracle, page, D, kb, vb):
    """Dequantization of a per-token-key page written out in numpy (fp64); only
    the bit unpacking (pinned by the pack/unpack identity) is the oracle's."""
    kc = oracle.unpack_block(page[:32 * D * kb // 8], D, kb, False).astype(np.float64)
    vc = oracle.unpack_block(page[32 * D * kb // 8:32 * D * (kb + vb) // 8], D, vb, True).astype(np.float64)
    ks, kz, vs, vz = _meta(page, D, kb, vb)
    return kc * ks[:, None] + kz[:, None], vc * vs[:, None] + vz[:, None]


@pytest.mark.parametrize("pair", [(4, 4), (2, 8), (8, 2)])
@pytest.mark.parametrize("G", [1, 4])
def test_per_token_attention_brute_force(oracle, pair, G):
    rng = np.random.default_rng(pair[0] * 7 + pair[1] + G)
    H, D, T = 2, 64, 75
    K, V = _kv(rng, T, H, D)
    L = oracle.OracleLayer(*pair, 1, H, D, key_mode=PT)
    L.append(K, V, [T])
    Q = _bf16(rng.standard_normal((1, H * G, D)))
    out = L.attend(Q)
    ex = L.export()
    pb = oracle.page_bytes(*pair, D, key_mode=PT)
    per_head = 2 * pb + 2 * (T % 32) * D * 2
    for h in range(H):
        blob = ex[h * per_head:(h + 1) * per_head]
        Ks, Vs = [], []
        for pg in range(2):
            k_, v_ = _dequant_numpy(oracle, blob[pg * pb:(pg + 1) * pb], D, *pair)
            Ks.append(k_)
            Vs.append(v_)
        win = blob[2 * pb:].view(np.uint16)
        W = T % 32
        Ks.append((win[:W * D].astype(np.uint32) << 16).view(np.float32).reshape(W, D).astype(np.float64))
        Vs.append((win[W * D:].astype(np.uint32) << 16).view(np.float32).reshape(W, D).astype(np.float64))
        Kd, Vd = np.concatenate(Ks), np.concatenate(Vs)
        for gq in range(G):
            q = Q[0, h * G + gq].astype(np.float64)
            s = Kd @ q / np.sqrt(D)
            p = np.exp(s - s.max())
            ref = (p[:, None] * Vd).sum(0) / p.sum()
            np.testing.assert_allclose(out[0, h * G + gq], ref, rtol=0, atol=1e-12)


def test_per_token_attention_closed_forms(oracle):
    rng = np.random.default_rng(12)
    H, D, T = 1, 64, 70
    K, V = _kv(rng, T, H, D)
    L = oracle.OracleLayer(4, 4, 1, H, D, key_mode=PT)
    L.append(K, V, [T])
    Vd = L.dequant(0, 0)[1]
    out = L.attend(np.zeros((1, 1, D), dtype=np.float32))
    np.testing.assert_allclose(out[0, 0], Vd.mean(0), rtol=0, atol=1e-12)
    # all key tokens equal and all quantized (T a multiple of 32): per-token
    # quantization maps them to one vector, so every score is equal and the
    # output is the mean of the values
    Le = oracle.OracleLayer(2, 8, 1, H, D, key_mode=PT)
    Le.append(np.repeat(K[:1], 64, axis=0), V[:64], [64])
    out = Le.attend(_bf16(rng.standard_normal((1, 1, D))))
    np.testing.assert_allclose(out[0, 0], Le.dequant(0, 0)[1].mean(0), rtol=0, atol=1e-12)
