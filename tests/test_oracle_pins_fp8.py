"""Pins of the oracle's FP8 (e4m3) layer format against the pages, mathematics
and an independent library routine (torch's float8_e4m3fn conversion).

The pages' FP8 facts: machinoai Q&A section 2 worked example (32 layers, 8 kept
in BF16 and 24 in FP8 = 2,000 MiB, a 37.5% saving, FP8 layer half a BF16 one);
llms-explorer facts page (vLLM FP8 KV cache with per-attention-head scales and
BF16 skip layers). Format: each element of KV head h stored as e4m3(x / s_h),
round to nearest even, saturating at 448; value e4m3 * s_h.
"""

import numpy as np
import pytest
import torch

FP8 = 1


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _bits(x):
    return (_bf16(x).view(np.uint32) >> 16).astype(np.uint16)


def _torch_e4m3(x):
    """torch's fp32 -> e4m3 bit patterns (round to nearest even; NaN past 464)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_values_match_torch(oracle):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(v) and c & 0x7F == 0x7F
        else:
            assert v == ref[c], (c, v, ref[c])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_torch_in_range(oracle):
    rng = np.random.default_rng(8)
    grid = np.array([oracle.e4m3_value(c) for c in range(256) if c & 0x7F != 0x7F])
    pos = np.unique(np.abs(grid))
    mids = (pos[1:] + pos[:-1]) / 2                     # exact ties -> even mantissa
    xs = np.concatenate([grid, mids, -mids, pos[1:] * (1 + 1e-3), pos[1:] * (1 - 1e-3),
                         rng.standard_normal(4000) * 30, rng.uniform(-2e-3, 2e-3, 2000),
                         [0.0, -0.0, 449.0, 463.9, -463.9, 464.0]]).astype(np.float32)
    got = np.array([oracle.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    np.testing.assert_array_equal(got, _torch_e4m3(xs))


def test_e4m3_saturates_above_448(oracle):
    for x in (464.0, 465.0, 1000.0, 3.0e38, float("inf")):
        assert oracle.e4m3_encode(x) == 0x7E
        assert oracle.e4m3_encode(-x) == 0xFE


def test_worked_example_fp8_exact_with_metadata(oracle):
    # 32 layers, 8 BF16 + 24 FP8, head_dim 128, 8 KV heads, 25,600 tokens: the
    # FP8 format carries no per-page metadata, so the count with metadata is
    # exactly the pages' 2,000 MiB (BF16 layer 100 MiB, FP8 layer 50 MiB).
    MiB = 1 << 20
    bf16 = oracle.layer_bytes(16, 16, 25600, 8, 128, with_meta=True)
    fp8 = oracle.layer_bytes(8, 8, 25600, 8, 128, with_meta=True, fmt=FP8)
    assert bf16 == 100 * MiB and fp8 == 50 * MiB
    total = 8 * bf16 + 24 * fp8
    assert total == 2000 * MiB
    assert 1 - total / (32 * bf16) == 0.375
    assert oracle.page_bytes(8, 8, 128, fmt=FP8) == 64 * 128


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("ks,vs", [(1.0, 1.0), (0.0390625, 0.5), (3.0, 0.0078125)])
def test_fp8_page_codes_and_round_trip(oracle, D, ks, vs):
    rng = np.random.default_rng(int(D + 100 * ks + 1000 * vs))
    K = rng.standard_normal((32, D)).astype(np.float32)
    K[:, 5] *= 40
    V = (rng.standard_normal((32, D)) * 2).astype(np.float32)
    K, V = _bf16(K), _bf16(V)
    page = oracle.build_page(_bits(K), _bits(V), D, 8, 8, fmt=FP8, k_scale=ks, v_scale=vs)
    assert page.size == 64 * D
    kc = oracle.unpack_block(page[:32 * D], D, 8, False).astype(np.uint8)
    vc = oracle.unpack_block(page[32 * D:], D, 8, True).astype(np.uint8)
    for codes, x, s in ((kc, K, ks), (vc, V, vs)):
        y = (x / np.float32(s)).astype(np.float32)      # one fp32 division per element
        want = _torch_e4m3(y)
        sat = np.abs(y) >= 464
        want[sat] = np.where(y[sat] > 0, 0x7E, 0xFE)
        np.testing.assert_array_equal(codes, want)
    Kh, Vh = oracle.dequant_page(page, D, 8, 8, fmt=FP8, k_scale=ks, v_scale=vs)
    for xh, x, s in ((Kh, K, ks), (Vh, V, vs)):
        y = np.abs(x.astype(np.float64) / s)
        ok = y < 448
        # half an e4m3 step: 2^-4 relative for normals, 2^-10 absolute below 2^-6
        step = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3), 2.0 ** -9)
        assert np.all(np.abs(xh[ok] / s - x[ok] / s) <= step[ok] / 2 * (1 + 1e-9))


def _kv(rng, n, H, D):
    K = rng.standard_normal((n, H, D)).astype(np.float32)
    K[:, :, 3] *= 10
    V = rng.standard_normal((n, H, D)).astype(np.float32)
    return _bf16(K), _bf16(V)


def test_fp8_chunking_invariance_and_per_head_scales(oracle):
    rng = np.random.default_rng(21)
    H, D, T = 2, 64, 97
    ksc, vsc = np.array([0.25, 2.0], np.float32), np.array([1.0, 0.125], np.float32)
    K, V = _kv(rng, T, H, D)
    whole = oracle.OracleLayer(8, 8, 1, H, D, fmt=FP8, k_scales=ksc, v_scales=vsc)
    whole.append(K, V, [T])
    ones = oracle.OracleLayer(8, 8, 1, H, D, fmt=FP8, k_scales=ksc, v_scales=vsc)
    for i in range(T):
        ones.append(K[i:i + 1], V[i:i + 1], [1])
    a = whole.export()
    np.testing.assert_array_equal(a, ones.export())
    pb = oracle.page_bytes(8, 8, D, fmt=FP8)
    assert a.size == H * ((T // 32) * pb + 2 * (T % 32) * D * 2)
    # head h's pages use head h's scales
    for h in range(H):
        first = oracle.build_page(_bits(K[:32, h]), _bits(V[:32, h]), D, 8, 8, fmt=FP8, k_scale=ksc[h],
                                  v_scale=vsc[h])
        off = h * (3 * pb + 2 * (T % 32) * D * 2)
        np.testing.assert_array_equal(a[off:off + pb], first)


@pytest.mark.parametrize("G", [1, 4, 7])
def test_fp8_attention_brute_force(oracle, G):
    rng = np.random.default_rng(30 + G)
    H, D, T = 2, 64, 75
    ksc, vsc = np.array([0.5, 0.03125], np.float32), np.array([0.25, 1.5], np.float32)
    K, V = _kv(rng, T, H, D)
    L = oracle.OracleLayer(8, 8, 1, H, D, fmt=FP8, k_scales=ksc, v_scales=vsc)
    L.append(K, V, [T])
    Q = _bf16(rng.standard_normal((1, H * G, D)))
    out = L.attend(Q)
    pb = oracle.page_bytes(8, 8, D, fmt=FP8)
    ex = L.export()
    per_head = 2 * pb + 2 * (T % 32) * D * 2
    val = np.array([oracle.e4m3_value(c) for c in range(256)])
    for h in range(H):
        blob = ex[h * per_head:(h + 1) * per_head]
        Ks, Vs = [], []
        for pg in range(2):
            pgb = blob[pg * pb:(pg + 1) * pb]
            Ks.append(val[oracle.unpack_block(pgb[:32 * D], D, 8, False)] * float(ksc[h]))
            Vs.append(val[oracle.unpack_block(pgb[32 * D:], D, 8, True)] * float(vsc[h]))
        W = T % 32
        win = blob[2 * pb:].view(np.uint16)
        Ks.append((win[:W * D].astype(np.uint32) << 16).view(np.float32).reshape(W, D).astype(np.float64))
        Vs.append((win[W * D:].astype(np.uint32) << 16).view(np.float32).reshape(W, D).astype(np.float64))
        Kd, Vd = np.concatenate(Ks), np.concatenate(Vs)
        for gq in range(G):
            q = Q[0, h * G + gq].astype(np.float64)
            s = Kd @ q / np.sqrt(D)
            p = np.exp(s - s.max())
            np.testing.assert_allclose(out[0, h * G + gq], (p[:, None] * Vd).sum(0) / p.sum(), rtol=0, atol=1e-12)
