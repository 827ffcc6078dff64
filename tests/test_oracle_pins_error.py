"""Pins of the oracle's per-layer quantization error report.

The pages track quantization error layer by layer (OpenReview rebuttal, Table 3
and the layer-wise attention error figures it cites; key error matters more
than value error). The report holds sums over every flushed element of
(x - x_hat)^2 and x^2 for keys and values. Pinned by recomputing the sums from
the layer's own bf16 inputs and a numpy dequantization of the exported pages,
and by closed forms.
"""

import numpy as np
import pytest
import torch


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _kv(rng, n, H, D):
    K = rng.standard_normal((n, H, D)).astype(np.float32)
    K[:, :, 3] *= 10
    V = rng.standard_normal((n, H, D)).astype(np.float32)
    return _bf16(K), _bf16(V)


@pytest.mark.parametrize("pair,mode", [((2, 2), 0), ((4, 8), 0), ((4, 4), 1), ((8, 2), 1)])
def test_error_sums_recomputed(oracle, pair, mode):
    rng = np.random.default_rng(sum(pair) + 10 * mode)
    H, D, T = 2, 64, 75   # two flushed pages per head, 11 window tokens not counted
    K, V = _kv(rng, T, H, D)
    L = oracle.OracleLayer(*pair, 1, H, D, key_mode=mode)
    L.append(K, V, [T])
    ek, k2, ev, v2, n = L.error()
    assert n == H * 64 * D
    want = np.zeros(4)
    for h in range(H):
        Kh, Vh = L.dequant(0, h)           # window rows equal the inputs exactly
        want += [((Kh[:64] - K[:64, h]) ** 2).sum(), (K[:64, h].astype(np.float64) ** 2).sum(),
                 ((Vh[:64] - V[:64, h]) ** 2).sum(), (V[:64, h].astype(np.float64) ** 2).sum()]
    np.testing.assert_allclose([ek, k2, ev, v2], want, rtol=1e-12)
    # error bounds of the quantizer: at most (s/2)^2 per element
    assert 0 < ek < k2 and 0 < ev < v2


def test_error_closed_forms(oracle):
    H, D = 1, 64
    # constant channels/tokens of fp16-representable values are exact: zero error
    K = np.tile(np.linspace(-2, 2, D, dtype=np.float32), (32, H, 1))      # channel-constant keys
    V = np.full((32, H, D), 0.75, np.float32)                             # token-constant values
    L = oracle.OracleLayer(4, 4, 1, H, D)
    L.append(_bf16(K), _bf16(V), [32])
    ek, k2, ev, v2, n = L.error()
    assert ek == 0.0 and ev == 0.0 and n == 32 * D
    assert v2 == 32 * D * 0.75 ** 2
    # two-level values {0, 3} at 2 bits: z = 0, s = 1 -> exact
    V2 = np.where(np.arange(D) % 2 == 0, 0.0, 3.0).astype(np.float32)[None, None, :].repeat(32, 0)
    L2 = oracle.OracleLayer(4, 2, 1, H, D)
    L2.append(_bf16(K), V2, [32])
    assert L2.error()[2] == 0.0
    # nothing is counted before a page flushes, and bf16 layers add nothing
    L3 = oracle.OracleLayer(4, 4, 1, H, D)
    L3.append(_bf16(K[:31]), _bf16(V[:31]), [31])
    assert L3.error() == (0.0, 0.0, 0.0, 0.0, 0)
    Lb = oracle.OracleLayer(16, 16, 1, H, D)
    Lb.append(_bf16(K), _bf16(V), [32])
    assert Lb.error() == (0.0, 0.0, 0.0, 0.0, 0)


def test_error_orders_like_the_pages(oracle):
    # more bits, less error; per-channel keys beat per-token keys on channel
    # outliers (facts page, rebuttal section 4)
    rng = np.random.default_rng(3)
    H, D, T = 2, 128, 128
    K, V = _kv(rng, T, H, D)
    rel = {}
    for pair, mode in (((2, 2), 0), ((4, 4), 0), ((8, 8), 0), ((4, 4), 1)):
        L = oracle.OracleLayer(*pair, 1, H, D, key_mode=mode)
        L.append(K, V, [T])
        ek, k2, ev, v2, _ = L.error()
        rel[(pair, mode)] = (ek / k2, ev / v2)
    assert rel[((2, 2), 0)][0] > rel[((4, 4), 0)][0] > rel[((8, 8), 0)][0]
    assert rel[((2, 2), 0)][1] > rel[((4, 4), 0)][1] > rel[((8, 8), 0)][1]
    assert rel[((4, 4), 1)][0] > 2 * rel[((4, 4), 0)][0]
