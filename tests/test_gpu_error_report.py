"""GPU parity of the per-layer quantization error report (kvq_layer_error)
with the oracle's: same element counts, sums within the rounding of the GPU's
per-element terms (fp32 in the append kernel for groups of moderate magnitude,
fp64 otherwise and in the fused step's flush) and of the summation order."""

import numpy as np
import pytest
import torch

from test_gpu_parity import Pair, _inputs, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu


def _same_report(got, want):
    # the append kernel forms each element's terms in fp32 for groups of
    # moderate magnitude: a dx moves by at most 2^-24 |x - z| with |x - z| <=
    # (qmax + 1) s, i.e. at most about 2^-23 * 256 * 3 < 1e-4 relative on the
    # sum of dx^2 for 8-bit codes (fp32 summation over <= 32 terms adds ~2e-6)
    assert got[4] == want[4]
    np.testing.assert_allclose(got[:4], want[:4], rtol=1e-4, atol=0)


@pytest.mark.parametrize("pair", [(2, 2), (4, 8), (8, 4), (4, 4, 1), (2, 8, 1), (8, 8, 0, 1), (16, 16)])
@pytest.mark.parametrize("D", [64, 128])
def test_error_report_matches_oracle(kvq, oracle, pair, D):
    rng = np.random.default_rng(hash((pair, D, "err")) % 2**32)
    batch, hkv = 3, 2
    scales = ([0.05, 0.2], [0.02, 0.5]) if len(pair) > 3 else None
    P = Pair(kvq, oracle, pair, batch, hkv * 4, hkv, D, 256, fp8_scales=scales)
    try:
        K, V = _inputs(rng, 150, hkv, D)
        P.append(K, V, [30, 64, 56])
        _same_report(kvq.kvq_layer_error(P.cache, 0), P.ref.error())
        for _ in range(40):   # decode-style appends cross more page boundaries
            K, V = _inputs(rng, batch, hkv, D)
            P.append(K, V, [1] * batch)
        got, want = kvq.kvq_layer_error(P.cache, 0), P.ref.error()
        _same_report(got, want)
        if pair == (16, 16):
            assert got == (0.0, 0.0, 0.0, 0.0, 0)
        else:
            # (2-bit per-token keys on outlier channels can lose more than the signal)
            assert got[4] > 0 and got[0] > 0 and 0 < got[2] < got[3]
        kvq.kvq_cache_reset(P.cache)
        assert kvq.kvq_layer_error(P.cache, 0) == (0.0, 0.0, 0.0, 0.0, 0)
    finally:
        P.close()


@pytest.mark.parametrize("scale", [1e13, 1e-13, 3e4])
@pytest.mark.parametrize("pair", [(4, 4), (8, 2), (2, 8, 1)])
def test_error_report_at_extreme_magnitudes(kvq, oracle, pair, scale):
    # groups with magnitudes outside [2^-14, 2^40) take the fp64 terms (1e-13:
    # below fp16's resolution, where z and s are coarse next to the data); 3e4
    # (beyond fp16's range) takes the clamping path
    rng = np.random.default_rng(hash((pair, scale, "err-x")) % 2**32)
    batch, hkv, D = 2, 2, 64
    P = Pair(kvq, oracle, pair, batch, hkv * 4, hkv, D, 200)
    try:
        K, V = _inputs(rng, 160, hkv, D)
        K = torch.from_numpy(K * scale).to(torch.bfloat16).float().numpy()
        V = torch.from_numpy(V * scale).to(torch.bfloat16).float().numpy()
        P.append(K, V, [96, 64])
        P.check_pages()
        _same_report(kvq.kvq_layer_error(P.cache, 0), P.ref.error())
    finally:
        P.close()
