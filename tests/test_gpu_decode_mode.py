"""Both work splits of the tensor-core decode kernel against the oracle.

With G <= 4 each warp may attend whole (sequence, KV head) segments (the warp
split: automatic for short sequences and many segments, or forced up to a page
limit), or the CTAs of a persistent grid share each segment's pages and merge
split records (the shared split). The
split changes only the rounding order, so both must meet the parity bar on the
same cache, and agree with each other within it.
"""

import numpy as np
import pytest

from test_gpu_parity import PAIRS, Pair, _check_attention, _inputs, _q, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu


def _attend_modes(P, kvq, Q, modes):
    outs = {}
    for m in modes:
        kvq.kvq_set_decode_mode(P.cache, m)
        outs[m], ref = P.attend(Q)
    return outs, ref


MODES = [0, -1, 1 << 20]  # shared split only, automatic (the default), one warp per segment at any length


@pytest.mark.parametrize("pair", PAIRS + [(4, 4, 1), (2, 8, 1), (8, 8, 0, 1)])
@pytest.mark.parametrize("G", [1, 3, 4])
def test_modes_short_and_ragged(kvq, oracle, pair, G):
    rng = np.random.default_rng(hash((pair, G, "modes")) % 2**32)
    batch, hkv, D = 9, 2, 128
    lens = [0, 1, 31, 32, 33, 64, 100, 255, 511]
    scales = ([0.5, 2.0], [1.5, 0.25]) if len(pair) > 3 else None
    P = Pair(kvq, oracle, pair, batch, hkv * G, hkv, D, 600, fp8_scales=scales)
    try:
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        K, V = _inputs(rng, batch, hkv, D)
        P.append(K, V, [1] * batch)
        P.check_pages()
        outs, ref = _attend_modes(P, kvq, _q(rng, batch, hkv * G, D), MODES)
        for m, got in outs.items():
            _check_attention(got, ref, f"{pair} G{G} mode {m}")
        _check_attention(outs[MODES[-1]], outs[0].astype(np.float64), f"{pair} G{G} warp vs shared")
    finally:
        P.close()


@pytest.mark.parametrize("D", [64, 128])
def test_warp_mode_long_sequences_and_many_segments(kvq, oracle, D):
    # long sequences forced through the warp split; 320 segments over the resident warps
    rng = np.random.default_rng(77 + D)
    batch, hkv, G = 40, 8, 4
    lens = [int(x) for x in rng.integers(0, 1400, size=batch)]
    P = Pair(kvq, oracle, (4, 2), batch, hkv * G, hkv, D, 1500)
    try:
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        Q = _q(rng, batch, hkv * G, D)
        outs, ref = _attend_modes(P, kvq, Q, [0, 1 << 20])
        for m, got in outs.items():
            _check_attention(got, ref, f"D{D} mode {m}")
    finally:
        P.close()


def test_decode_mode_rejects_negative(kvq):
    cache = kvq.kvq_cache_create([(4, 4)], 8, 2, 64, 1, 64)
    try:
        with pytest.raises(RuntimeError):
            kvq.kvq_set_decode_mode(cache, -2)
        for m in (-1, 0, 5):
            kvq.kvq_set_decode_mode(cache, m)
    finally:
        kvq.kvq_cache_destroy(cache)
