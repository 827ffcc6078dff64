"""Decode launches whose page copies start under the preceding kernel's tail.

With the lengths in the launch parameters, a decode (or fused step) kernel may
copy pages below those lengths before the kernel launched right before it on
the stream has finished, unless that kernel is one of the cache's own that
wrote the same layer. This is the pattern of a layer-stack decode step (layer
l's kernel follows layer l-1's): every launch below except the first of each
pair takes the early path, and the results must match the oracle's as in any
other order.
"""

import numpy as np
import pytest
import torch

from test_gpu_parity import Pair, _check_attention, _inputs, _q, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pairs,G", [([(4, 4), (4, 2)], 4), ([(8, 8), (16, 16)], 4), ([(4, 4), (8, 4, 1)], 7)])
def test_alternating_layers(kvq, oracle, pairs, G):
    rng = np.random.default_rng(61 + G)
    B, hkv, D = 6, 2, 128
    lens = [31, 90, 200, 0, 64, 129]
    cache = kvq.kvq_cache_create(pairs, hkv * G, hkv, D, B, 320)
    refs = []
    try:
        kvq.kvq_set_decode_mode(cache, 0)  # the shared split (the one with early copies)
        for layer, pair in enumerate(pairs):
            ref = oracle.OracleLayer(pair[0], pair[1], B, hkv, D, key_mode=pair[2] if len(pair) > 2 else 0)
            K, V = _inputs(rng, sum(lens), hkv, D)
            kvq.kvq_append(cache, layer, torch.from_numpy(K).cuda().bfloat16(),
                           torch.from_numpy(V).cuda().bfloat16(), lens)
            ref.append(K, V, lens)
            refs.append(ref)
        out = torch.empty((B, hkv * G, D), device="cuda", dtype=torch.float32)
        for step in range(40):
            for layer in range(len(pairs)):
                K, V = _inputs(rng, B, hkv, D)
                Q = _q(rng, B, hkv * G, D)
                Qt = torch.from_numpy(Q).cuda().bfloat16()
                kvq.kvq_decode_step(cache, layer, torch.from_numpy(K).cuda().bfloat16(),
                                    torch.from_numpy(V).cuda().bfloat16(), Qt, out)
                refs[layer].append(K, V, [1] * B)
                if step % 9 == 0 or step == 39:
                    torch.cuda.synchronize()
                    _check_attention(out.cpu().numpy(), refs[layer].attend(Q), f"step {step} layer {layer}")
                    # a second decode of the same layer right after: its predecessor wrote
                    # this layer (no early copies); a third: the predecessor only read it
                    for _ in range(2):
                        kvq.kvq_decode_attn(cache, layer, Qt, out)
                        torch.cuda.synchronize()
                        _check_attention(out.cpu().numpy(), refs[layer].attend(Q), f"re-read {step} {layer}")
        for layer in range(len(pairs)):
            np.testing.assert_array_equal(kvq.kvq_export_layer(cache, layer, B), refs[layer].export(B))
        kvq.kvq_sync(cache)
    finally:
        kvq.kvq_cache_destroy(cache)
