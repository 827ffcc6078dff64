"""A decode step (one-token append + decode attention for each layer) captured
in a CUDA graph and replayed matches the oracle step for step; the host's
length mirror catches up with kvq_refresh_lengths; a replay past max_tokens
leaves the full sequences unchanged and kvq_sync reports KVQ_ECAPACITY."""

import numpy as np
import pytest
import torch

from test_gpu_parity import _check_attention, _inputs, _q, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu


def _setup(kvq, oracle, layer_map, B, hkv, G, D, max_tokens, lens, rng):
    cache = kvq.kvq_cache_create(layer_map, hkv * G, hkv, D, B, max_tokens)
    refs = []
    for layer, pair in enumerate(layer_map):
        ref = oracle.OracleLayer(pair[0], pair[1], B, hkv, D, key_mode=pair[2] if len(pair) > 2 else 0)
        K, V = _inputs(rng, sum(lens), hkv, D)
        kvq.kvq_append(cache, layer, torch.from_numpy(K).cuda().bfloat16(), torch.from_numpy(V).cuda().bfloat16(),
                       lens)
        ref.append(K, V, lens)
        refs.append(ref)
    return cache, refs


def _capture(kvq, cache, n_layers, B, Kb, Vb, Qb, Ob):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for layer in range(n_layers):
            kvq.kvq_append(cache, layer, Kb[layer], Vb[layer], [1] * B)
            kvq.kvq_decode_attn(cache, layer, Qb[layer], Ob[layer])
    torch.cuda.current_stream().wait_stream(s)
    return g


def test_graph_replay_matches_oracle(kvq, oracle):
    rng = np.random.default_rng(31)
    layer_map = [(4, 4), (2, 8, 1)]
    B, hkv, G, D = 4, 2, 4, 128
    lens = [40, 63, 64, 100]
    cache, refs = _setup(kvq, oracle, layer_map, B, hkv, G, D, 256, lens, rng)
    try:
        Kb = [torch.empty((B, hkv, D), device="cuda", dtype=torch.bfloat16) for _ in layer_map]
        Vb = [torch.empty_like(k) for k in Kb]
        Qb = [torch.empty((B, hkv * G, D), device="cuda", dtype=torch.bfloat16) for _ in layer_map]
        Ob = [torch.empty((B, hkv * G, D), device="cuda", dtype=torch.float32) for _ in layer_map]

        def fill(step_inputs):
            for layer, (K, V, Q) in enumerate(step_inputs):
                Kb[layer].copy_(torch.from_numpy(K))
                Vb[layer].copy_(torch.from_numpy(V))
                Qb[layer].copy_(torch.from_numpy(Q))

        def draw():
            out = []
            for _ in layer_map:
                K, V = _inputs(rng, B, hkv, D)
                out.append((K, V, _q(rng, B, hkv * G, D)))
            return out

        # eager warm-up step (also initialises the kernels' launch attributes)
        step = draw()
        fill(step)
        for layer in range(len(layer_map)):
            kvq.kvq_append(cache, layer, Kb[layer], Vb[layer], [1] * B)
            kvq.kvq_decode_attn(cache, layer, Qb[layer], Ob[layer])
            refs[layer].append(step[layer][0], step[layer][1], [1] * B)
        torch.cuda.synchronize()
        g = _capture(kvq, cache, len(layer_map), B, Kb, Vb, Qb, Ob)
        for it in range(30):
            step = draw()
            fill(step)
            g.replay()
            torch.cuda.synchronize()
            for layer in range(len(layer_map)):
                refs[layer].append(step[layer][0], step[layer][1], [1] * B)
                if it % 7 == 0 or it == 29:
                    _check_attention(Ob[layer].cpu().numpy(), refs[layer].attend(step[layer][2]),
                                     f"replay {it} layer {layer}")
        kvq.kvq_sync(cache)
        kvq.kvq_refresh_lengths(cache)
        for layer in range(len(layer_map)):
            for b in range(B):
                assert kvq.kvq_seq_len(cache, layer, b) == lens[b] + 31
            np.testing.assert_array_equal(kvq.kvq_export_layer(cache, layer, B), refs[layer].export(B))
        del g
    finally:
        kvq.kvq_cache_destroy(cache)


def test_graph_replay_stops_at_capacity(kvq, oracle):
    rng = np.random.default_rng(32)
    B, hkv, G, D = 2, 2, 4, 64
    lens = [60, 29]
    max_tokens = 64
    cache, refs = _setup(kvq, oracle, [(8, 4)], B, hkv, G, D, max_tokens, lens, rng)
    try:
        Kb = [torch.zeros((B, hkv, D), device="cuda", dtype=torch.bfloat16)]
        Vb = [torch.zeros_like(Kb[0])]
        Qb = [torch.zeros((B, hkv * G, D), device="cuda", dtype=torch.bfloat16)]
        Ob = [torch.zeros((B, hkv * G, D), device="cuda", dtype=torch.float32)]
        kvq.kvq_decode_attn(cache, 0, Qb[0], Ob[0])      # warm-up of the launch attributes
        torch.cuda.synchronize()
        g = _capture(kvq, cache, 1, B, Kb, Vb, Qb, Ob)
        for it in range(6):
            K, V = _inputs(rng, B, hkv, D)
            Kb[0].copy_(torch.from_numpy(K))
            Vb[0].copy_(torch.from_numpy(V))
            g.replay()
            torch.cuda.synchronize()
            # the oracle appends only while a sequence has room
            for b in range(B):
                if lens[b] + it < max_tokens:
                    refs[0].append(K[b:b + 1], V[b:b + 1], [0] * b + [1] + [0] * (B - b - 1))
        with pytest.raises(kvq.KVQError) as e:
            kvq.kvq_sync(cache)
        assert e.value.status == kvq.KVQ_ECAPACITY
        kvq.kvq_refresh_lengths(cache)
        assert [kvq.kvq_seq_len(cache, 0, b) for b in range(B)] == [64, 35]
        np.testing.assert_array_equal(kvq.kvq_export_layer(cache, 0, B), refs[0].export(B))
        kvq.kvq_sync(cache)                              # the flag was cleared
        del g
    finally:
        kvq.kvq_cache_destroy(cache)


@pytest.mark.parametrize("mode", [0, 1 << 20])
def test_graph_of_fused_steps_matches_oracle(kvq, oracle, mode):
    """kvq_decode_step captured per layer (one kernel per layer-step; the shared
    split reads the device lengths and its last CTA publishes the new ones, the
    warp split publishes per sequence), replayed across group completions."""
    rng = np.random.default_rng(33 + mode)
    layer_map = [(4, 4), (8, 2, 1), (16, 16)]
    B, hkv, G, D = 3, 2, 4, 128
    lens = [30, 62, 95]
    cache, refs = _setup(kvq, oracle, layer_map, B, hkv, G, D, 200, lens, rng)
    try:
        kvq.kvq_set_decode_mode(cache, mode)
        Kb = [torch.empty((B, hkv, D), device="cuda", dtype=torch.bfloat16) for _ in layer_map]
        Vb = [torch.empty_like(k) for k in Kb]
        Qb = [torch.empty((B, hkv * G, D), device="cuda", dtype=torch.bfloat16) for _ in layer_map]
        Ob = [torch.empty((B, hkv * G, D), device="cuda", dtype=torch.float32) for _ in layer_map]

        def step_inputs():
            out = []
            for layer in range(len(layer_map)):
                K, V = _inputs(rng, B, hkv, D)
                Q = _q(rng, B, hkv * G, D)
                Kb[layer].copy_(torch.from_numpy(K))
                Vb[layer].copy_(torch.from_numpy(V))
                Qb[layer].copy_(torch.from_numpy(Q))
                out.append((K, V, Q))
            return out

        st = step_inputs()
        for layer in range(len(layer_map)):   # eager step (launch attributes)
            kvq.kvq_decode_step(cache, layer, Kb[layer], Vb[layer], Qb[layer], Ob[layer])
            refs[layer].append(st[layer][0], st[layer][1], [1] * B)
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for layer in range(len(layer_map)):
                kvq.kvq_decode_step(cache, layer, Kb[layer], Vb[layer], Qb[layer], Ob[layer])
        torch.cuda.current_stream().wait_stream(s)
        for it in range(35):
            st = step_inputs()
            g.replay()
            torch.cuda.synchronize()
            for layer in range(len(layer_map)):
                refs[layer].append(st[layer][0], st[layer][1], [1] * B)
                if it % 5 == 0 or it == 34:
                    _check_attention(Ob[layer].cpu().numpy(), refs[layer].attend(st[layer][2]),
                                     f"mode {mode} replay {it} layer {layer}")
        kvq.kvq_sync(cache)
        kvq.kvq_refresh_lengths(cache)
        for layer in range(len(layer_map)):
            for b in range(B):
                assert kvq.kvq_seq_len(cache, layer, b) == lens[b] + 36
            np.testing.assert_array_equal(kvq.kvq_export_layer(cache, layer, B), refs[layer].export(B))
        del g
    finally:
        kvq.kvq_cache_destroy(cache)


def test_graph_of_fused_steps_stops_at_capacity(kvq, oracle):
    rng = np.random.default_rng(34)
    B, hkv, G, D = 2, 2, 4, 64
    lens = [60, 29]
    max_tokens = 64
    cache, refs = _setup(kvq, oracle, [(8, 4)], B, hkv, G, D, max_tokens, lens, rng)
    try:
        kvq.kvq_set_decode_mode(cache, 0)
        Kb = torch.zeros((B, hkv, D), device="cuda", dtype=torch.bfloat16)
        Vb = torch.zeros_like(Kb)
        Qb = torch.zeros((B, hkv * G, D), device="cuda", dtype=torch.bfloat16)
        Ob = torch.zeros((B, hkv * G, D), device="cuda", dtype=torch.float32)
        kvq.kvq_decode_attn(cache, 0, Qb, Ob)      # warm-up of the launch attributes
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            kvq.kvq_decode_step(cache, 0, Kb, Vb, Qb, Ob)
        torch.cuda.current_stream().wait_stream(s)
        for it in range(6):
            K, V = _inputs(rng, B, hkv, D)
            Kb.copy_(torch.from_numpy(K))
            Vb.copy_(torch.from_numpy(V))
            g.replay()
            torch.cuda.synchronize()
            for b in range(B):
                if lens[b] + it < max_tokens:
                    refs[0].append(K[b:b + 1], V[b:b + 1], [0] * b + [1] + [0] * (B - b - 1))
        with pytest.raises(kvq.KVQError) as e:
            kvq.kvq_sync(cache)
        assert e.value.status == kvq.KVQ_ECAPACITY
        kvq.kvq_refresh_lengths(cache)
        assert [kvq.kvq_seq_len(cache, 0, b) for b in range(B)] == [64, 35]
        np.testing.assert_array_equal(kvq.kvq_export_layer(cache, 0, B), refs[0].export(B))
        del g
    finally:
        kvq.kvq_cache_destroy(cache)
