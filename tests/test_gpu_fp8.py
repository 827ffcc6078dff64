"""GPU parity of the FP8 (e4m3) layer format with the oracle.

FP8 KV layers with per-attention-head scales next to BF16 layers are the
pages' worked example (machinoai Q&A section 2) and the vLLM practice the
llms-explorer facts page describes. Bar: pages bit-exact, attention within
max-abs 2e-3 and relative L2 1e-3 of the oracle's fp64 attention.
"""

import numpy as np
import pytest
import torch

from layer_wise_mixed_kvq_b200 import synth
from test_gpu_parity import Pair, _check_attention, _inputs, _q, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu

FP8 = (8, 8, 0, 1)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 7])
def test_fp8_append_and_decode(kvq, oracle, D, G):
    rng = np.random.default_rng(D * 10 + G)
    batch, hkv = 3, 2
    lens = [0, 45, 97]
    scales = ([0.0625, 0.5], [0.03125, 1.5])
    P = Pair(kvq, oracle, FP8, batch, hkv * G, hkv, D, 256, fp8_scales=scales)
    try:
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        P.check_pages()
        for _ in range(20):
            K, V = _inputs(rng, batch, hkv, D)
            P.append(K, V, [1] * batch)
        P.check_pages()
        got, ref = P.attend(_q(rng, batch, hkv * G, D))
        _check_attention(got, ref, f"fp8 D{D} G{G}")
    finally:
        P.close()


def test_fp8_saturation_and_subnormals(kvq, oracle):
    # scales that push |x / s| past 448 (saturation) and below 2^-6 (subnormals)
    rng = np.random.default_rng(5)
    batch, hkv, D, T = 2, 2, 128, 96
    P = Pair(kvq, oracle, FP8, batch, 8, hkv, D, 128, fp8_scales=([2.0 ** -7, 64.0], [2.0 ** -6, 32.0]))
    try:
        K, V = _inputs(rng, batch * T, hkv, D)
        P.append(K * 4, V * 4, [T, T])
        P.check_pages()
        got, ref = P.attend(_q(rng, batch, 8, D))
        _check_attention(got, ref, "fp8 saturation")
    finally:
        P.close()


@pytest.mark.parametrize("fp32", [False, True])
def test_fp8_fp32_inputs_and_windows(kvq, oracle, fp32):
    rng = np.random.default_rng(6 + fp32)
    dtype = torch.float32 if fp32 else torch.bfloat16
    P = Pair(kvq, oracle, FP8, 2, 16, 4, 64, 200, dtype=dtype, fp8_scales=([0.25] * 4, [0.125] * 4))
    try:
        for n in (31, 1, 33, 1):
            K, V = _inputs(rng, 2 * n, 4, 64, f32=fp32)
            P.append(K, V, [n, n])
            P.check_pages()
            got, ref = P.attend(_q(rng, 2, 16, 64))
            _check_attention(got, ref, f"fp8 window n={n}")
    finally:
        P.close()


def test_fp8_scale_rules(kvq):
    cache = kvq.kvq_cache_create([FP8, (4, 4)], 8, 2, 64, 2, 64)
    try:
        with pytest.raises(kvq.KVQError):                    # not an fp8 layer
            kvq.kvq_set_fp8_scales(cache, 1, [1.0, 1.0], [1.0, 1.0])
        with pytest.raises(kvq.KVQError):                    # scales must be finite and > 0
            kvq.kvq_set_fp8_scales(cache, 0, [1.0, 0.0], [1.0, 1.0])
        with pytest.raises(kvq.KVQError):
            kvq.kvq_set_fp8_scales(cache, 0, [1.0, float("nan")], [1.0, 1.0])
        kvq.kvq_set_fp8_scales(cache, 0, [0.5, 2.0], [1.0, 1.0])
        K = torch.randn(2, 2, 64, device="cuda").bfloat16()
        kvq.kvq_append(cache, 0, K, K, [1, 1])
        with pytest.raises(kvq.KVQError):                    # the layer is no longer empty
            kvq.kvq_set_fp8_scales(cache, 0, [1.0, 1.0], [1.0, 1.0])
        kvq.kvq_cache_reset(cache)
        kvq.kvq_set_fp8_scales(cache, 0, [1.0, 1.0], [1.0, 1.0])
    finally:
        kvq.kvq_cache_destroy(cache)


def test_fp8_worked_example_layer_map(kvq, oracle):
    """8 BF16 + 24 FP8 layers: byte accounting equals the pages' split, and a
    BF16 and an FP8 layer of the same cache match their oracle layers."""
    w = synth.WORKLOADS["llama_fp8_bf16"]
    batch, T = 2, 200
    cache = kvq.kvq_cache_create(list(w.layer_map), w.n_q_heads, w.n_kv_heads, w.head_dim, batch, T + 8)
    try:
        for layer, pair in enumerate(w.layer_map):
            if len(pair) > 3:
                kvq.kvq_set_fp8_scales(cache, layer, *w.fp8_scales)
        T32 = 192  # whole pages only, so the bytes compare without windows
        for layer in range(w.n_layers):
            K, V = synth.kv_tokens(w, layer, batch * T32)
            kvq.kvq_append(cache, layer, torch.from_numpy(K).cuda().bfloat16(), torch.from_numpy(V).cuda().bfloat16(),
                           [T32] * batch)
        bf16 = kvq.kvq_bytes(cache, 0, batch, 1)
        fp8 = kvq.kvq_bytes(cache, 10, batch, 1)
        assert fp8 * 2 == bf16
        total = sum(kvq.kvq_bytes(cache, l, batch, 1) for l in range(w.n_layers))
        assert total == 8 * bf16 + 24 * fp8 == 20 * bf16
        assert 1 - total / (32 * bf16) == 0.375          # the pages' saving against an all-BF16 cache
        for layer in (0, 10):
            pair = w.layer_map[layer]
            fmt = pair[3] if len(pair) > 3 else 0
            ks, vs = w.fp8_scales if fmt else (None, None)
            ref = oracle.OracleLayer(pair[0], pair[1], batch, w.n_kv_heads, w.head_dim, fmt=fmt, k_scales=ks,
                                     v_scales=vs)
            K, V = synth.kv_tokens(w, layer, batch * T32)
            ref.append(K, V, [T32] * batch)
            np.testing.assert_array_equal(kvq.kvq_export_layer(cache, layer, batch), ref.export(batch))
            Q = synth.queries(w, layer, batch=batch)
            out = torch.empty((batch, w.n_q_heads, w.head_dim), device="cuda")
            kvq.kvq_decode_attn(cache, layer, torch.from_numpy(Q).cuda().bfloat16(), out)
            torch.cuda.synchronize()
            _check_attention(out.cpu().numpy(), ref.attend(Q), f"layer {layer}")
    finally:
        kvq.kvq_cache_destroy(cache)


def test_full_fp8_layer(kvq, oracle):
    """Full-size FP8 layer of llama_fp8_bf16 (batch 16, 8 KV heads, 4097 tokens)."""
    w = synth.WORKLOADS["llama_fp8_bf16"]
    lens = synth.context_lengths(w)
    layer = 12
    P = Pair(kvq, oracle, w.layer_map[layer], len(lens), w.n_q_heads, w.n_kv_heads, w.head_dim, int(max(lens)) + 2,
             fp8_scales=w.fp8_scales)
    try:
        K, V = synth.kv_tokens(w, layer, int(sum(lens)))
        P.append(K, V, [int(x) for x in lens])
        K1, V1 = synth.kv_tokens(w, layer, len(lens), salt=1)
        P.append(K1, V1, [1] * len(lens))
        P.check_pages()
        seqs = (0, 8, 15)
        got, ref = P.attend(synth.queries(w, layer), seqs=seqs)
        _check_attention(got[list(seqs)], ref[list(seqs)], "llama_fp8_bf16")
    finally:
        P.close()


def test_fp8_simt_kernel_matches_oracle(kvq, oracle):
    """The CUDA-core kernel on fp8 layers, in a fresh process."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    code = (
        "import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
        "import pytest\n"
        "sys.exit(pytest.main(['-q', '-x', '-m', 'gpu', %r, '-k', "
        "'test_fp8_append_and_decode or test_fp8_saturation']))\n"
    ) % (os.path.dirname(here), here, os.path.abspath(__file__))
    env = dict(os.environ, KVQ_DECODE_KERNEL="simt")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
