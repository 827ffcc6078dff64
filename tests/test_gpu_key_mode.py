"""GPU parity of the per-token key mode (third pair field 1) with the oracle.

Per-token asymmetric keys are the second key mode the KVTuner pages compare
(OpenReview rebuttal, section 4 "Per-channel vs. per-token quantization").
Same bar as the per-channel path: pages bit-exact, attention within max-abs
2e-3 and relative L2 1e-3 of the oracle's fp64 attention. G <= 4 runs the
token-row tensor-core formulation, G > 4 the head-row one.
"""

import numpy as np
import pytest
import torch

from layer_wise_mixed_kvq_b200 import synth
from test_gpu_parity import Pair, _check_attention, _inputs, _q, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu

QPAIRS = [(2, 2), (2, 4), (2, 8), (4, 2), (4, 4), (4, 8), (8, 2), (8, 4), (8, 8)]


@pytest.mark.parametrize("pair", QPAIRS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [4, 7])
def test_per_token_append_and_decode(kvq, oracle, pair, D, G):
    rng = np.random.default_rng(hash((pair, D, G, "pt")) % 2**32)
    batch, hkv = 3, 2
    lens = [0, 45, 97]
    P = Pair(kvq, oracle, (pair[0], pair[1], 1), batch, hkv * G, hkv, D, 256)
    try:
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        P.check_pages()
        for _ in range(20):
            K, V = _inputs(rng, batch, hkv, D)
            P.append(K, V, [1] * batch)
        P.check_pages()
        got, ref = P.attend(_q(rng, batch, hkv * G, D))
        _check_attention(got, ref, f"per-token {pair} D{D} G{G}")
    finally:
        P.close()


@pytest.mark.parametrize("T", [1, 31, 32, 33, 64, 65, 257, 1790])
def test_per_token_window_boundaries_and_splits(kvq, oracle, T):
    rng = np.random.default_rng(T + 7)
    P = Pair(kvq, oracle, (2, 8, 1), 4, 16, 4, 128, T + 8)
    try:
        K, V = _inputs(rng, 4 * T, 4, 128)
        P.append(K, V, [T] * 4)
        P.check_pages()
        got, ref = P.attend(_q(rng, 4, 16, 128))
        _check_attention(got, ref, f"T={T}")
    finally:
        P.close()


def test_mixed_key_modes_in_one_cache(kvq, oracle):
    """One cache whose layers mix key modes, pairs and a bf16 layer; each layer
    is checked against its own oracle layer."""
    layer_map = [(4, 4, 0), (4, 4, 1), (2, 8, 1), (16, 16), (8, 2, 0)]
    rng = np.random.default_rng(77)
    batch, hkv, G, D = 2, 2, 4, 128
    lens = [70, 131]
    cache = kvq.kvq_cache_create(layer_map, hkv * G, hkv, D, batch, 256)
    try:
        for layer, pair in enumerate(layer_map):
            ref = oracle.OracleLayer(pair[0], pair[1], batch, hkv, D, key_mode=pair[2] if len(pair) > 2 else 0)
            K, V = _inputs(rng, sum(lens), hkv, D)
            kvq.kvq_append(cache, layer, torch.from_numpy(K).cuda().bfloat16(), torch.from_numpy(V).cuda().bfloat16(),
                           lens)
            ref.append(K, V, lens)
            got = kvq.kvq_export_layer(cache, layer, batch)
            np.testing.assert_array_equal(got, ref.export(batch))
            Q = _q(rng, batch, hkv * G, D)
            out = torch.empty((batch, hkv * G, D), device="cuda")
            kvq.kvq_decode_attn(cache, layer, torch.from_numpy(Q).cuda().bfloat16(), out)
            torch.cuda.synchronize()
            _check_attention(out.cpu().numpy(), ref.attend(Q), f"layer {layer} {pair}")
        # byte accounting follows each layer's metadata
        assert kvq.kvq_bytes(cache, 1, batch, 1) < kvq.kvq_bytes(cache, 0, batch, 1)
        assert kvq.kvq_bytes(cache, 1, batch, 0) == kvq.kvq_bytes(cache, 0, batch, 0)
    finally:
        kvq.kvq_cache_destroy(cache)


def test_full_llama_k4v4_per_token_layer(kvq, oracle):
    """Full-size layer of the per-token workload (batch 16, 8 KV heads, 4097
    tokens), sampled sequences checked against the oracle."""
    w = synth.WORKLOADS["llama_k4v4_pt"]
    lens = synth.context_lengths(w)
    layer = 3
    P = Pair(kvq, oracle, w.layer_map[layer], len(lens), w.n_q_heads, w.n_kv_heads, w.head_dim, int(max(lens)) + 2)
    try:
        K, V = synth.kv_tokens(w, layer, int(sum(lens)))
        P.append(K, V, [int(x) for x in lens])
        K1, V1 = synth.kv_tokens(w, layer, len(lens), salt=1)
        P.append(K1, V1, [1] * len(lens))
        P.check_pages()
        seqs = (0, 9, 15)
        got, ref = P.attend(synth.queries(w, layer), seqs=seqs)
        _check_attention(got[list(seqs)], ref[list(seqs)], "llama_k4v4_pt")
    finally:
        P.close()


def test_per_token_simt_kernel_matches_oracle(kvq, oracle):
    """The CUDA-core kernel in per-token mode, in a fresh process."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    code = (
        "import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
        "import pytest\n"
        "sys.exit(pytest.main(['-q', '-x', '-m', 'gpu', %r, '-k', "
        "'test_per_token_append_and_decode or test_per_token_window']))\n"
    ) % (os.path.dirname(here), here, os.path.abspath(__file__))
    env = dict(os.environ, KVQ_DECODE_KERNEL="simt")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
