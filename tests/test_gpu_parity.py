"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar: packed pages, scales, zeros and the bf16 window bit-exact; decode attention
within max-abs 2e-3 and relative L2 1e-3 of the oracle's fp64 attention over the
same (bit-identical) cache.
"""

import numpy as np
import pytest
import torch

from layer_wise_mixed_kvq_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3
PAIRS = [(2, 2), (2, 4), (2, 8), (4, 2), (4, 4), (4, 8), (8, 2), (8, 4), (8, 8), (16, 16)]


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from layer_wise_mixed_kvq_b200 import build
    build.build()
    from layer_wise_mixed_kvq_b200 import kvq as _kvq
    return _kvq


def _check_attention(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    diff = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert diff.max() <= MAX_ABS, f"{what}: max-abs {diff.max():.3e}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e}"
    return diff.max(), rel


class Pair:
    """A one-layer GPU cache and its oracle twin, fed the same inputs."""

    def __init__(self, kvq, oracle, pair, batch, hq, hkv, D, max_tokens, dtype=torch.bfloat16, fp8_scales=None):
        self.kvq, self.pair, self.batch, self.hq, self.hkv, self.D = kvq, pair, batch, hq, hkv, D
        self.dtype = dtype
        self.cache = kvq.kvq_cache_create([pair], hq, hkv, D, batch, max_tokens)
        fmt = pair[3] if len(pair) > 3 else 0
        ks = vs = None
        if fmt:
            ks, vs = fp8_scales if fp8_scales is not None else ([1.0] * hkv, [1.0] * hkv)
            kvq.kvq_set_fp8_scales(self.cache, 0, ks, vs)
        self.ref = oracle.OracleLayer(pair[0], pair[1], batch, hkv, D, key_mode=pair[2] if len(pair) > 2 else 0,
                                      fmt=fmt, k_scales=ks, v_scales=vs)

    def close(self):
        self.kvq.kvq_cache_destroy(self.cache)

    def append(self, K, V, n_new):
        Kt = torch.from_numpy(np.ascontiguousarray(K)).to("cuda", self.dtype)
        Vt = torch.from_numpy(np.ascontiguousarray(V)).to("cuda", self.dtype)
        self.kvq.kvq_append(self.cache, 0, Kt, Vt, list(n_new))
        self.ref.append(K, V, n_new)

    def check_pages(self):
        got = self.kvq.kvq_export_layer(self.cache, 0, self.batch)
        want = self.ref.export(self.batch)
        assert got.size == want.size
        if not np.array_equal(got, want):
            bad = np.nonzero(got != want)[0]
            raise AssertionError(f"{bad.size} bytes differ, first at {bad[0]} of {got.size}")

    def attend(self, Q, seqs=None):
        Qt = torch.from_numpy(np.ascontiguousarray(Q)).to("cuda", torch.bfloat16)
        out = torch.empty((Q.shape[0], self.hq, self.D), device="cuda", dtype=torch.float32)
        self.kvq.kvq_decode_attn(self.cache, 0, Qt, out)
        torch.cuda.synchronize()
        ref = self.ref.attend(Q, seqs=seqs)
        return out.cpu().numpy(), ref


def _inputs(rng, n, hkv, D, f32=False):
    K = rng.standard_normal((n, hkv, D)).astype(np.float32)
    K[:, :, ::17] *= 8.0
    V = rng.standard_normal((n, hkv, D)).astype(np.float32)
    if not f32:
        K = torch.from_numpy(K).to(torch.bfloat16).float().numpy()
        V = torch.from_numpy(V).to(torch.bfloat16).float().numpy()
    return K, V


def _q(rng, batch, hq, D):
    return torch.from_numpy(rng.standard_normal((batch, hq, D)).astype(np.float32)).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("pair", PAIRS)
@pytest.mark.parametrize("D", [64, 128])
def test_append_and_decode_small(kvq, oracle, pair, D):
    rng = np.random.default_rng(hash((pair, D)) % 2**32)
    batch, hkv, G = 3, 2, 4
    lens = [0, 45, 97]
    P = Pair(kvq, oracle, pair, batch, hkv * G, hkv, D, 256)
    try:
        # one multi-token call (ragged), then two decode-style single-token calls
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        P.check_pages()
        for _ in range(20):
            K, V = _inputs(rng, batch, hkv, D)
            P.append(K, V, [1] * batch)
        P.check_pages()
        got, ref = P.attend(_q(rng, batch, hkv * G, D))
        _check_attention(got, ref, f"{pair} D{D}")
    finally:
        P.close()


@pytest.mark.parametrize("pair", [(8, 4), (4, 2), (16, 16)])
def test_fp32_inputs_rounded_on_entry(kvq, oracle, pair):
    rng = np.random.default_rng(3)
    P = Pair(kvq, oracle, pair, 2, 4, 2, 64, 200, dtype=torch.float32)
    try:
        K, V = _inputs(rng, 140, 2, 64, f32=True)
        P.append(K, V, [70, 70])
        P.check_pages()
        got, ref = P.attend(_q(rng, 2, 4, 64))
        _check_attention(got, ref)
    finally:
        P.close()


@pytest.mark.parametrize("T", [1, 31, 32, 33, 63, 64, 65, 255, 257])
def test_window_boundaries(kvq, oracle, T):
    rng = np.random.default_rng(T)
    P = Pair(kvq, oracle, (4, 8), 1, 8, 2, 128, 300)
    try:
        K, V = _inputs(rng, T, 2, 128)
        P.append(K, V, [T])
        P.check_pages()
        got, ref = P.attend(_q(rng, 1, 8, 128))
        _check_attention(got, ref, f"T={T}")
    finally:
        P.close()


def test_chunking_invariance_on_gpu(kvq, oracle):
    rng = np.random.default_rng(9)
    T, hkv, D = 150, 2, 64
    K, V = _inputs(rng, T, hkv, D)
    exports = []
    for chunks in ([150], [1] * 150, [7, 25, 1, 32, 64, 21]):
        P = Pair(kvq, oracle, (2, 4), 1, 2, hkv, D, 160)
        try:
            i = 0
            for n in chunks:
                P.append(K[i:i + n], V[i:i + n], [n])
                i += n
            P.check_pages()
            exports.append(kvq.kvq_export_layer(P.cache, 0, 1))
        finally:
            P.close()
    assert all(np.array_equal(exports[0], e) for e in exports[1:])


def test_empty_and_zero_appends(kvq, oracle):
    rng = np.random.default_rng(10)
    P = Pair(kvq, oracle, (4, 4), 3, 6, 3, 64, 100)
    try:
        K, V = _inputs(rng, 40, 3, 64)
        P.append(K, V, [0, 40, 0])
        P.check_pages()
        got, ref = P.attend(_q(rng, 3, 6, 64))
        assert np.all(got[0] == 0) and np.all(got[2] == 0)
        _check_attention(got, ref)
    finally:
        P.close()


def test_capacity_error_leaves_cache_unchanged(kvq, oracle):
    rng = np.random.default_rng(11)
    P = Pair(kvq, oracle, (8, 8), 2, 2, 1, 64, 64)
    try:
        K, V = _inputs(rng, 100, 1, 64)
        P.append(K[:60], V[:60], [30, 30])
        before = kvq.kvq_export_layer(P.cache, 0, 2)
        Kt = torch.from_numpy(K[60:100]).to("cuda", torch.bfloat16)
        Vt = torch.from_numpy(V[60:100]).to("cuda", torch.bfloat16)
        with pytest.raises(kvq.KVQError) as e:
            kvq.kvq_append(P.cache, 0, Kt, Vt, [5, 35])
        assert e.value.status == kvq.KVQ_ECAPACITY
        assert kvq.kvq_seq_len(P.cache, 0, 1) == 30
        np.testing.assert_array_equal(before, kvq.kvq_export_layer(P.cache, 0, 2))
        with pytest.raises(kvq.KVQError) as e:
            kvq.kvq_append(P.cache, 3, Kt, Vt, [5, 35])
        assert e.value.status == kvq.KVQ_EINVAL
    finally:
        P.close()


@pytest.mark.parametrize("split", [1, 2, 3, 0])
def test_split_count_does_not_change_results(kvq, oracle, split):
    rng = np.random.default_rng(12)
    P = Pair(kvq, oracle, (4, 2), 2, 14, 2, 128, 800)
    try:
        K, V = _inputs(rng, 1400, 2, 128)
        P.append(K, V, [700, 700])
        kvq.kvq_set_split_pages(P.cache, split)
        got, ref = P.attend(_q(rng, 2, 14, 128))
        _check_attention(got, ref, f"split={split}")
    finally:
        P.close()


@pytest.mark.parametrize("G", [1, 3, 5, 8])
def test_split_segments_odd_gqa(kvq, oracle, G):
    # more units than resident CTAs: slices hold the tail of one sequence-head and
    # the head of the next, so both split records of a CTA and the final merge run
    rng = np.random.default_rng(40 + G)
    batch, hkv, T = 8, 2, 1790
    P = Pair(kvq, oracle, (4, 4), batch, hkv * G, hkv, 128, T + 8)
    try:
        K, V = _inputs(rng, batch * T, hkv, 128)
        P.append(K, V, [T] * batch)
        got, ref = P.attend(_q(rng, batch, hkv * G, 128))
        _check_attention(got, ref, f"G={G}")
    finally:
        P.close()


@pytest.mark.parametrize("pair,G", [((4, 4), 4), ((8, 8), 4), ((4, 4), 7), ((16, 16), 1)])
def test_one_segment_over_the_whole_grid(kvq, oracle, pair, G):
    # a single (sequence, KV head) long enough that every CTA of the persistent
    # grid takes a slice of it: the last CTA merges hundreds of split records
    # (rounds of 16 with online rescaling between rounds)
    rng = np.random.default_rng(70 + G + pair[0])
    T = 24000 + 17
    P = Pair(kvq, oracle, pair, 1, G, 1, 128, T + 8)
    try:
        K, V = _inputs(rng, T, 1, 128)
        P.append(K, V, [T])
        kvq.kvq_set_decode_mode(P.cache, 0)  # shared split
        got, ref = P.attend(_q(rng, 1, G, 128))
        _check_attention(got, ref, f"{pair} G={G}")
    finally:
        P.close()


def test_tiny_k8v4_workload(kvq, oracle):
    """The 1-layer K8V4 workload: batch 1, 2 = 2 heads, D 64, 256 tokens + 1."""
    w = synth.WORKLOADS["tiny_k8v4"]
    P = Pair(kvq, oracle, w.layer_map[0], 1, w.n_q_heads, w.n_kv_heads, w.head_dim, 300, dtype=torch.float32)
    try:
        K, V = synth.kv_tokens(w, 0, w.context)
        P.append(K, V, [w.context])
        K1, V1 = synth.kv_tokens(w, 0, 1, salt=1)
        P.append(K1, V1, [1])
        P.check_pages()
        got, ref = P.attend(synth.queries(w, 0))
        _check_attention(got, ref, "tiny")
    finally:
        P.close()


# ------------------------------------------------ full-size sampled parity --

def _full_layer(kvq, oracle, w, layer, lens, decode_steps=1, sample_seqs=(0,)):
    pair = w.layer_map[layer]
    batch = len(lens)
    P = Pair(kvq, oracle, pair, batch, w.n_q_heads, w.n_kv_heads, w.head_dim, int(max(lens)) + decode_steps + 1)
    try:
        K, V = synth.kv_tokens(w, layer, int(sum(lens)))
        P.append(K, V, [int(x) for x in lens])
        for step in range(decode_steps):
            K1, V1 = synth.kv_tokens(w, layer, batch, salt=1 + step)
            P.append(K1, V1, [1] * batch)
        P.check_pages()
        got, ref = P.attend(synth.queries(w, layer), seqs=sample_seqs)
        idx = list(sample_seqs)
        return _check_attention(got[idx], ref[idx], f"{w.name} layer {layer}")
    finally:
        P.close()


def test_full_llama_k4v4_layer(kvq, oracle):
    w = synth.WORKLOADS["llama_k4v4"]
    _full_layer(kvq, oracle, w, 5, synth.context_lengths(w), 1, sample_seqs=(0, 7, 15))


@pytest.mark.parametrize("layer", [0, 10, 25])
def test_full_qwen_layers(kvq, oracle, layer):
    w = synth.WORKLOADS["qwen_mixed40"]
    _full_layer(kvq, oracle, w, layer, synth.context_lengths(w), 1, sample_seqs=(0, 31))


@pytest.mark.parametrize("layer", [0, 5, 28])
def test_full_llama_mixed_decode_run(kvq, oracle, layer):
    # 128-token prefill then 512 single-token appends (the decode path)
    w = synth.WORKLOADS["llama_mixed325"]
    _full_layer(kvq, oracle, w, layer, synth.context_lengths(w), 512, sample_seqs=(0, 33, 63))


@pytest.mark.parametrize("layer", [0, 1])
def test_full_ragged_long(kvq, oracle, layer):
    w = synth.WORKLOADS["ragged_long"]
    _full_layer(kvq, oracle, w, layer, synth.context_lengths(w), 2, sample_seqs=(0, 3))


def test_simt_kernel_matches_oracle(kvq, oracle, tmp_path):
    """The CUDA-core kernel (KVQ_DECODE_KERNEL=simt) is a second implementation;
    run a few cases through it in a fresh process."""
    import os
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "import pytest\n"
        "sys.exit(pytest.main(['-q', '-x', '-m', 'gpu', %r, '-k', "
        "'test_append_and_decode_small or test_window_boundaries or test_split_count']))\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))), os.path.abspath(__file__))
    env = dict(os.environ, KVQ_DECODE_KERNEL="simt")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


@pytest.mark.parametrize("mode", [0, 1])
def test_max_batch_and_gqa(kvq, oracle, mode):
    """The largest batch (1024 sequences) at the largest GQA ratio (8 query heads
    per KV head, head-row formulation) with ragged short contexts: exercises the
    unit scan over many sequences, many small segments per CTA and empty ones."""
    rng = np.random.default_rng(1024 + mode)
    batch, hkv, G, D = 1024, 1, 8, 64
    lens = [int(x) for x in rng.integers(0, 70, size=batch)]
    P = Pair(kvq, oracle, (4, 2, mode), batch, hkv * G, hkv, D, 80)
    try:
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        K1, V1 = _inputs(rng, batch, hkv, D)
        P.append(K1, V1, [1] * batch)
        P.check_pages()
        seqs = [0, 1, 511, 777, 1023] + [i for i, n in enumerate(lens) if n == 0][:3]
        got, ref = P.attend(_q(rng, batch, hkv * G, D), seqs=seqs)
        _check_attention(got[seqs], ref[seqs], f"batch 1024 mode {mode}")
    finally:
        P.close()
