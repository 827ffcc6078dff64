"""kvq_decode_step (append one token per sequence, then attend) against the
oracle doing the same two steps.

With the one-warp-per-segment split the step is one kernel in which each warp
writes its segment's new token into the window, or quantizes and packs the
completed group into the next page, before attending; otherwise it runs the
append and attention kernels. Either way the pages, window and lengths must be
bit-identical to the oracle's, the attention within the parity bar, and the
error report within fp64 summation-order rounding.
"""

import numpy as np
import pytest
import torch

from test_gpu_parity import Pair, _check_attention, _inputs, _q, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu

FUSED = 1 << 20   # decode mode: the warp split (so the fused kernel) at any length


def _step(P, kvq, rng, batch, hkv, D, G, seqs=None):
    K, V = _inputs(rng, batch, hkv, D)
    Q = _q(rng, batch, hkv * G, D)
    Kt = torch.from_numpy(np.ascontiguousarray(K)).to("cuda", torch.bfloat16)
    Vt = torch.from_numpy(np.ascontiguousarray(V)).to("cuda", torch.bfloat16)
    Qt = torch.from_numpy(np.ascontiguousarray(Q)).to("cuda", torch.bfloat16)
    out = torch.empty((batch, hkv * G, D), device="cuda", dtype=torch.float32)
    kvq.kvq_decode_step(P.cache, 0, Kt, Vt, Qt, out)
    torch.cuda.synchronize()
    P.ref.append(K, V, [1] * batch)
    return out.cpu().numpy(), P.ref.attend(Q, seqs=seqs)


def _same_report(got, want):
    # the append kernel forms each element's terms in fp32 for groups of
    # moderate magnitude: a dx moves by at most 2^-24 |x - z| with |x - z| <=
    # (qmax + 1) s, i.e. at most about 2^-23 * 256 * 3 < 1e-4 relative on the
    # sum of dx^2 for 8-bit codes (fp32 summation over <= 32 terms adds ~2e-6)
    assert got[4] == want[4]
    np.testing.assert_allclose(got[:4], want[:4], rtol=1e-4, atol=0)


@pytest.mark.parametrize("pair", [(2, 2), (2, 4), (4, 2), (4, 4), (4, 8), (8, 2), (8, 8), (16, 16),
                                  (4, 4, 1), (2, 8, 1), (8, 8, 0, 1)])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mode", [FUSED, 0])
def test_decode_step_matches_append_then_attend(kvq, oracle, pair, D, mode):
    rng = np.random.default_rng(hash((pair, D, mode, "step")) % 2**32)
    batch, hkv, G = 5, 2, 4
    lens = [0, 1, 30, 31, 62]  # every sequence completes a group within the steps below
    scales = ([0.05, 0.2], [0.02, 0.5]) if len(pair) > 3 else None
    P = Pair(kvq, oracle, pair, batch, hkv * G, hkv, D, 200, fp8_scales=scales)
    try:
        kvq.kvq_set_decode_mode(P.cache, mode)
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        for i in range(36):
            got, ref = _step(P, kvq, rng, batch, hkv, D, G)
            _check_attention(got, ref, f"{pair} D{D} mode {mode} step {i}")
        P.check_pages()
        for b in range(batch):
            assert kvq.kvq_seq_len(P.cache, 0, b) == lens[b] + 36
        _same_report(kvq.kvq_layer_error(P.cache, 0), P.ref.error())
        kvq.kvq_sync(P.cache)
    finally:
        P.close()


@pytest.mark.parametrize("G", [1, 3, 7])
def test_decode_step_query_groups(kvq, oracle, G):
    # G = 7 has no warp split: the step runs the two kernels
    rng = np.random.default_rng(500 + G)
    batch, hkv, D = 4, 2, 128
    P = Pair(kvq, oracle, (4, 4), batch, hkv * G, hkv, D, 300)
    try:
        kvq.kvq_set_decode_mode(P.cache, FUSED)
        K, V = _inputs(rng, 4 * 63, hkv, D)
        P.append(K, V, [63] * 4)
        for i in range(3):
            got, ref = _step(P, kvq, rng, batch, hkv, D, G)
            _check_attention(got, ref, f"G{G} step {i}")
        P.check_pages()
    finally:
        P.close()


def test_decode_step_many_segments_and_device_lengths(kvq, oracle):
    # 64 sequences x 8 KV heads (512 warps), ragged; then a CUDA graph of the step
    # (the eager steps before the capture set the kernel's launch attributes)
    rng = np.random.default_rng(9)
    batch, hkv, G, D = 64, 8, 4, 128
    lens = [int(x) for x in rng.integers(0, 200, size=batch)]
    P = Pair(kvq, oracle, (4, 2), batch, hkv * G, hkv, D, 400)
    try:
        K, V = _inputs(rng, sum(lens), hkv, D)
        P.append(K, V, lens)
        seqs = [0, 13, 31, 63]
        for i in range(4):
            got, ref = _step(P, kvq, rng, batch, hkv, D, G, seqs=seqs)
            _check_attention(got[seqs], ref[seqs], f"step {i}")
        P.check_pages()
        # captured once, replayed: the device-side lengths advance by one per replay
        K, V = _inputs(rng, batch, hkv, D)
        Q = _q(rng, batch, hkv * G, D)
        Kt = torch.from_numpy(K).to("cuda", torch.bfloat16)
        Vt = torch.from_numpy(V).to("cuda", torch.bfloat16)
        Qt = torch.from_numpy(Q).to("cuda", torch.bfloat16)
        out = torch.empty((batch, hkv * G, D), device="cuda", dtype=torch.float32)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):     # captured, not run
            kvq.kvq_decode_step(P.cache, 0, Kt, Vt, Qt, out)
        torch.cuda.current_stream().wait_stream(s)
        for _ in range(2):
            graph.replay()
            P.ref.append(K, V, [1] * batch)
        torch.cuda.synchronize()
        kvq.kvq_refresh_lengths(P.cache)
        _check_attention(out.cpu().numpy()[seqs], P.ref.attend(Q, seqs=seqs)[seqs], "graph replay")
        P.check_pages()
        del graph
    finally:
        P.close()


def test_decode_step_capacity(kvq, oracle):
    rng = np.random.default_rng(4)
    batch, hkv, G, D = 2, 2, 4, 64
    P = Pair(kvq, oracle, (4, 4), batch, hkv * G, hkv, D, 64)
    try:
        kvq.kvq_set_decode_mode(P.cache, FUSED)
        K, V = _inputs(rng, 64 + 10, hkv, D)
        P.append(K, V, [64, 10])
        before = kvq.kvq_export_layer(P.cache, 0, batch)
        Kt = torch.zeros((batch, hkv, D), device="cuda", dtype=torch.bfloat16)
        Qt = torch.zeros((batch, hkv * G, D), device="cuda", dtype=torch.bfloat16)
        out = torch.empty((batch, hkv * G, D), device="cuda", dtype=torch.float32)
        with pytest.raises(RuntimeError):
            kvq.kvq_decode_step(P.cache, 0, Kt, Kt, Qt, out)
        assert np.array_equal(kvq.kvq_export_layer(P.cache, 0, batch), before)
        assert kvq.kvq_seq_len(P.cache, 0, 1) == 10
    finally:
        P.close()
