"""kvq_decode_attn_noalloc: decode attention for callers that cannot allocate
device memory (their memory belongs to an engine arena or a host runtime, or
the call sits in a loop that must not hit cudaMalloc). The library keeps its
split-K scratch in a fixed static device array instead.

The layer state is rebuilt in caller-owned tensors from kvq_export_layer, and
two calls in a row must match both kvq_decode_attn on the original cache and
the CPU oracle's fp64 attention within the parity tolerance, with
kvq_noalloc_check reporting no lost page copy. This file sorts last so a
stop-at-first-failure run has already run every other test.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from layer_wise_mixed_kvq_b200 import build
    build.build()
    from layer_wise_mixed_kvq_b200 import kvq as _kvq
    return _kvq


def _caller_buffers(kvq, cache, pair, batch, hkv, D, max_pages, lens):
    """Lay the exported layer out in the documented caller-owned format."""
    blob = kvq.kvq_export_layer(cache, 0, batch)
    pb = kvq.kvq_page_bytes(pair, D)
    pages = np.zeros((batch, hkv, max_pages, pb), dtype=np.uint8)
    window = np.zeros((batch, hkv, 2, 32, D), dtype=np.uint16)
    off = 0
    for b in range(batch):
        P, W = lens[b] // 32, lens[b] % 32
        for h in range(hkv):
            pages[b, h, :P] = blob[off:off + P * pb].reshape(P, pb)
            off += P * pb
            for kv in range(2):
                window[b, h, kv, :W] = blob[off:off + W * D * 2].view(np.uint16).reshape(W, D)
                off += W * D * 2
    assert off == blob.size
    dev = torch.device("cuda")
    return (torch.from_numpy(pages).to(dev), torch.from_numpy(window.view(np.int16)).to(dev).view(torch.bfloat16),
            torch.tensor(lens, dtype=torch.int32, device=dev))


def _close(got, want):
    got, want = got.double().cpu().numpy(), want.double().cpu().numpy()
    assert np.abs(got - want).max() <= MAX_ABS
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= REL_L2


@pytest.mark.parametrize("pair,D,G", [((4, 4), 128, 4), ((8, 2), 64, 7), ((16, 16), 128, 1), ((2, 4, 1), 128, 4),
                                      ((4, 8, 1), 64, 7)])
def test_noalloc_matches_decode_attn_twice(kvq, oracle, pair, D, G):
    rng = np.random.default_rng(77)
    batch, hkv, max_tokens = 3, 2, 1100
    lens = [700, 33, 1000]
    cache = kvq.kvq_cache_create([pair], hkv * G, hkv, D, batch, max_tokens)
    ref = oracle.OracleLayer(pair[0], pair[1], batch, hkv, D, key_mode=pair[2] if len(pair) > 2 else 0)
    try:
        n = sum(lens) - batch
        K = torch.from_numpy(rng.standard_normal((n, hkv, D)).astype(np.float32)).cuda().to(torch.bfloat16)
        V = torch.from_numpy(rng.standard_normal((n, hkv, D)).astype(np.float32)).cuda().to(torch.bfloat16)
        kvq.kvq_append(cache, 0, K, V, [x - 1 for x in lens])
        ref.append(K.float().cpu().numpy(), V.float().cpu().numpy(), [x - 1 for x in lens])
        K1 = torch.randn((batch, hkv, D), device="cuda").to(torch.bfloat16)
        V1 = torch.randn((batch, hkv, D), device="cuda").to(torch.bfloat16)
        kvq.kvq_append(cache, 0, K1, V1, [1] * batch)
        ref.append(K1.float().cpu().numpy(), V1.float().cpu().numpy(), [1] * batch)
        Q = torch.randn((batch, hkv * G, D), device="cuda").to(torch.bfloat16)
        want = torch.empty((batch, hkv * G, D), device="cuda", dtype=torch.float32)
        kvq.kvq_decode_attn(cache, 0, Q, want)
        exact = ref.attend(Q.float().cpu().numpy())
        max_pages = max_tokens // 32
        pages, window, seq_len = _caller_buffers(kvq, cache, pair, batch, hkv, D, max_pages, lens)
        for _ in range(2):
            out = torch.full((batch, hkv * G, D), float("nan"), device="cuda", dtype=torch.float32)
            kvq.kvq_decode_attn_noalloc(pair, D, hkv * G, hkv, pages, max_pages, window, seq_len, max(lens), Q, out)
            torch.cuda.synchronize()
            _close(out, want)
            _close(out, torch.from_numpy(exact))
        kvq.kvq_noalloc_check()
    finally:
        kvq.kvq_cache_destroy(cache)


def test_noalloc_with_the_cuda_core_kernel(kvq):
    """The same calls with KVQ_DECODE_KERNEL=simt (the CUDA-core kernel, whose split
    slots come from the static array too), in a fresh process."""
    import os
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "import pytest\n"
        "sys.exit(pytest.main(['-q', '-x', '-m', 'gpu', %r, '-k', 'test_noalloc_matches_decode_attn_twice']))\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))), os.path.abspath(__file__))
    env = dict(os.environ, KVQ_DECODE_KERNEL="simt")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900,
                       cwd=os.path.dirname(os.path.abspath(__file__)))
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_noalloc_rejects_oversized_scratch(kvq):
    # 1024 sequences x 8192 KV heads need 32 MiB of merge counters alone
    dev = torch.device("cuda")
    pages = torch.zeros(16, dtype=torch.uint8, device=dev)
    window = torch.zeros(8, dtype=torch.bfloat16, device=dev)
    seq_len = torch.zeros(1024, dtype=torch.int32, device=dev)
    Q = torch.zeros((1024, 1, 8), dtype=torch.bfloat16, device=dev)
    out = torch.zeros((1024, 1, 8), dtype=torch.float32, device=dev)
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attn_noalloc((4, 4), 128, 8192, 8192, pages, 0, window, seq_len, 0, Q, out)
    assert e.value.status == kvq.KVQ_ECAPACITY
    assert "16 MiB" in str(e.value)
