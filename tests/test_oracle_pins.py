"""Pins for the CPU oracle: checks against what the KVTuner pages and plain
mathematics fix, never against the oracle itself.

Every check here is chosen so that a plausible slip in the oracle (a dropped
term, a wrong rounding direction, a transposed operand, a wrong GQA index)
fails at least one of them.
"""

import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = v
    return vals


# ------------------------------------------------------------ layer maps --

def _llama_325_map():
    # OpenReview rebuttal: layers 0, 1, 2, 31 of Llama-3.1-8B-Instruct take K4V8.
    return [(4, 8) if l in (0, 1, 2, 31) else (4, 2) if l <= 26 else (2, 2) for l in range(32)]


def _qwen_40_map():
    return [(8, 4) if l <= 3 else (4, 4) if l <= 19 else (4, 2) for l in range(28)]


def test_equiv_bits_printed_values(oracle):
    g = _golden("equiv_bits.txt")
    assert oracle.equiv_bits(_llama_325_map()) == pytest.approx(float(g["llama_3.1_8b_map"][0]), abs=0)
    assert oracle.equiv_bits(_qwen_40_map()) == pytest.approx(float(g["qwen2.5_7b_map"][0]), abs=0)
    assert oracle.equiv_bits([(8, 2)]) == float(g["k8v2"][0])
    assert oracle.equiv_bits([(4, 8)]) == float(g["k4v8"][0])


def test_equiv_bits_closed_forms(oracle):
    # bf16 layers count 16 bits: 2 bf16 + 30 K8V8 -> (2*16 + 30*8)/32 = 8.5
    assert oracle.equiv_bits([(16, 16)] * 2 + [(8, 8)] * 30) == 8.5
    # the worked example's map: 8 bf16 + 24 8-bit layers -> (8*16 + 24*8)/32 = 10
    assert oracle.equiv_bits([(16, 16)] * 8 + [(8, 8)] * 24) == 10.0
    # asymmetric pairs: mean of k and v, not of max/min
    assert oracle.equiv_bits([(2, 8), (8, 2)]) == 5.0
    assert oracle.equiv_bits([(2, 4)]) == 3.0


def test_c344_memory_vs_kivi4(oracle):
    # A 25-layer map with mean (k+v)/2 = 3.44: 11 x K4V4 + 14 x K4V2.
    m = [(4, 4)] * 11 + [(4, 2)] * 14
    assert oracle.equiv_bits(m) == pytest.approx(3.44, abs=1e-12)
    tokens, H, D = 4096, 2, 128
    ours = sum(oracle.layer_bytes(k, v, tokens, H, D) for k, v in m)
    kivi4 = sum(oracle.layer_bytes(4, 4, tokens, H, D) for _ in m)
    g = _golden("equiv_bits.txt")
    assert ours / kivi4 == pytest.approx(float(g["c3.44_over_kivi4"][0]), abs=1e-12)


def test_worked_example_bytes(oracle):
    g = {k: float(v[0]) for k, v in _golden("worked_example_bytes.txt").items()}
    MiB = 1 << 20
    tokens, H, D = 25600, 8, 128
    bf16 = oracle.layer_bytes(16, 16, tokens, H, D)
    int8 = oracle.layer_bytes(8, 8, tokens, H, D)
    assert bf16 == g["bf16_layer_mib"] * MiB
    assert int8 == g["fp8_layer_mib"] * MiB
    n = int(g["n_layers"])
    assert n * bf16 == g["all_bf16_mib"] * MiB
    assert n * int8 == g["all_fp8_mib"] * MiB
    mixed = int(g["sensitive_bf16_layers"]) * bf16 + int(g["fp8_layers"]) * int8
    assert mixed == g["mixed_mib"] * MiB
    assert (n * bf16 - mixed) / (n * bf16) * 100 == g["saving_vs_bf16_percent"]
    assert mixed - n * int8 == g["extra_vs_fp8_mib"] * MiB


def test_worked_example_with_metadata(oracle):
    # Our extension of the idealised count: fp16 scale+zero per 32-token key
    # channel group (D*4/32 bytes per token) and per value token (4 bytes).
    tokens, H, D = 25600, 8, 128
    meta = oracle.layer_bytes(8, 8, tokens, H, D, with_meta=True) - oracle.layer_bytes(8, 8, tokens, H, D)
    assert meta == tokens * H * (D * 4 // 32 + 4)
    total = 8 * oracle.layer_bytes(16, 16, tokens, H, D) + 24 * oracle.layer_bytes(8, 8, tokens, H, D, True)
    assert total / (1 << 20) == pytest.approx(2093.75, abs=1e-9)


def test_bf16_cache_size_batch4_8k(oracle):
    # OpenReview rebuttal: batch 4 with 8K tokens is ~4 GB of bf16 KV for
    # Llama-3.1-8B (32 layers, 8 KV heads, head_dim 128).
    total = 32 * oracle.layer_bytes(16, 16, 4 * 8192, 8, 128)
    assert total == 4 * (1 << 30)


def test_page_bytes_closed_form(oracle):
    # codes 32*D*(k+v)/8 + key scale/zero 4*D + value scale/zero 128
    for D in (64, 128):
        for k in (2, 4, 8):
            for v in (2, 4, 8):
                assert oracle.page_bytes(k, v, D) == 4 * D * (k + v) + 4 * D + 128
                assert oracle.page_bytes(k, v, D) % 16 == 0
        assert oracle.page_bytes(16, 16, D) == 32 * D * 2 * 2
    # per token per head at D=128: 84 (K2V2) .. 276 (K8V8) bytes
    assert oracle.page_bytes(2, 2, 128) / 32 == 84
    assert oracle.page_bytes(4, 4, 128) / 32 == 148
    assert oracle.page_bytes(8, 8, 128) / 32 == 276


# ---------------------------------------------------------- number formats --

def test_bf16_rounding_matches_torch(oracle):
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 3000),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, 65504.0], dtype=np.float32),
        # exact ties between two bf16 values: 1 + 2^-8 and 1 + 3*2^-8
        np.array([1.00390625, 1.01171875], dtype=np.float32),
    ])
    ours = np.array([oracle.f32_to_bf16_bits(v) for v in x], dtype=np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_f16_directed_rounding_exhaustive_representable(oracle):
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    finite = np.isfinite(vals)
    for b, v in zip(bits[finite][::7], vals[finite][::7]):
        f = np.float32(v)
        assert oracle.f32_to_f16_rd_bits(f) == b or (v == 0)
        assert oracle.f32_to_f16_ru_bits(f) == b or (v == 0)
        assert oracle.f16_value(int(b)) == float(v)


def test_f16_directed_rounding_brackets_numpy_rn(oracle):
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(4000) * 10.0 ** rng.uniform(-9, 4.4, 4000)).astype(np.float32)
    for v in x:
        rd = oracle.f16_value(oracle.f32_to_f16_rd_bits(v))
        ru = oracle.f16_value(oracle.f32_to_f16_ru_bits(v))
        rn = float(np.float16(v))
        assert rd <= float(v) <= ru
        assert rn in (rd, ru)
        if rd != ru:
            # adjacent fp16 values: nothing representable strictly between
            assert float(np.nextafter(np.float16(rd), np.float16(np.inf))) == ru
        else:
            assert rd == float(v)


def test_f16_directed_rounding_overflow(oracle):
    assert oracle.f16_value(oracle.f32_to_f16_rd_bits(70000.0)) == 65504.0
    assert oracle.f16_value(oracle.f32_to_f16_ru_bits(70000.0)) == float("inf")
    assert oracle.f16_value(oracle.f32_to_f16_rd_bits(-70000.0)) == float("-inf")
    assert oracle.f16_value(oracle.f32_to_f16_ru_bits(-70000.0)) == -65504.0
    # below the smallest subnormal: one step of 2^-24 up, zero down
    assert oracle.f16_value(oracle.f32_to_f16_ru_bits(1e-9)) == 2.0 ** -24
    assert oracle.f16_value(oracle.f32_to_f16_rd_bits(1e-9)) == 0.0


# --------------------------------------------------------------- quantizer --

def test_quantizer_hand_example(oracle):
    g = _golden("quantizer_example.txt")
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)
    codes, sb, zb = oracle.quantize(x, int(g["bits"][0]))
    assert list(codes) == [int(c) for c in g["codes"]]
    assert sb == int(g["scale_bits"][0], 16)
    assert zb == int(g["zero_bits"][0], 16)


def _sets(rng, n):
    yield rng.standard_normal(n).astype(np.float32)
    yield (rng.standard_t(3.0, n) * 16).astype(np.float32)
    yield rng.uniform(-1e-3, 1e-3, n).astype(np.float32)
    yield (rng.standard_normal(n) * 1e-6 + 3.0).astype(np.float32)
    yield rng.uniform(100, 30000, n).astype(np.float32)
    x = rng.standard_normal(n).astype(np.float32)
    x[rng.integers(0, n)] = 40.0
    yield x


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("n", [32, 64, 128])
def test_quantizer_invariants(oracle, bits, n):
    qmax = (1 << bits) - 1
    rng = np.random.default_rng(bits * 1000 + n)
    for trial in range(6):
        for x in _sets(rng, n):
            x = oracle.bf16_round(x)
            codes, sb, zb = oracle.quantize(x, bits)
            s, z = oracle.f16_value(sb), oracle.f16_value(zb)
            assert codes.min() >= 0 and codes.max() <= qmax
            # the stored range covers the data: z <= min, z + qmax*s >= max
            assert z <= float(x.min())
            assert z + qmax * s >= float(x.max()) * (1 - 2 ** -20) - 1e-30
            xh = codes.astype(np.float64) * s + z
            err = np.abs(xh - x.astype(np.float64))
            slack = s * qmax * 2.0 ** -21 + np.abs(x) * 2.0 ** -22
            assert np.all(err <= s / 2 + slack), (bits, n, trial, err.max(), s)
            # brute force: every code is a nearest level
            levels = np.arange(qmax + 1, dtype=np.float64) * s + z
            best = np.min(np.abs(x.astype(np.float64)[:, None] - levels[None, :]), axis=1)
            assert np.all(err <= best + slack)
            if s >= 2.0 ** -14:  # normal fp16 scale
                assert codes[np.argmin(x)] == 0
                assert codes[np.argmax(x)] == qmax


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_quantizer_constant_channel_exact(oracle, bits):
    for v in (0.0, 1.0, -2.5, 0.1015625, 3.0e4, -1.0e-3):
        x = oracle.bf16_round(np.full(32, v, dtype=np.float32))
        codes, sb, zb = oracle.quantize(x, bits)
        xv = float(x[0])
        if float(np.float16(xv)) == xv:
            assert oracle.f16_value(sb) == 0.0 and np.all(codes == 0)
            assert oracle.f16_value(zb) == xv
        else:  # not fp16-representable: still inside half a step
            s, z = oracle.f16_value(sb), oracle.f16_value(zb)
            assert np.all(np.abs(codes * s + z - xv) <= s / 2 + abs(xv) * 2 ** -22)


def test_quantizer_signed_zero_minimum(oracle):
    # {-0, +0, 1}: the zero point is +0 whichever zero comes first
    for x in ([-0.0, 0.0, 1.0], [0.0, -0.0, 1.0], [1.0, -0.0, 0.0]):
        codes, sb, zb = oracle.quantize(np.array(x * 11, dtype=np.float32)[:32], 4)
        assert zb == 0x0000
        assert list(codes[:3]) == [0 if v == 0 else 15 for v in x]
    codes, sb, zb = oracle.quantize(np.array([-0.0] * 32, dtype=np.float32), 2)
    assert zb == 0x0000 and sb == 0x0000


def test_quantizer_two_level_set(oracle):
    # {a, b} with a < b, both fp16-representable: z = a, s = ru((b-a)/qmax),
    # a -> code 0, b -> qmax.
    for bits in (2, 4, 8):
        x = np.array([0.5, 2.5] * 16, dtype=np.float32)
        codes, sb, zb = oracle.quantize(x, bits)
        qmax = (1 << bits) - 1
        assert oracle.f16_value(zb) == 0.5
        assert oracle.f16_value(sb) >= 2.0 / qmax
        assert list(codes[:2]) == [0, qmax]


# ------------------------------------------------------------------ layout --

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bits", [2, 4, 8, 16])
@pytest.mark.parametrize("is_value", [False, True])
def test_pack_unpack_identity(oracle, D, bits, is_value):
    rng = np.random.default_rng(D + bits)
    hi = (1 << bits) if bits < 16 else (1 << 16)
    vals = rng.integers(0, hi, size=(32, D)).astype(np.uint16)
    blk = oracle.pack_block(vals, D, bits, is_value)
    assert blk.size == 32 * D * bits // 8
    np.testing.assert_array_equal(oracle.unpack_block(blk, D, bits, is_value), vals)
    # every bit of the block carries exactly one element's bit (a bijection)
    ones = oracle.pack_block(np.full((32, D), hi - 1, dtype=np.uint16), D, bits, is_value)
    assert np.all(ones == 0xFF)


def test_layout_example_word(oracle):
    # 4-bit key tile 0, lane 0 (g=0, t=0): elements e0..e7 are
    # (tok,dim) = (0,0) (0,1) (8,0) (8,1) (0,8) (0,9) (8,8) (8,9); with code =
    # (tok + dim) % 16 they are 0,1,8,9,8,9,0,1 and sit in nibbles
    # [e0 e2 e4 e6 e1 e3 e5 e7] -> 0,8,8,0,1,9,9,1 -> word 0x19910880.
    D = 64
    t, d = np.meshgrid(np.arange(32), np.arange(D), indexing="ij")
    vals = ((t + d) % 16).astype(np.uint16)
    blk = oracle.pack_block(vals, D, 4, False)
    assert int.from_bytes(bytes(blk[0:4]), "little") == 0x19910880


# ---------------------------------------------------------------- window --

def _kv(rng, n, H, D, f32=False):
    K = rng.standard_normal((n, H, D)).astype(np.float32)
    K[:, :, 3] *= 10
    V = rng.standard_normal((n, H, D)).astype(np.float32)
    if not f32:
        K = torch.from_numpy(K).to(torch.bfloat16).float().numpy()
        V = torch.from_numpy(V).to(torch.bfloat16).float().numpy()
    return K, V


@pytest.mark.parametrize("pair", [(8, 4), (2, 2), (4, 8), (16, 16)])
def test_window_chunking_invariance(oracle, pair):
    rng = np.random.default_rng(5)
    H, D, T = 2, 64, 97
    K, V = _kv(rng, T, H, D)
    whole = oracle.OracleLayer(*pair, 1, H, D)
    whole.append(K, V, [T])
    ones = oracle.OracleLayer(*pair, 1, H, D)
    for i in range(T):
        ones.append(K[i:i + 1], V[i:i + 1], [1])
    rnd = oracle.OracleLayer(*pair, 1, H, D)
    i = 0
    while i < T:
        n = int(rng.integers(1, 40))
        n = min(n, T - i)
        rnd.append(K[i:i + n], V[i:i + n], [n])
        i += n
    a, b, c = whole.export(), ones.export(), rnd.export()
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(a, c)
    # W = T mod 32 bf16 tokens; floor(T/32) pages
    pb = oracle.page_bytes(*pair, D)
    assert a.size == H * ((T // 32) * pb + 2 * (T % 32) * D * 2)
    assert whole.length(0) == T


def test_window_holds_bf16_of_input(oracle):
    rng = np.random.default_rng(6)
    H, D = 1, 64
    K, V = _kv(rng, 5, H, D, f32=True)
    L = oracle.OracleLayer(4, 4, 1, H, D)
    L.append(K, V, [5])
    Kh, Vh = L.dequant(0, 0)
    ref = lambda x: torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(Kh, ref(K[:, 0]))
    np.testing.assert_array_equal(Vh, ref(V[:, 0]))


@pytest.mark.parametrize("pair", [(2, 2), (4, 2), (4, 4), (8, 4), (4, 8), (8, 8)])
def test_dequant_round_trip_error(oracle, pair):
    # dequantized cache vs the bf16 inputs: keys within half a channel step,
    # values within half a token step (pins quantizer + layout round trip)
    rng = np.random.default_rng(7)
    H, D, T = 2, 128, 64
    K, V = _kv(rng, T, H, D)
    L = oracle.OracleLayer(*pair, 1, H, D)
    L.append(K, V, [T])
    for h in range(H):
        Kh, Vh = L.dequant(0, h)
        for g in range(2):
            blk = K[32 * g:32 * g + 32, h]
            qk = (1 << pair[0]) - 1
            step = np.maximum((blk.max(0) - blk.min(0)) / qk, 1e-30)
            assert np.all(np.abs(Kh[32 * g:32 * g + 32] - blk) <= step * 0.5 * (1 + 2 ** -9) + 1e-6)
            vb = V[32 * g:32 * g + 32, h]
            qv = (1 << pair[1]) - 1
            vstep = np.maximum((vb.max(1) - vb.min(1)) / qv, 1e-30)[:, None]
            assert np.all(np.abs(Vh[32 * g:32 * g + 32] - vb) <= vstep * 0.5 * (1 + 2 ** -9) + 1e-6)


# --------------------------------------------------------------- attention --

def _sdpa_fp64(q, K, V, G):
    """Textbook SDPA with torch (fp64): q [Hq, D], K/V [T, Hkv, D]."""
    qt = torch.from_numpy(q).double()[None, :, None, :]                      # [1, Hq, 1, D]
    kt = torch.from_numpy(K).double().permute(1, 0, 2).repeat_interleave(G, 0)[None]  # [1, Hq, T, D]
    vt = torch.from_numpy(V).double().permute(1, 0, 2).repeat_interleave(G, 0)[None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0, :].numpy()


@pytest.mark.parametrize("G", [1, 4, 7])
@pytest.mark.parametrize("T", [1, 31, 32, 33, 70])
def test_bf16_layer_attention_equals_sdpa(oracle, G, T):
    rng = np.random.default_rng(G * 100 + T)
    H, D, B = 2, 64, 2
    K, V = _kv(rng, B * T, H, D)
    L = oracle.OracleLayer(16, 16, B, H, D)
    L.append(K, V, [T] * B)
    Q = torch.from_numpy(rng.standard_normal((B, H * G, D)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    out = L.attend(Q)
    for b in range(B):
        ref = _sdpa_fp64(Q[b], K[b * T:(b + 1) * T], V[b * T:(b + 1) * T], G)
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("pair", [(8, 4), (2, 2), (4, 8)])
def test_quantized_attention_equals_sdpa_on_dequantized(oracle, pair):
    rng = np.random.default_rng(11)
    H, D, G, T = 2, 64, 4, 75
    K, V = _kv(rng, T, H, D)
    L = oracle.OracleLayer(*pair, 1, H, D)
    L.append(K, V, [T])
    Q = torch.from_numpy(rng.standard_normal((1, H * G, D)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    out = L.attend(Q)
    Kd = np.stack([L.dequant(0, h)[0] for h in range(H)], axis=1)
    Vd = np.stack([L.dequant(0, h)[1] for h in range(H)], axis=1)
    np.testing.assert_allclose(out[0], _sdpa_fp64(Q[0], Kd, Vd, G), rtol=0, atol=1e-12)
    # and close to attention over the unquantized inputs (quantization error only)
    err = np.abs(out[0] - _sdpa_fp64(Q[0], K, V, G)).max()
    assert err < {2: 1.0, 4: 0.3, 8: 0.05}[min(pair)]


def test_attention_closed_forms(oracle):
    rng = np.random.default_rng(12)
    H, D, T = 1, 64, 70
    K, V = _kv(rng, T, H, D)
    L = oracle.OracleLayer(4, 4, 1, H, D)
    L.append(K, V, [T])
    Vd = L.dequant(0, 0)[1]
    # q = 0: uniform weights -> mean of the dequantized values
    out = L.attend(np.zeros((1, 1, D), dtype=np.float32))
    np.testing.assert_allclose(out[0, 0], Vd.mean(0), rtol=0, atol=1e-12)
    # one token: output is that token's (bf16) value
    L1 = oracle.OracleLayer(4, 4, 1, H, D)
    L1.append(K[:1], V[:1], [1])
    out = L1.attend(rng.standard_normal((1, 1, D)).astype(np.float32))
    np.testing.assert_array_equal(out[0, 0], torch.from_numpy(V[0, 0]).to(torch.bfloat16).double().numpy())
    # all keys equal: every score is equal -> mean of the values
    Ke = np.repeat(K[:1], T, axis=0)
    Le = oracle.OracleLayer(8, 8, 1, H, D)
    Le.append(Ke, V, [T])
    out = Le.attend(rng.standard_normal((1, 1, D)).astype(np.float32))
    np.testing.assert_allclose(out[0, 0], Le.dequant(0, 0)[1].mean(0), rtol=0, atol=1e-12)
    # empty sequence -> zeros
    L0 = oracle.OracleLayer(4, 4, 1, H, D)
    assert np.all(L0.attend(np.ones((1, 1, D), dtype=np.float32)) == 0)


def test_gqa_head_mapping(oracle):
    # q head h reads KV head h // G: give each KV head a distinct constant value
    # vector; the output of q head h must be KV head h//G's vector.
    H, G, D, T = 3, 2, 64, 40
    K = np.zeros((T, H, D), dtype=np.float32)
    V = np.zeros((T, H, D), dtype=np.float32)
    for h in range(H):
        V[:, h, :] = float(h + 1)
    L = oracle.OracleLayer(16, 16, 1, H, D)
    L.append(K, V, [T])
    out = L.attend(np.ones((1, H * G, D), dtype=np.float32))
    for hq in range(H * G):
        np.testing.assert_allclose(out[0, hq], float(hq // G + 1), rtol=0, atol=1e-12)


def test_threaded_attention_equals_single_thread(oracle):
    """The oracle's multi-threaded driver (used to time it on every host core)
    shares out (sequence, KV head) units only: its output is the single-thread
    output bit for bit, including empty and window-only sequences."""
    rng = np.random.default_rng(21)
    lens = [0, 5, 32, 70, 129]
    L = oracle.OracleLayer(4, 2, len(lens), 3, 64)
    K = rng.standard_normal((sum(lens), 3, 64)).astype(np.float32)
    V = rng.standard_normal((sum(lens), 3, 64)).astype(np.float32)
    L.append(K, V, lens)
    Q = rng.standard_normal((len(lens), 6, 64)).astype(np.float32)
    one = L.attend(Q)
    for n in (2, 3, 64):
        assert np.array_equal(L.attend(Q, threads=n), one)
    assert np.array_equal(L.attend(Q, seqs=[1, 4], threads=4)[[1, 4]], one[[1, 4]])
