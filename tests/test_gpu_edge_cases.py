"""The quantizer's degenerate and extreme inputs on every GPU quantizer, against
the oracle.

Each case prefills a few sequences with one multi-token kvq_append (the CTA-wide
flush of the append kernel), then runs 33 single-token steps through one of
three routes, so every sequence completes at least one more 32-token group on
that route:

* ``append``: one-token kvq_append, then kvq_decode_attn;
* ``step_warp``: kvq_decode_step with the one-warp-per-segment split (the
  warp-level flush fused into the attention kernel);
* ``step_shared``: kvq_decode_step with the shared split.

Inputs (facts page: per-channel asymmetric keys; OpenReview rebuttal:
per-token asymmetric values):

* ``constant``   -- key channels constant over each 32-token group (some at
  exactly 0) and value tokens constant over head_dim: scale 0, codes 0 and the
  zero point equal to the value, so the group is reconstructed exactly;
* ``signed_zero`` -- sets whose minimum or maximum is -0.0 or +0.0, and sets
  made only of signed zeros;
* ``beyond_f16`` -- bf16 values beyond fp16's range (|x| up to 1e6), where the
  zero point clamps at -65504 and the scale at 65504;
* ``tiny`` / ``huge`` -- keys and values scaled by 1e-5 and by 1e4 (value scales
  above 255 and far below fp16's normal range);
* ``mixed_scale`` -- value tokens whose magnitudes span 1e-4 to 1e3 in one page.

Bar: pages, scales, zeros and window bit-exact; attention within max-abs 2e-3
and relative L2 1e-3 of the oracle's fp64 attention. The max-abs bar is taken
on outputs divided by max(1, max |reference|), so it means the same for outputs
of magnitude 1e4 as for unit-scale ones (relative L2 is scale-free already).
"""

import zlib

import numpy as np
import pytest
import torch

from test_gpu_parity import MAX_ABS, REL_L2, Pair, _q, kvq  # noqa: F401  (kvq is a fixture)

pytestmark = pytest.mark.gpu

FUSED = 1 << 20
STEPS = 33


def _seed(*key):
    return zlib.crc32(repr(key).encode())


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _const_key(grp, c, h):
    """Key channel c of KV head h over 32-token group grp: fp16-representable
    bf16 values, a quarter of them exactly 0."""
    return np.where((grp + c) % 4 == 0, 0.0, ((grp * 7 + c * 3 + h) % 41 - 20) / 8.0)


def _const_value(tok):
    return ((tok % 13) - 6) / 4.0


def _draw(case, rng, tok, hkv, D):
    """K, V rows [n, hkv, D] for absolute token positions `tok` ([n]) of one sequence."""
    n = tok.size
    K = rng.standard_normal((n, hkv, D)).astype(np.float32)
    V = rng.standard_normal((n, hkv, D)).astype(np.float32)
    K[:, :, 5::16] *= 8.0  # channel outliers
    grp = tok // 32
    if case == "constant":
        for h in range(hkv):
            for c in range(0, D, 3):
                K[:, h, c] = _const_key(grp, c, h)
        const_tok = (tok % 5) == 0
        V[const_tok] = _const_value(tok[const_tok])[:, None, None]
    elif case == "signed_zero":
        for c in range(0, D, 4):
            col = np.abs(K[:, :, c])
            col[(tok % 3) == 0] = -0.0 if c % 8 == 0 else 0.0
            K[:, :, c] = col
        K[:, :, 2::8] = np.where(rng.random((n, hkv, D // 8)) < 0.5, -0.0, 0.0)
        neg = (tok % 4) == 1
        V[neg] = -np.abs(V[neg])
        V[neg, :, 3] = 0.0
        V[neg, :, 9] = -0.0
        V[(tok % 7) == 2] = np.where(rng.random((int(((tok % 7) == 2).sum()), hkv, D)) < 0.5, -0.0, 0.0)
    elif case == "beyond_f16":
        K[:, :, 7::16] *= 2.0e5
        K[:, :, 11::32] = 1.0e6
        big = (tok % 6) == 0
        V[big] *= 1.0e5
    elif case == "tiny":
        K *= 1e-5
        V *= 1e-5
    elif case == "huge":
        K *= 1e4
        V *= 1e4
    elif case == "mixed_scale":
        V *= (10.0 ** ((tok % 8) - 4.0))[:, None, None]
    else:
        raise ValueError(case)
    return _bf16(K), _bf16(V)


def _check(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    scale = max(1.0, float(np.abs(ref).max()))
    diff = np.abs(got - ref).max() / scale
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert diff <= MAX_ABS, f"{what}: max-abs (scaled) {diff:.3e}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e}"


def _run(kvq, oracle, case, pair, D, route, G=4, seed=0):
    rng = np.random.default_rng(seed)
    batch, hkv = 3, 2
    lens = [5, 31, 64]
    P = Pair(kvq, oracle, pair, batch, hkv * G, hkv, D, 160)
    try:
        kvq.kvq_set_decode_mode(P.cache, FUSED if route == "step_warp" else 0)
        rows = [_draw(case, rng, np.arange(T), hkv, D) for T in lens]
        P.append(np.concatenate([r[0] for r in rows]), np.concatenate([r[1] for r in rows]), lens)
        P.check_pages()
        for s in range(STEPS):
            kv = [_draw(case, rng, np.array([T + s]), hkv, D) for T in lens]
            K = np.concatenate([r[0] for r in kv])
            V = np.concatenate([r[1] for r in kv])
            Q = _q(rng, batch, hkv * G, D)
            Qt = torch.from_numpy(Q).to("cuda", torch.bfloat16)
            out = torch.empty((batch, hkv * G, D), device="cuda", dtype=torch.float32)
            if route == "append":
                P.append(K, V, [1] * batch)
                kvq.kvq_decode_attn(P.cache, 0, Qt, out)
            else:
                Kt = torch.from_numpy(K).to("cuda", torch.bfloat16)
                Vt = torch.from_numpy(V).to("cuda", torch.bfloat16)
                kvq.kvq_decode_step(P.cache, 0, Kt, Vt, Qt, out)
                P.ref.append(K, V, [1] * batch)
            if s in (0, STEPS - 1):
                torch.cuda.synchronize()
                _check(out.cpu().numpy(), P.ref.attend(Q), f"{case} {pair} D{D} {route} step {s}")
        P.check_pages()
        kvq.kvq_sync(P.cache)
        return P.ref
    finally:
        P.close()


ROUTES = ["append", "step_warp", "step_shared"]
INT_PAIRS = [(2, 2), (2, 4), (2, 8), (4, 2), (4, 4), (4, 8), (8, 2), (8, 4), (8, 8)]


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("pair", INT_PAIRS + [(4, 4, 1), (2, 8, 1), (8, 2, 1)])
def test_constant_sets_reconstructed_exactly(kvq, oracle, pair, route):
    ref = _run(kvq, oracle, "constant", pair, 128, route, seed=_seed(pair, route))
    # The GPU pages are byte-identical to the oracle's (checked in _run), so the
    # oracle's dequantization is the GPU cache's: constant key channels (per-
    # channel mode) and constant value tokens come back exactly.
    per_channel = (pair[2] if len(pair) > 2 else 0) == 0
    for b in range(3):
        full = (ref.length(b) // 32) * 32
        tok = np.arange(full)
        for h in range(2):
            Kd, Vd = ref.dequant(b, h)
            if per_channel:
                for c in range(0, 128, 3):
                    assert np.array_equal(Kd[:full, c], _const_key(tok // 32, c, h)), (b, h, c)
            ct = tok[(tok % 5) == 0]
            assert np.array_equal(Vd[ct], np.repeat(_const_value(ct)[:, None], 128, axis=1)), (b, h)


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("pair", INT_PAIRS + [(4, 4, 1), (16, 16), (8, 8, 0, 1)])
def test_signed_zeros(kvq, oracle, pair, route):
    _run(kvq, oracle, "signed_zero", pair, 64, route, seed=_seed(pair, route, "z"))


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("pair", [(2, 2), (4, 4), (8, 8), (4, 8, 1), (8, 2), (16, 16)])
def test_beyond_fp16_range(kvq, oracle, pair, route):
    _run(kvq, oracle, "beyond_f16", pair, 128, route, seed=_seed(pair, route, "b"))


@pytest.mark.parametrize("case", ["tiny", "huge", "mixed_scale"])
@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("pair,G", [((2, 2), 4), ((4, 4), 4), ((8, 8), 4), ((4, 2, 1), 4), ((4, 8), 7),
                                    ((8, 4, 1), 7), ((16, 16), 4)])
def test_extreme_magnitudes(kvq, oracle, case, pair, G, route):
    _run(kvq, oracle, case, pair, 128, route, G=G, seed=_seed(pair, route, case))


@pytest.mark.parametrize("pair", [(4, 4), (8, 2), (2, 8, 1), (16, 16)])
@pytest.mark.parametrize("mode", [0, FUSED])
def test_closed_forms_zero_query_and_equal_keys(kvq, oracle, pair, mode):
    """q = 0, and every key equal: each query head's output is the mean of the
    dequantized values of its KV head."""
    rng = np.random.default_rng(41)
    batch, hkv, G, D = 2, 2, 4, 64
    lens = [70, 129]
    for which in ("zero_query", "equal_keys"):
        P = Pair(kvq, oracle, pair, batch, hkv * G, hkv, D, 200)
        try:
            kvq.kvq_set_decode_mode(P.cache, mode)
            n = sum(lens)
            K = _bf16(rng.standard_normal((n, hkv, D)))
            if which == "equal_keys":
                # one value for every key element: quantized exactly in both key modes
                # (a constant channel and a constant token), so every dequantized key
                # equals the window's bf16 keys
                K[:] = 0.625
            V = _bf16(rng.standard_normal((n, hkv, D)))
            P.append(K, V, lens)
            Q = _q(rng, batch, hkv * G, D)
            if which == "zero_query":
                Q[:] = 0.0
            got, ref = P.attend(Q)
            for b in range(batch):
                for h in range(hkv):
                    _, Vd = P.ref.dequant(b, h)
                    mean = Vd.mean(axis=0)
                    for g in range(G):
                        np.testing.assert_allclose(ref[b, h * G + g], mean, rtol=0, atol=1e-12)
            _check(got, ref, f"{which} {pair} mode {mode}")
        finally:
            P.close()
