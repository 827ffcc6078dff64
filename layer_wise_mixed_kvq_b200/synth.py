"""Seeded synthetic workloads for the mixed-precision KV decode path.

This module only draws random inputs (keys, values, queries, sequence lengths)
with the shapes and distributions of the five workloads below. It holds none of
the method's arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it.

Workloads (model shapes from the KVTuner pages: Llama-3.1-8B has 32 layers,
32 query / 8 KV heads, head_dim 128; Qwen2.5-7B has 28 layers, 28 query / 4 KV
heads, head_dim 128; layer maps from the OpenReview rebuttal's per-layer facts
and the 3.25 / 4.0-bit results):

* ``tiny_k8v4``      -- 1 layer K8V4, batch 1, 2 query = 2 KV heads, D 64,
  256 cached tokens + 1 decode token, fp32 N(0,1) with 2 key channels x10.
* ``llama_k4v4``     -- 32 layers K4V4, batch 16, context 4096 + 1.
* ``llama_k4v4_pt``  -- the same shapes, draws and seed with per-token keys
  (third pair field 1: the per-token-asym key mode).
* ``llama_fp8_bf16``  -- the worked example's split of 32 layers: 8 kept in
  BF16 (the four boundary layers at each end) and 24 FP8 e4m3 layers (pair
  (8, 8, 0, 1)) with fixed per-KV-head scales; llama shapes, batch 16,
  context 4096 + 1, seed 5.
* ``llama_mixed325`` -- layers 0,1,2,31 K4V8; 3-26 K4V2; 27-30 K2V2; batch 64,
  prefill 128 then 512 decode steps.
* ``qwen_mixed40``   -- 28 layers: 0-3 K8V4, 4-19 K4V4, 20-27 K4V2; batch 32,
  context 8192 + 1; keys Student-t(3) with 8 channels x16.
* ``ragged_long``    -- layers 0 and 31 bf16, the rest K8V8; batch 4, context per
  sequence uniform in [8192, 32768]; prefill then 64 decode steps.

The bf16 workloads draw in fp32 and round to bf16 with torch's conversion.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

BF16 = (16, 16)


@dataclass(frozen=True)
class Workload:
    name: str
    layer_map: tuple            # ((k_bits, v_bits[, key_mode]), ...) one per layer
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int                # tokens cached before the timed decode (mean for ragged)
    decode_steps: int
    key_dist: str               # "normal" | "student_t3"
    n_outlier: int              # outlier key channels per KV head
    outlier_scale: float
    input_dtype: str            # "f32" | "bf16"
    seed: int
    ragged: tuple = ()          # (lo, hi) per-sequence context range, or ()
    notes: str = field(default="")
    fp8_scales: tuple = ()      # fp8 layers: ((k scale per KV head), (v scale per KV head)), or ()

    @property
    def n_layers(self) -> int:
        return len(self.layer_map)

    @property
    def gqa(self) -> int:
        return self.n_q_heads // self.n_kv_heads


def _llama_mixed_map():
    m = []
    for layer in range(32):
        if layer in (0, 1, 2, 31):
            m.append((4, 8))
        elif 3 <= layer <= 26:
            m.append((4, 2))
        else:
            m.append((2, 2))
    return tuple(m)


def _fp8_bf16_map():
    return tuple((16, 16) if (layer < 4 or layer >= 28) else (8, 8, 0, 1) for layer in range(32))


def _qwen_map():
    m = []
    for layer in range(28):
        if layer <= 3:
            m.append((8, 4))
        elif layer <= 19:
            m.append((4, 4))
        else:
            m.append((4, 2))
    return tuple(m)


def _ragged_map():
    return tuple(BF16 if layer in (0, 31) else (8, 8) for layer in range(32))


WORKLOADS = {
    "tiny_k8v4": Workload("tiny_k8v4", ((8, 4),), 1, 2, 2, 64, 256, 1, "normal", 2, 10.0, "f32", 0),
    "llama_k4v4": Workload("llama_k4v4", tuple([(4, 4)] * 32), 16, 32, 8, 128, 4096, 1, "normal", 4,
                           8.0, "bf16", 1),
    "llama_fp8_bf16": Workload("llama_fp8_bf16", _fp8_bf16_map(), 16, 32, 8, 128, 4096, 1, "normal", 4,
                               8.0, "bf16", 5,
                               fp8_scales=(tuple(0.0625 * (1 + h / 8) for h in range(8)),
                                           tuple(0.03125 * (1 + h / 16) for h in range(8)))),
    "llama_k4v4_pt": Workload("llama_k4v4_pt", tuple([(4, 4, 1)] * 32), 16, 32, 8, 128, 4096, 1, "normal", 4,
                              8.0, "bf16", 1),
    "llama_mixed325": Workload("llama_mixed325", _llama_mixed_map(), 64, 32, 8, 128, 128, 512, "normal",
                               4, 8.0, "bf16", 2),
    "qwen_mixed40": Workload("qwen_mixed40", _qwen_map(), 32, 28, 4, 128, 8192, 1, "student_t3", 8, 16.0,
                             "bf16", 3),
    "ragged_long": Workload("ragged_long", _ragged_map(), 4, 32, 8, 128, 20480, 64, "normal", 4, 8.0,
                            "bf16", 4, ragged=(8192, 32768)),
}


def context_lengths(w: Workload, batch: int | None = None) -> np.ndarray:
    """Per-sequence prefill lengths (ragged workloads draw them from their seed)."""
    batch = w.batch if batch is None else batch
    if w.ragged:
        rng = np.random.default_rng(np.random.SeedSequence([w.seed, 7777]))
        lo, hi = w.ragged
        return rng.integers(lo, hi + 1, size=batch).astype(np.int64)
    return np.full(batch, w.context, dtype=np.int64)


def outlier_channels(w: Workload, layer: int, head_dim: int | None = None) -> np.ndarray:
    """[n_kv_heads, n_outlier] channel indices drawn per (layer, KV head)."""
    D = w.head_dim if head_dim is None else head_dim
    rng = np.random.default_rng(np.random.SeedSequence([w.seed, 1000 + layer]))
    return np.stack([rng.choice(D, size=w.n_outlier, replace=False) for _ in range(w.n_kv_heads)])


def _rng(w: Workload, layer: int, stream: int, salt: int = 0):
    return np.random.default_rng(np.random.SeedSequence([w.seed, layer, stream, salt]))


def _to_input_dtype(w: Workload, x: np.ndarray) -> np.ndarray:
    if w.input_dtype == "f32":
        return x.astype(np.float32)
    import torch
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def kv_tokens(w: Workload, layer: int, n_tokens: int, salt: int = 0, n_kv_heads: int | None = None):
    """Draw K, V of shape [n_tokens, n_kv_heads, head_dim] (float32 holding input-dtype values).

    `salt` separates independent draws of the same layer (prefill vs each decode step).
    """
    H = w.n_kv_heads if n_kv_heads is None else n_kv_heads
    D = w.head_dim
    rk = _rng(w, layer, 1, salt)
    rv = _rng(w, layer, 2, salt)
    if w.key_dist == "student_t3":
        K = rk.standard_t(3.0, size=(n_tokens, H, D))
    else:
        K = rk.standard_normal((n_tokens, H, D))
    oc = outlier_channels(w, layer)
    for h in range(H):
        K[:, h, oc[h % w.n_kv_heads]] *= w.outlier_scale
    V = rv.standard_normal((n_tokens, H, D))
    return _to_input_dtype(w, K), _to_input_dtype(w, V)


def queries(w: Workload, layer: int, batch: int | None = None, salt: int = 0) -> np.ndarray:
    """Draw Q of shape [batch, n_q_heads, head_dim], rounded to bf16 (the path's query dtype)."""
    import torch
    batch = w.batch if batch is None else batch
    r = _rng(w, layer, 3, salt)
    q = r.standard_normal((batch, w.n_q_heads, w.head_dim)).astype(np.float32)
    return torch.from_numpy(q).to(torch.bfloat16).to(torch.float32).numpy()


def torch_kv_tokens(w: Workload, layer: int, n_tokens: int, device, generator, n_kv_heads=None):
    """Device-side draw with the same recipe (for filling large caches quickly).

    Returns bf16 tensors [n_tokens, n_kv_heads, head_dim]. Values differ from the
    numpy draw; the distribution is the same.
    """
    import torch
    H = w.n_kv_heads if n_kv_heads is None else n_kv_heads
    D = w.head_dim
    if w.key_dist == "student_t3":
        # Student-t(3) = N(0,1) / sqrt(chi2_3 / 3)
        z = torch.randn((n_tokens, H, D), device=device, generator=generator)
        g = torch.randn((3, n_tokens, H, D), device=device, generator=generator)
        K = z / torch.sqrt((g * g).sum(0) / 3.0)
    else:
        K = torch.randn((n_tokens, H, D), device=device, generator=generator)
    oc = outlier_channels(w, layer)
    scale = torch.ones((H, D), device=device)
    for h in range(H):
        scale[h, torch.as_tensor(oc[h % w.n_kv_heads], device=device)] = w.outlier_scale
    K = K * scale
    V = torch.randn((n_tokens, H, D), device=device, generator=generator)
    return K.to(torch.bfloat16), V.to(torch.bfloat16)
