"""CPU oracle for layer-wise mixed-precision KV decode (KVTuner).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``. The product package never imports it.

The arithmetic lives in ``kvq_oracle.cpp`` (plain C++, fp32 quantization with
no FMA contraction, fp64 attention). This module only compiles it with g++ and
marshals numpy arrays through ctypes.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-pthread"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (no-op when up to date)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call(["g++", *_CXXFLAGS, "-o", tmp, _SRC])
            os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        c = ctypes
        P = c.c_void_p
        sig = {
            "oracle_f32_to_bf16": (c.c_uint16, [c.c_float]),
            "oracle_f32_to_f16_rd": (c.c_uint16, [c.c_float]),
            "oracle_f32_to_f16_ru": (c.c_uint16, [c.c_float]),
            "oracle_f16_value": (c.c_double, [c.c_uint16]),
            "oracle_equiv_bits": (c.c_double, [P, P, c.c_int]),
            "oracle_layer_bytes": (c.c_int64, [c.c_int, c.c_int, c.c_int, c.c_int, c.c_int64, c.c_int, c.c_int,
                                               c.c_int]),
            "oracle_quantize": (None, [P, c.c_int, c.c_int, P, P, P]),
            "oracle_page_bytes": (c.c_int64, [c.c_int, c.c_int, c.c_int, c.c_int, c.c_int]),
            "oracle_e4m3_encode": (c.c_uint8, [c.c_float]),
            "oracle_e4m3_value": (c.c_double, [c.c_uint8]),
            "oracle_pack_block": (None, [P, P, c.c_int, c.c_int, c.c_int]),
            "oracle_unpack_block": (None, [P, P, c.c_int, c.c_int, c.c_int]),
            "oracle_build_page": (None, [P, P, P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_float,
                                         c.c_float]),
            "oracle_dequant_page": (None, [P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_float, c.c_float,
                                           P, P]),
            "oracle_layer_new": (P, [c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int]),
            "oracle_layer_set_fp8_scales": (None, [P, P, P]),
            "oracle_layer_free": (None, [P]),
            "oracle_layer_len": (c.c_int64, [P, c.c_int]),
            "oracle_layer_error": (c.c_int64, [P, P]),
            "oracle_layer_append": (None, [P, P, P, P, c.c_int]),
            "oracle_layer_export_bytes": (c.c_int64, [P, c.c_int]),
            "oracle_layer_export": (None, [P, c.c_int, P]),
            "oracle_layer_dequant": (None, [P, c.c_int, c.c_int, P, P]),
            "oracle_layer_attend": (None, [P, P, c.c_int, c.c_int, P, P]),
            "oracle_layer_attend_threads": (None, [P, P, c.c_int, c.c_int, P, P, c.c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


# ---------------------------------------------------------------- scalars --
def f32_to_bf16_bits(x: float) -> int:
    return int(lib().oracle_f32_to_bf16(float(x)))


def f32_to_f16_rd_bits(x: float) -> int:
    return int(lib().oracle_f32_to_f16_rd(float(x)))


def f32_to_f16_ru_bits(x: float) -> int:
    return int(lib().oracle_f32_to_f16_ru(float(x)))


def f16_value(bits: int) -> float:
    return float(lib().oracle_f16_value(int(bits) & 0xFFFF))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (RNE) with the oracle's own routine; fp32 result."""
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    L = lib()
    bits = np.array([L.oracle_f32_to_bf16(float(v)) for v in x], dtype=np.uint32)
    return (bits << 16).view(np.float32)


# ------------------------------------------------------------- layer maps --
def equiv_bits(pairs) -> float:
    """Mean over layers of (k_bits + v_bits)/2; bf16 layers are (16, 16)."""
    k = np.array([p[0] for p in pairs], dtype=np.uint8)
    v = np.array([p[1] for p in pairs], dtype=np.uint8)
    return float(lib().oracle_equiv_bits(_ptr(k), _ptr(v), len(pairs)))


#: key modes: per-channel keys over the 32-token group, or per-token keys
KEY_PER_CHANNEL, KEY_PER_TOKEN = 0, 1
#: layer formats: integer codes with fp16 scale/zero, or fp8 e4m3 with per-head scales
FMT_INT, FMT_FP8 = 0, 1


def layer_bytes(k_bits: int, v_bits: int, tokens: int, n_kv_heads: int, head_dim: int,
                with_meta: bool = False, key_mode: int = KEY_PER_CHANNEL, fmt: int = FMT_INT) -> int:
    return int(lib().oracle_layer_bytes(k_bits, v_bits, key_mode, fmt, tokens, n_kv_heads, head_dim,
                                        int(with_meta)))


def page_bytes(k_bits: int, v_bits: int, head_dim: int, key_mode: int = KEY_PER_CHANNEL, fmt: int = FMT_INT) -> int:
    return int(lib().oracle_page_bytes(k_bits, v_bits, head_dim, key_mode, fmt))


def e4m3_encode(x: float) -> int:
    """fp32 -> e4m3 bits (round to nearest even, saturating at 448)."""
    return int(lib().oracle_e4m3_encode(float(x)))


def e4m3_value(bits: int) -> float:
    return float(lib().oracle_e4m3_value(int(bits) & 0xFF))


# -------------------------------------------------------------- quantizer --
def quantize(x: np.ndarray, bits: int):
    """Quantize one set of values. Returns (codes uint8[n], scale_bits, zero_bits)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.size, dtype=np.uint8)
    sb = np.zeros(1, dtype=np.uint16)
    zb = np.zeros(1, dtype=np.uint16)
    lib().oracle_quantize(_ptr(x), x.size, bits, _ptr(codes), _ptr(sb), _ptr(zb))
    return codes, int(sb[0]), int(zb[0])


def pack_block(vals: np.ndarray, head_dim: int, bits: int, is_value: bool) -> np.ndarray:
    vals = np.ascontiguousarray(vals, dtype=np.uint16).reshape(32, head_dim)
    out = np.zeros(32 * head_dim * bits // 8, dtype=np.uint8)
    lib().oracle_pack_block(_ptr(out), _ptr(vals), head_dim, bits, int(is_value))
    return out


def unpack_block(blk: np.ndarray, head_dim: int, bits: int, is_value: bool) -> np.ndarray:
    blk = np.ascontiguousarray(blk, dtype=np.uint8)
    vals = np.zeros((32, head_dim), dtype=np.uint16)
    lib().oracle_unpack_block(_ptr(blk), _ptr(vals), head_dim, bits, int(is_value))
    return vals


def build_page(k_bf16_bits: np.ndarray, v_bf16_bits: np.ndarray, head_dim: int, k_bits: int,
               v_bits: int, key_mode: int = KEY_PER_CHANNEL, fmt: int = FMT_INT, k_scale: float = 1.0,
               v_scale: float = 1.0) -> np.ndarray:
    kb = np.ascontiguousarray(k_bf16_bits, dtype=np.uint16).reshape(32, head_dim)
    vb = np.ascontiguousarray(v_bf16_bits, dtype=np.uint16).reshape(32, head_dim)
    page = np.zeros(page_bytes(k_bits, v_bits, head_dim, key_mode, fmt), dtype=np.uint8)
    lib().oracle_build_page(_ptr(page), _ptr(kb), _ptr(vb), head_dim, k_bits, v_bits, key_mode, fmt,
                            float(k_scale), float(v_scale))
    return page


def dequant_page(page: np.ndarray, head_dim: int, k_bits: int, v_bits: int, key_mode: int = KEY_PER_CHANNEL,
                 fmt: int = FMT_INT, k_scale: float = 1.0, v_scale: float = 1.0):
    page = np.ascontiguousarray(page, dtype=np.uint8)
    K = np.zeros((32, head_dim), dtype=np.float64)
    V = np.zeros((32, head_dim), dtype=np.float64)
    lib().oracle_dequant_page(_ptr(page), head_dim, k_bits, v_bits, key_mode, fmt, float(k_scale), float(v_scale),
                              _ptr(K), _ptr(V))
    return K, V


# ------------------------------------------------------------ layer cache --
class OracleLayer:
    """One layer's KV cache for `batch` sequences, mirroring the library's semantics."""

    def __init__(self, k_bits: int, v_bits: int, batch: int, n_kv_heads: int, head_dim: int,
                 key_mode: int = KEY_PER_CHANNEL, fmt: int = FMT_INT, k_scales=None, v_scales=None):
        self.k_bits, self.v_bits, self.key_mode, self.fmt = k_bits, v_bits, key_mode, fmt
        self.batch, self.n_kv_heads, self.head_dim = batch, n_kv_heads, head_dim
        self._h = lib().oracle_layer_new(k_bits, v_bits, key_mode, fmt, batch, n_kv_heads, head_dim)
        if k_scales is not None or v_scales is not None:
            ks = np.ascontiguousarray(np.ones(n_kv_heads) if k_scales is None else k_scales, dtype=np.float32)
            vs = np.ascontiguousarray(np.ones(n_kv_heads) if v_scales is None else v_scales, dtype=np.float32)
            assert ks.size == n_kv_heads and vs.size == n_kv_heads
            lib().oracle_layer_set_fp8_scales(self._h, _ptr(ks), _ptr(vs))

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            lib().oracle_layer_free(h)
            self._h = None

    def length(self, b: int) -> int:
        return int(lib().oracle_layer_len(self._h, b))

    def error(self):
        """(sum (k-k^)^2, sum k^2, sum (v-v^)^2, sum v^2, quantized elements per K and per V)."""
        out = np.zeros(4, dtype=np.float64)
        n = int(lib().oracle_layer_error(self._h, _ptr(out)))
        return (*[float(x) for x in out], n)

    def append(self, K: np.ndarray, V: np.ndarray, n_new) -> None:
        """K, V: [sum(n_new), n_kv_heads, head_dim] values (fp32 or bf16-valued)."""
        K = np.ascontiguousarray(K, dtype=np.float32)
        V = np.ascontiguousarray(V, dtype=np.float32)
        n = np.ascontiguousarray(np.asarray(n_new, dtype=np.int32))
        assert K.shape == V.shape and K.shape[0] == int(n.sum())
        assert K.shape[1:] == (self.n_kv_heads, self.head_dim)
        lib().oracle_layer_append(self._h, _ptr(K), _ptr(V), _ptr(n), n.size)

    def export(self, batch: int | None = None) -> np.ndarray:
        batch = self.batch if batch is None else batch
        n = int(lib().oracle_layer_export_bytes(self._h, batch))
        out = np.zeros(n, dtype=np.uint8)
        lib().oracle_layer_export(self._h, batch, _ptr(out))
        return out

    def dequant(self, b: int, h: int):
        T = self.length(b)
        K = np.zeros((T, self.head_dim), dtype=np.float64)
        V = np.zeros((T, self.head_dim), dtype=np.float64)
        if T:
            lib().oracle_layer_dequant(self._h, b, h, _ptr(K), _ptr(V))
        return K, V

    def attend(self, Q: np.ndarray, batch: int | None = None, seqs=None, threads: int = 1) -> np.ndarray:
        """Q: [batch, Hq, D] (bf16 values). Returns fp64 [batch, Hq, D].

        threads > 1 shares the (sequence, KV head) units out over that many host
        threads; the result is the same."""
        Q = np.ascontiguousarray(Q, dtype=np.float32)
        batch = Q.shape[0] if batch is None else batch
        hq = Q.shape[1]
        assert hq % self.n_kv_heads == 0
        out = np.zeros((batch, hq, self.head_dim), dtype=np.float64)
        mask = None
        mptr = None
        if seqs is not None:
            mask = np.zeros(batch, dtype=np.uint8)
            mask[list(seqs)] = 1
            mptr = _ptr(mask)
        if threads > 1:
            lib().oracle_layer_attend_threads(self._h, _ptr(Q), hq, batch, mptr, _ptr(out), int(threads))
        else:
            lib().oracle_layer_attend(self._h, _ptr(Q), hq, batch, mptr, _ptr(out))
        return out
