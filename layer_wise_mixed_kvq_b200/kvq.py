"""Python binding of libkvq (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
computation of its own: tensors are passed as device pointers, the current
torch stream as cudaStream_t. If libkvq.so is missing the import fails; there
is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK, KVQ_EINVAL, KVQ_ECAPACITY, KVQ_ENOMEM, KVQ_ECUDA = 0, 1, 2, 3, 4
KVQ_BF16, KVQ_F32 = 0, 1
KVQ_KEY_PER_CHANNEL, KVQ_KEY_PER_TOKEN = 0, 1
KVQ_FMT_INT, KVQ_FMT_FP8 = 0, 1

#: every symbol the C header declares
EXPORTS = (
    "kvq_page_bytes", "kvq_equiv_bits", "kvq_cache_pool_bytes", "kvq_cache_create", "kvq_cache_destroy",
    "kvq_cache_reset", "kvq_append", "kvq_decode_attn", "kvq_decode_attn_noalloc", "kvq_set_split_pages", "kvq_seq_len", "kvq_bytes",
    "kvq_export_bytes", "kvq_export_layer", "kvq_sync", "kvq_launch_count", "kvq_last_error",
    "kvq_status_string", "kvq_set_fp8_scales", "kvq_layer_error", "kvq_refresh_lengths",
    "kvq_set_decode_mode", "kvq_decode_step", "kvq_noalloc_check",
)


class kvq_pair(ctypes.Structure):
    _fields_ = [("k_bits", ctypes.c_uint8), ("v_bits", ctypes.c_uint8), ("key_mode", ctypes.c_uint8),
                ("format", ctypes.c_uint8)]


def _pair(p) -> kvq_pair:
    """(k_bits, v_bits[, key_mode[, format]]) -> kvq_pair."""
    return kvq_pair(int(p[0]), int(p[1]), int(p[2]) if len(p) > 2 else KVQ_KEY_PER_CHANNEL,
                    int(p[3]) if len(p) > 3 else KVQ_FMT_INT)


class kvq_error_stats(ctypes.Structure):
    _fields_ = [("k_sq_err", ctypes.c_double), ("k_sq", ctypes.c_double), ("v_sq_err", ctypes.c_double),
                ("v_sq", ctypes.c_double), ("elements", ctypes.c_int64)]


class KVQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libkvq.so not found at {LIB_PATH}; build it with `python -m layer_wise_mixed_kvq_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    c = ctypes
    P = c.c_void_p
    sig = {
        "kvq_page_bytes": (c.c_int64, [kvq_pair, c.c_int]),
        "kvq_equiv_bits": (c.c_double, [P, c.c_int]),
        "kvq_cache_pool_bytes": (c.c_size_t, [P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int64]),
        "kvq_cache_create": (c.c_int, [P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int64, P, c.c_size_t,
                                       c.POINTER(P)]),
        "kvq_cache_destroy": (None, [P]),
        "kvq_cache_reset": (c.c_int, [P, P]),
        "kvq_append": (c.c_int, [P, c.c_int, P, P, c.c_int, P, c.c_int, P]),
        "kvq_decode_attn": (c.c_int, [P, c.c_int, P, c.c_int, P, P]),
        "kvq_decode_attn_noalloc": (c.c_int, [kvq_pair, c.c_int, c.c_int, c.c_int, P, c.c_int64, P, P, c.c_int64, P,
                                              c.c_int, P, P]),
        "kvq_noalloc_check": (c.c_int, []),
        "kvq_set_split_pages": (c.c_int, [P, c.c_int]),
        "kvq_set_decode_mode": (c.c_int, [P, c.c_int]),
        "kvq_decode_step": (c.c_int, [P, c.c_int, P, P, P, c.c_int, P, P]),
        "kvq_seq_len": (c.c_int64, [P, c.c_int, c.c_int]),
        "kvq_bytes": (c.c_int64, [P, c.c_int, c.c_int, c.c_int]),
        "kvq_export_bytes": (c.c_int64, [P, c.c_int, c.c_int]),
        "kvq_export_layer": (c.c_int, [P, c.c_int, c.c_int, P, c.c_size_t]),
        "kvq_sync": (c.c_int, [P]),
        "kvq_launch_count": (c.c_int64, [P]),
        "kvq_last_error": (c.c_char_p, []),
        "kvq_status_string": (c.c_char_p, [c.c_int]),
        "kvq_set_fp8_scales": (c.c_int, [P, c.c_int, P, P]),
        "kvq_layer_error": (c.c_int, [P, c.c_int, c.POINTER(kvq_error_stats)]),
        "kvq_refresh_lengths": (c.c_int, [P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def _status_name(st: int) -> str:
    return lib.kvq_status_string(st).decode()


def _check(st: int) -> None:
    if st != KVQ_OK:
        raise KVQError(st, lib.kvq_last_error().decode())


def _pairs(layer_map):
    arr = (kvq_pair * len(layer_map))()
    for i, p in enumerate(layer_map):
        arr[i] = _pair(p)
    return arr


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


# ----------------------------------------------------------------- host-only --
def kvq_page_bytes(pair, head_dim: int) -> int:
    return int(lib.kvq_page_bytes(_pair(pair), int(head_dim)))


def kvq_equiv_bits(layer_map) -> float:
    return float(lib.kvq_equiv_bits(_pairs(layer_map), len(layer_map)))


def kvq_cache_pool_bytes(layer_map, n_q_heads, n_kv_heads, head_dim, max_batch, max_tokens) -> int:
    return int(lib.kvq_cache_pool_bytes(_pairs(layer_map), len(layer_map), n_q_heads, n_kv_heads, head_dim,
                                        max_batch, max_tokens))


# -------------------------------------------------------------------- cache --
def kvq_cache_create(layer_map, n_q_heads, n_kv_heads, head_dim, max_batch, max_tokens, device_pool=None):
    """Returns an opaque handle (int). device_pool: optional uint8 CUDA tensor."""
    out = ctypes.c_void_p()
    pool = _dev_ptr(device_pool) if device_pool is not None else None
    nbytes = device_pool.numel() * device_pool.element_size() if device_pool is not None else 0
    _check(lib.kvq_cache_create(_pairs(layer_map), len(layer_map), n_q_heads, n_kv_heads, head_dim, max_batch,
                                max_tokens, pool, nbytes, ctypes.byref(out)))
    return out.value


def kvq_cache_destroy(cache) -> None:
    lib.kvq_cache_destroy(ctypes.c_void_p(cache))


def kvq_cache_reset(cache, stream=None) -> None:
    _check(lib.kvq_cache_reset(ctypes.c_void_p(cache), _stream(stream)))


def kvq_append(cache, layer, K, V, n_new, stream=None) -> None:
    """K, V: CUDA tensors [sum(n_new), n_kv_heads, head_dim], bf16 or fp32; n_new: ints per sequence."""
    import torch
    if K.dtype != V.dtype:
        raise ValueError("K and V must have the same dtype")
    if K.dtype == torch.bfloat16:
        dt = KVQ_BF16
    elif K.dtype == torch.float32:
        dt = KVQ_F32
    else:
        raise ValueError("K/V dtype must be bfloat16 or float32")
    n = (ctypes.c_int32 * len(n_new))(*[int(x) for x in n_new])
    _check(lib.kvq_append(ctypes.c_void_p(cache), int(layer), _dev_ptr(K), _dev_ptr(V), dt, n, len(n_new),
                          _stream(stream)))


def kvq_decode_attn(cache, layer, Q, out, stream=None) -> None:
    """Q: bf16 CUDA [batch, n_q_heads, head_dim]; out: fp32 CUDA, same shape."""
    import torch
    if Q.dtype != torch.bfloat16 or out.dtype != torch.float32:
        raise ValueError("Q must be bfloat16 and out float32")
    _check(lib.kvq_decode_attn(ctypes.c_void_p(cache), int(layer), _dev_ptr(Q), int(Q.shape[0]), _dev_ptr(out),
                               _stream(stream)))


def kvq_decode_step(cache, layer, K, V, Q, out, stream=None) -> None:
    """Append one token per sequence (K, V: bf16 CUDA [batch, n_kv_heads, head_dim]) and attend
    (Q: bf16 CUDA [batch, n_q_heads, head_dim]; out: fp32 CUDA, same shape)."""
    import torch
    if K.dtype != torch.bfloat16 or V.dtype != torch.bfloat16 or Q.dtype != torch.bfloat16:
        raise ValueError("K, V and Q must be bfloat16")
    if out.dtype != torch.float32:
        raise ValueError("out must be float32")
    if K.shape[0] != Q.shape[0] or V.shape[0] != Q.shape[0]:
        raise ValueError("K, V and Q must have the same batch")
    _check(lib.kvq_decode_step(ctypes.c_void_p(cache), int(layer), _dev_ptr(K), _dev_ptr(V), _dev_ptr(Q),
                               int(Q.shape[0]), _dev_ptr(out), _stream(stream)))


def kvq_decode_attn_noalloc(pair, head_dim, n_q_heads, n_kv_heads, pages, max_pages, window, seq_len,
                            max_seq_len, Q, out, stream=None) -> None:
    """Decode attention over caller-owned layer buffers; the library allocates nothing.

    pages: uint8 CUDA [batch, n_kv_heads, max_pages, page_bytes]; window: bf16 CUDA
    [batch, n_kv_heads, 2, 32, head_dim]; seq_len: int32 CUDA [batch]; Q bf16 / out fp32 CUDA.
    """
    import torch
    if Q.dtype != torch.bfloat16 or out.dtype != torch.float32 or seq_len.dtype != torch.int32:
        raise ValueError("Q must be bfloat16, out float32 and seq_len int32")
    _check(lib.kvq_decode_attn_noalloc(_pair(pair), int(head_dim), int(n_q_heads),
                                       int(n_kv_heads), _dev_ptr(pages), int(max_pages), _dev_ptr(window),
                                       _dev_ptr(seq_len), int(max_seq_len), _dev_ptr(Q), int(Q.shape[0]),
                                       _dev_ptr(out), _stream(stream)))


def kvq_noalloc_check() -> None:
    """Raise if a kvq_decode_attn_noalloc call on the current device gave up on a page copy
    (waits for the device; clears the flag)."""
    _check(lib.kvq_noalloc_check())


def kvq_layer_error(cache, layer):
    """(sum (k-k^)^2, sum k^2, sum (v-v^)^2, sum v^2, quantized elements) of `layer` (synchronises)."""
    out = kvq_error_stats()
    _check(lib.kvq_layer_error(ctypes.c_void_p(cache), int(layer), ctypes.byref(out)))
    return (out.k_sq_err, out.k_sq, out.v_sq_err, out.v_sq, int(out.elements))


def kvq_set_fp8_scales(cache, layer, k_scale, v_scale) -> None:
    """Per-KV-head scales of an fp8 layer (sequences of n_kv_heads floats; host)."""
    ks = (ctypes.c_float * len(k_scale))(*[float(x) for x in k_scale])
    vs = (ctypes.c_float * len(v_scale))(*[float(x) for x in v_scale])
    _check(lib.kvq_set_fp8_scales(ctypes.c_void_p(cache), int(layer), ctypes.cast(ks, ctypes.c_void_p),
                                  ctypes.cast(vs, ctypes.c_void_p)))


def kvq_set_split_pages(cache, pages_per_split: int) -> None:
    _check(lib.kvq_set_split_pages(ctypes.c_void_p(cache), int(pages_per_split)))


def kvq_set_decode_mode(cache, max_pages_per_warp: int) -> None:
    _check(lib.kvq_set_decode_mode(ctypes.c_void_p(cache), int(max_pages_per_warp)))


def kvq_seq_len(cache, layer, seq) -> int:
    return int(lib.kvq_seq_len(ctypes.c_void_p(cache), int(layer), int(seq)))


def kvq_bytes(cache, layer, batch, include_metadata=True) -> int:
    return int(lib.kvq_bytes(ctypes.c_void_p(cache), int(layer), int(batch), int(bool(include_metadata))))


def kvq_export_bytes(cache, layer, batch) -> int:
    return int(lib.kvq_export_bytes(ctypes.c_void_p(cache), int(layer), int(batch)))


def kvq_export_layer(cache, layer, batch):
    """Returns the layer's stored state as a numpy uint8 array (synchronises)."""
    import numpy as np
    n = kvq_export_bytes(cache, layer, batch)
    if n < 0:
        raise KVQError(KVQ_EINVAL, "bad layer or batch")
    buf = np.zeros(max(n, 1), dtype=np.uint8)
    _check(lib.kvq_export_layer(ctypes.c_void_p(cache), int(layer), int(batch),
                                ctypes.c_void_p(buf.ctypes.data), buf.size))
    return buf[:n]


def kvq_refresh_lengths(cache) -> None:
    _check(lib.kvq_refresh_lengths(ctypes.c_void_p(cache)))


def kvq_sync(cache) -> None:
    _check(lib.kvq_sync(ctypes.c_void_p(cache)))


def kvq_launch_count(cache) -> int:
    return int(lib.kvq_launch_count(ctypes.c_void_p(cache)))
