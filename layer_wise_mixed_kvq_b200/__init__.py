"""libkvq: B200 decode attention over a layer-wise mixed-precision KV cache (KVTuner).

Submodules:
  kvq    -- Python binding of the C ABI in include/kvq.h (loads libkvq.so)
  build  -- compiles libkvq.so in-tree for sm_100a
  synth  -- seeded synthetic workloads (shapes and distributions only)
"""

__all__ = ["kvq", "build", "synth"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
