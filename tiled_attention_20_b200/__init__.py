"""B200-native exact attention (forward and backward) behind a C ABI.

``tiled_attention_20_b200.fa`` is the Python binding of ``libfa.so``; it is
imported lazily so that the CPU-only parts (input generation, host helpers)
work on machines without the CUDA library or a GPU.
"""
__all__ = ["fa", "inputs", "perf"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
