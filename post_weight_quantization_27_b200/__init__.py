"""B200-native layer-wise 4-bit post-training weight quantization (GPTQ + RTN).

The compute path is the C-ABI library ``libgq.so`` (hand-written CUDA for
sm_100a, declared in ``include/gq.h``); ``post_weight_quantization_27_b200.gq``
is its thin ctypes binding.  ``inputs`` draws the seeded synthetic layers.
Importing this package does not load the library; ``gq`` loads it and fails
loudly if it is missing.
"""
__all__ = ["gq", "inputs"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
