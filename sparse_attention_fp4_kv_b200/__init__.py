"""B200-native CSA2 decode hot path (DeepSeek V4.1 Flash sparse attention over
an FP4 main-KV cache).

The compute lives in the C-ABI library ``libcsa2.so`` (hand-written CUDA for
sm_100a, declared in ``include/csa2.h``). ``binding`` is the thin ctypes layer
over it; importing it loads the library and raises if it has not been built.
``synth`` draws the seeded synthetic inputs.
"""
import importlib

__all__ = ["binding", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
