"""B200-native fused W4 + sparse-residual linear (MosaicQuant / ZipperEngine).

The compute path lives in the C-ABI library ``libmosaicq.so`` built from
``csrc/`` (hand-written CUDA for sm_100a); ``mosaicq`` is its thin ctypes
binding. ``synth`` holds the seeded synthetic input generators.

The binding is imported lazily so that ``synth`` works without the library.
"""

import importlib

__all__ = ["synth", "mosaicq"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
