"""ETA (Elastic Threshold Attention) block-sparse long-context decode step for
NVIDIA B200 (sm_100a).

The compute path is libeta.so (hand-written CUDA behind the C ABI of
include/eta.h); `_lib` binds it with ctypes and `api.EtaDecoder` wraps one
decode step.  Importing the package does not load the library; the first call
does, and fails loudly if it has not been built.
"""
from . import synth  # noqa: F401  (seeded input generator, no method arithmetic)

__all__ = ["synth", "api", "_lib"]


def __getattr__(name):
    if name in ("api", "_lib"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
