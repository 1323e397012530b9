"""B200-native BigVGAN alias-free waveform decoder.

The computation lives in libbv.so (CUDA for sm_100a, C ABI in include/bv.h);
``native`` is its Python binding and ``synth`` the seeded synthetic inputs.
"""
from . import synth  # noqa: F401


def __getattr__(name):
    if name == "native":
        import importlib
        return importlib.import_module(".native", __name__)
    raise AttributeError(name)
