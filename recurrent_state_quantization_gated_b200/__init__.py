"""B200-native quantized gated Delta-rule decode (STEPQuant-style recurrent-state quantisation).

The compute path is libstepq.so (CUDA, sm_100a) behind the C ABI of include/stepq.h;
``api`` binds it for PyTorch CUDA tensors, ``runtime`` holds the offline calibration and the
state container built on those calls, and ``synth`` draws the seeded synthetic workloads.
"""
from . import synth  # noqa: F401  (NumPy only)

__version__ = "0.1.0"


def __getattr__(name):
    if name in ("api", "runtime"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
