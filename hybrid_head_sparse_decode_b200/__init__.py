"""libychee: the hybrid-head sparse decode-attention step of LycheeDecode on B200.

The compute path is liblychee.so (hand-written sm_100a CUDA kernels behind a C
ABI, include/lychee.h); ``ops`` is its torch-facing binding and ``inputs`` holds
the seeded synthetic workloads.  Importing the package loads nothing: the
library is loaded on the first call.
"""
__all__ = ["ops", "inputs", "build"]
__version__ = "0.1.0"


def __getattr__(name):
    if name in ("ops", "inputs", "build", "_native"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
