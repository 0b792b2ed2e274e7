"""B200-native (sm_100a) differentiable tile-based Gaussian-splat rasteriser.

The compute path is the CUDA library built from csrc/ (C ABI in
include/gs_api.h); `native` is its ctypes binding and `model` sequences one
training iteration over device-resident parameters. `scenes` generates the
seeded synthetic inputs. Importing the package does not load CUDA; the first
call into `native` does, and raises if the library is missing.
"""

__all__ = ["native", "scenes", "model"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
