"""SAGA + Atop-N single-token decode attention for NVIDIA B200 (sm_100a).

The compute path is libsaga.so (C ABI, include/saga.h) built from csrc/;
`saga` is its Python binding and `workload` draws seeded synthetic inputs.
Importing the package does not load the CUDA library; the binding loads it
on first use and raises if it has not been built.
"""
from . import workload  # noqa: F401

__all__ = ["workload", "saga", "build"]


def __getattr__(name):
    if name in ("saga", "build"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
