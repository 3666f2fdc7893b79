"""B200-native DSA lightning indexer: head-weighted ReLU scores and exact top-K.

The compute path is a C-ABI shared library (``libhwr_indexer.so``, built from
``csrc/``) of hand-written sm_100a kernels; ``indexer`` is a thin ctypes
binding over it.  ``workloads`` draws seeded synthetic inputs.
"""

__all__ = ["indexer", "workloads"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
