"""B200-native (sm_100a) block-sparse attention: ASA block masks, fixed block
patterns and attention over the kept blocks, behind the C ABI in include/bsa.h.

``block_sparse_attention_asa_b200.bsa`` is the Python binding (argument
marshalling over ctypes).  It is imported lazily so that the seeded workload
generator (``workloads``) can be used without the CUDA library.
"""
import importlib

__all__ = ["bsa", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
