"""CSA / HCA compressed attention on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libcsa.so`` (hand-written CUDA, see
``include/csa.h``); ``binding`` is a thin ctypes layer over it that only
marshals torch tensors.  ``synth`` draws the seeded synthetic workloads.
"""
__all__ = ["binding", "synth"]


def __getattr__(name):
    if name in ("binding", "synth"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
