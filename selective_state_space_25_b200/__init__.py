"""B200-native selective scan: Mamba's selective scan, VMamba's SS2D
four-direction scan and the one-token ``Mamba.step()`` state update, as
hand-written sm_100a CUDA kernels behind a C ABI (``include/ssmscan.h``).

``selective_state_space_25_b200.ssmscan`` is the thin Python binding (ctypes
over ``libssmscan.so``; argument marshalling only).  It is imported lazily so
that ``synthetic`` (seeded input generation) can be used without the CUDA
library; the binding raises at import when ``libssmscan.so`` is missing.
"""
__all__ = ["ssmscan", "synthetic"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
