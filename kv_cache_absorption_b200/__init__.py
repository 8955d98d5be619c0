"""ISPA warmup hot path on B200 (sm_100a): dual-stream attention, tf32 Gram
accumulation, Cholesky ridge solve for Delta W, and the reconstruction-error
ranking of layers -- CUDA kernels behind a C ABI (include/ispa.h), with a
thin ctypes binding in ``kv_cache_absorption_b200.ispa``."""

__all__ = ["ispa", "warmup"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
