"""B200-native chunked H2O sparse-attention step.

``kv_cache_sparse_b200.binding`` wraps the CUDA library (``libh2o.so``);
``kv_cache_sparse_b200.workloads`` draws the seeded synthetic inputs.
``H2OCache`` and ``CacheShape`` are imported from the binding on first use,
so a missing library fails loudly at that point.
"""

__all__ = ["H2OCache", "CacheShape", "binding", "workloads"]


def __getattr__(name):
    if name in ("H2OCache", "CacheShape", "H2OError"):
        from . import binding
        return getattr(binding, name)
    if name in ("binding", "workloads", "build"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
