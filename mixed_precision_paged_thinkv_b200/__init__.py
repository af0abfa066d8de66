"""ThinKV decode hot path for B200 (sm_100a).

    from mixed_precision_paged_thinkv_b200 import ThinKVCache

``ThinKVCache`` (``binding.py``) wraps the C ABI of ``libthinkv.so``
(``include/thinkv.h``): quantize-on-append into reused slots, evict to budget,
and decode attention over the mixed-precision pages.  ``workloads`` holds the
seeded synthetic inputs; ``runner`` drives a workload's setup on a cache.
Importing this package does not load the CUDA library; touching
``ThinKVCache`` does, and fails loudly if it was not built.
"""

__all__ = ["ThinKVCache", "ThinkvError", "workloads", "runner", "binding"]


def __getattr__(name):
    if name in ("ThinKVCache", "ThinkvError"):
        from . import binding
        return getattr(binding, name)
    if name in ("workloads", "runner", "binding", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
