"""CSA2 decode step on B200: FP4 main-KV cache, FP8 hierarchical sparse indexer.

The compute lives in ``libcsa2.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/csa2.h``).  ``kv_cache_decode_index_b200.csa2`` is the thin
ctypes binding over it; importing that module raises if the library is missing
or the machine has no CUDA device - there is no CPU fallback.

``kv_cache_decode_index_b200.workloads`` holds the seeded synthetic inputs and
does not touch the library.
"""

__all__ = ["csa2", "workloads"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
