"""Paged KV-cache decode attention for NVIDIA B200 (sm_100a).

The compute lives in ``libpa.so`` (hand-written CUDA, C ABI declared in
``include/pa.h``).  ``paged_kv_cache_382_b200.pa`` is the thin ctypes binding;
importing it loads the library and fails loudly if it has not been built.
``blocks`` is the host block manager, ``workloads`` the seeded synthetic
decode steps used by the tests and the benchmark.
"""

__all__ = ["pa", "blocks", "workloads"]


def __getattr__(name):
    if name in __all__:
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
