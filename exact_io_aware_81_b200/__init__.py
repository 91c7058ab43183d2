"""Exact, IO-aware scaled-dot-product attention for B200 (sm_100a).

The compute lives in ``libfa.so`` (hand-written CUDA for sm_100a behind a C ABI declared
in ``include/fa.h``).  This package holds the thin ctypes binding (``ops``), the build
step (``build``) and the seeded workload generators (``inputs``).  Nothing here computes
attention on the CPU: when the CUDA library is missing, every call raises.
"""
__all__ = ["fwd", "decode", "decode_workspace_size", "get_error", "set_wait_limit_ns", "FAError"]


def __getattr__(name):
    # The binding is imported lazily so that ``exact_io_aware_81_b200.inputs`` can be used
    # on machines where the CUDA library has not been built.
    if name in __all__:
        from . import ops
        return getattr(ops, name)
    raise AttributeError(name)
