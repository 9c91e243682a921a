"""Block-sparse attention prefill on B200 (sm_100a).

The compute path lives in the C-ABI shared library ``libsbsa.so`` (CUDA
kernels for pooling, selection and attention); ``sbsa`` is the thin ctypes
binding over it.  The binding is imported lazily so that the workload
generator can be used on machines without the built library.
"""
__all__ = ["sbsa", "workloads"]


def __getattr__(name):
    if name == "sbsa":
        from . import sbsa as mod
        return mod
    if name == "workloads":
        from . import workloads as mod
        return mod
    raise AttributeError(name)
