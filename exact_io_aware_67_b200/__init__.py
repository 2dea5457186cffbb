"""exact_io_aware_67_b200 -- exact IO-aware attention (FlashAttention-style
forward and recompute backward) as hand-written sm_100a CUDA kernels behind
a small C ABI (``include/fa.h``).

Submodules:
  ``ops``       -- Python binding of the C ABI (argument marshalling only);
  ``build``     -- nvcc build of ``libfa.so`` for sm_100a;
  ``workloads`` -- seeded synthetic inputs (no attention arithmetic);
  ``flops``     -- FLOP and byte accounting used by the benchmark.

The binding is imported lazily so that the pure-host modules work on a
machine without a GPU.
"""

__all__ = ["ops", "build", "workloads", "flops"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
