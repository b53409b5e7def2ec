"""B200-native block-causal chunk attention over a bounded streaming KV cache.

The product is the C-ABI library ``libfd.so`` (declared in ``include/fd.h``);
``binding`` marshals Python arguments to it and nothing more.  ``synth`` and
``workloads`` describe seeded synthetic inputs and workload shapes.
"""
__all__ = ["binding", "synth", "workloads"]
