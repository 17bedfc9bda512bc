"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This package holds input generation only and none of the method's
arithmetic: no scoring, no selection, no attention.  Two implementations of
one counter-based generator live here and are cross-checked bit for bit:

* ``gen.counter_hash`` -- host side, numpy;
* ``gen.device``       -- device side, a small CUDA library ``libsagen.so``.

``gen.recipes`` states the shapes, tensor ids and value distributions of the
benchmark workloads.
"""
