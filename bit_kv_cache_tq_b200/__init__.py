"""TurboQuant KV-cache compression and compressed decode attention on B200.

The compute path lives in the C-ABI shared library ``libtq.so`` built from
``csrc/`` (hand-written sm_100a CUDA kernels).  ``bit_kv_cache_tq_b200.tq``
is a thin ctypes binding with the library's own entry-point names; importing
it loads the library and raises if it is missing.  ``inputs`` (seeded
synthetic workloads) imports no compiled code.
"""

__all__ = ["tq", "inputs"]
