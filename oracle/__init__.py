"""CPU oracle for the paged KV cache hot path (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never imports,
links or calls it, and it shares no code with the CUDA path.

* :mod:`oracle.reference` wraps the plain-C fp64 oracle (``pkv_oracle.c``):
  paged decode attention, per-partition partials and their merge, the slot
  write and the copy-on-write block copy.
* :mod:`oracle.allocator_model` is a pure-Python model of the block pool with
  refcounts and copy-on-write, used to check the native allocator bit-exactly.
"""
