"""fp64 CPU oracle for batched lossless speculative-sampling verification.

TEST INFRASTRUCTURE ONLY: a plain, slow, single-threaded restatement of what
the CUDA path computes, used to check it. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import anything from here; the product path never
does and fails loudly when its CUDA library is missing.

Modules
-------
philox  : Philox4x32-10 (Salmon et al., SC'11) and the uniform map.
verify  : one speculative-sampling check, chain verification of a batch and
          the two-stage (L_d -> L_i -> L_f) round with its window.
commit  : paged block-table commit / rollback, KV scatter, hidden-row packing
          and the block-table invariants.
"""
