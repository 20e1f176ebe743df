"""Batched lossless speculative-sampling verification on NVIDIA B200.

The product is the C-ABI shared library ``libspecverify.so`` (declared in
``include/spec_verify.h``), built by ``build.py``. ``capi`` is its thin
Python binding (same entry-point names, torch tensors in place of pointers);
``workloads`` draws the seeded synthetic inputs.
"""
