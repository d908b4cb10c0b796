"""Paged-KV decode attention for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libpa_b200.so`` (include/pa.h): a
slot-mapped KV-cache append and a paged decode-attention kernel with
split-KV partials and a log-sum-exp merge, all hand-written CUDA.

Modules:
    build     -- compiles csrc/ into libpa_b200.so with nvcc for sm_100a
    binding   -- ctypes marshalling of torch tensors onto the C ABI
    workloads -- seeded synthetic decode batches (inputs only)
"""
