"""Block-sparse attention prefill on B200 (sm_100a).

The compute path lives in the C-ABI shared library ``libsbsa.so`` (CUDA
kernels for pooling, selection and attention); ``block_sparse_attention_
sbsa_b200.sbsa`` is the thin ctypes binding over it and
``block_sparse_attention_sbsa_b200.workloads`` the seeded input generator.
Submodules are imported explicitly so that the generator works on machines
without the built library.
"""
