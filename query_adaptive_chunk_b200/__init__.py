"""Query-adaptive chunk-sparse attention on B200 (sm_100a).

``query_adaptive_chunk_b200.csa`` is the Python binding of the C-ABI library
``libcsa.so`` (argument marshalling only; every step runs in CUDA kernels).
``query_adaptive_chunk_b200.synth`` draws the seeded synthetic workloads.
Importing the package itself loads nothing, so the input generator is usable
on a machine without the library.
"""
