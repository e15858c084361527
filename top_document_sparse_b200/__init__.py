"""B200-native Memory Sparse Attention (MSA) hot path.

The compute lives in ``libmsa.so`` (hand-written CUDA for sm_100a behind the C ABI declared in
``include/msa.h``); ``top_document_sparse_b200.msa`` is the thin ctypes binding over it and is
imported explicitly (``from top_document_sparse_b200 import msa``), so the seeded input generators
and workload definitions can be used without loading the library.
"""
from .workloads import WORKLOADS, Workload  # noqa: F401
