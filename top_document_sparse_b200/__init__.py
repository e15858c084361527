"""B200-native Memory Sparse Attention (MSA) hot path.

The compute lives in ``libmsa.so`` (hand-written CUDA for sm_100a behind a C ABI declared in
``include/msa.h``); ``top_document_sparse_b200.msa`` is the thin ctypes binding over it.  The
binding is imported lazily so that the seeded input generators and workload definitions can be
used without a GPU.
"""
from .workloads import WORKLOADS, Workload  # noqa: F401


def __getattr__(name):
    if name == "msa":
        from . import msa as _msa
        return _msa
    raise AttributeError(name)
