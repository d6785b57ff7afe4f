"""B200-native MiniMax Sparse Attention (MSA) forward path.

The CUDA library ``libmsa.so`` (built from ``csrc/``) does all the work; the
Python module :mod:`block_sparse_gqa_04_b200.msa` marshals torch tensors into
its C ABI.  The library is loaded on first use and its absence is an error.
"""
from .workload import WORKLOADS, Workload, make_inputs  # noqa: F401
