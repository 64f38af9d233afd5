"""SLoPe 2:4 double-pruned sparse linear layer with a lazy low-rank adapter,
as hand-written sm_100a CUDA kernels behind a C ABI (libslope.so).

Importing the package does not load the CUDA library; the first call of an op
in ``structured_sparse_pretraining_b200.ops`` does, and raises if it is missing.
"""
__all__ = ["ops", "inputs"]
