"""SSA (Sparse Sparse Attention) dual-stream attention for B200 (sm_100a).

The compute lives in ``libssa.so`` (C ABI, include/ssa.h), bound by
``block_sparse_full_b200.ssa``; ``block_sparse_full_b200.inputs`` draws the
seeded synthetic workloads.  Submodules are imported on demand so that the
input generator works without the built library.
"""
__all__ = ["ssa", "inputs", "build"]
