"""B200-native low-rank-assisted W4A4 linear layer (H-SVDQuant forward).

The compute path is the CUDA library ``libhsq.so`` built from ``csrc/``; the
Python module :mod:`w4a4_rank_assisted_b200.hsq` only marshals arguments to
its C ABI.
"""
