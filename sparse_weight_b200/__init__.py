"""sparse_weight_b200: tile-hybrid (dense | 2:4) weight GEMV for decode on B200.

``sparse_weight_b200.hyb`` binds the C-ABI library ``libhyb.so`` (CUDA,
sm_100a); ``sparse_weight_b200.inputs`` draws the seeded synthetic workloads.
Importing the package loads nothing; the binding loads the library on first
use and raises if it is missing.
"""
