"""Routed-MoE FFN layer (Hy3 shapes) on B200: CUDA kernels behind a C ABI.

The compute lives in ``libmoe_b200.so`` (built from ``csrc/``); this package
only marshals arguments to it. Importing the package does not load the
library; the first call into :mod:`.moe` does, and raises if it is missing.
"""
