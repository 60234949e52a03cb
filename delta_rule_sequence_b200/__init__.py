"""B200-native (sm_100a) gated delta-rule scan with a rank-L residual write.

The compute lives in ``libprism.so`` (hand-written CUDA kernels behind a C ABI, declared in
``include/prism.h``); ``delta_rule_sequence_b200.prism`` is the thin ctypes binding.  Importing
this package does not load the library; the first call does, and fails loudly if it is missing.
"""
__all__ = ["workloads"]
