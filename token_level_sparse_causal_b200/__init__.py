"""Token-level sparse causal attention (HySparse2-style prefill) on B200.

The compute path is libhs2.so (hand-written sm_100a CUDA behind a C ABI,
declared in include/hs2.h); `hs2` is its ctypes binding and `inputs` the
seeded workload generator."""
__all__ = ["hs2", "inputs", "build"]
