"""B200-native DSA decode/verify step: ReLU indexer scan, deterministic causal
top-k, gathered sparse GQA attention.  The compute runs in the CUDA library
``libdsa.so`` (sources under ``csrc/``); ``dsa`` is its thin Python binding.
Importing the package does not load the library; the first call does.
"""
__all__ = ["synth", "dsa"]
