"""B200-native HiKVP (hierarchical key-value pruning) knowledge-graph attention.

The compute path is the C-ABI library ``libatlaskv.so`` (CUDA, sm_100a) built
from ``csrc/``; ``binding`` marshals arguments to it.  Importing this package
does not load the library: the first call through ``binding`` does, and fails
loudly when the library is missing.
"""
__all__ = ["binding", "synth"]
