"""B200-native forward of a fine-grained (DeepSeekMoE-style) MoE FFN layer.

The compute path is the C-ABI library built from csrc/ (hand-written sm_100a
CUDA); `moe` is its thin Python binding.  Importing the package loads nothing;
the library is opened on first use and a missing or unloadable library is an
error, never a fallback.
"""
__all__ = ["moe", "inputs", "accounting"]
