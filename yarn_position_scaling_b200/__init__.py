"""B200-native YaRN-RoPE causal GQA attention (prefill and decode) for sm_100a.

The compute path is the C-ABI library ``libyarnattn.so`` (see ``include/yarnattn.h``);
``yarn_position_scaling_b200.api`` is a thin ctypes binding over it.  Importing
this package does not load the library; ``api`` does, and raises if it is missing.
"""
__all__ = ["api", "synth"]
