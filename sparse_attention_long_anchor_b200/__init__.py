"""Kascade sparse attention for B200 (sm_100a).

Import ``sparse_attention_long_anchor_b200.kascade`` for the CUDA library
binding (it loads ``libkascade.so`` and raises if the library is missing) and
``sparse_attention_long_anchor_b200.synth`` for the seeded synthetic inputs.
"""
__all__ = ["kascade", "synth"]
