"""B200-native mixed-head causal attention (Selective Attention Freezing).

Ordinary heads run causal softmax attention; replaced heads mix the current V
with a frozen causal pattern rebuilt from two length-T vectors (Eq. (3) of
"When Can Attention Heads Be Statically Defined?").  The compute runs in the
sm_100a CUDA library ``libsaf.so`` behind a C ABI (include/saf.h); the Python
module ``mixed_head_causal_b200.saf`` only marshals torch tensors into it.
"""
__all__ = ["inputs", "saf"]
