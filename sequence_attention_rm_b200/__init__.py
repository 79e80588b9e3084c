"""B200-native ring / striped / Ulysses attention hot path.

The compute lives in ``librm_attn.so`` (hand-written sm_100a CUDA behind a C
ABI declared in ``include/rm_attn.h``).  ``sequence_attention_rm_b200.rm``
is the thin Python binding: it marshals torch tensors to pointers and streams
and calls the C entry points of the same names.  Importing the binding on a
machine without the built library raises; there is no CPU fallback.
"""

__all__ = ["rm", "synthetic"]
