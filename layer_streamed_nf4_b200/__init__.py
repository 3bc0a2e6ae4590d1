"""Layer-streamed NF4 LoRA linears for B200 (sm_100a).

The compute lives in a C-ABI shared library (``liblsnf4.so``, declared in
``include/lsnf4.h``); :mod:`layer_streamed_nf4_b200.lsnf4` is its thin ctypes
binding with the same names.  :mod:`layer_streamed_nf4_b200.synth` holds the
seeded synthetic inputs.
"""
__all__ = ["lsnf4", "synth"]
