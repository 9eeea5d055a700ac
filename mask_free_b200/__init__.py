"""SAFE-DiT attention hot path for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI shared library ``libsafe_attn.so`` (declared
in ``include/safe_attn.h``); ``mask_free_b200.ops`` is the thin Python
binding over it. The library is loaded on first use, so importing the package
or its ``synth`` input generator needs no GPU.
"""

__all__ = ["ops", "synth"]
