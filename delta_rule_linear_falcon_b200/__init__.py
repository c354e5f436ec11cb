"""libfalcon: the Falcon fast-weight memory forward pass on NVIDIA B200 (sm_100a).

The compute lives in the C-ABI shared library ``libfalcon.so`` (hand-written
CUDA). ``delta_rule_linear_falcon_b200.falcon`` is a thin ctypes binding with
the library's entry-point names; importing this package does not load the
library, so ``inputs`` can be used on a machine without a GPU.
"""
__all__ = ["inputs", "falcon"]
