"""LittleBit sub-1-bit compressed linear layers on NVIDIA B200 (sm_100a).

The layer computes ``y = x . W^T`` with ``W = W_pri + W_res`` and each path
``diag(h) . U_sign . diag(l) . V_sign^T . diag(g)``, evaluated factor by factor
by hand-written CUDA kernels behind the C ABI in ``include/littlebit.h``.

Importing this package loads nothing; ``sub_bit_weight_b200.lib`` loads the
compiled library (and fails loudly if it is missing).
"""

__all__ = ["synth"]
