"""KLA (Kaczmarz Linear Attention) hot path for NVIDIA B200 (sm_100a).

The public calls live in :mod:`delta_rule_linear_kla_b200.api`; they marshal
torch tensors into the C ABI of ``libkla.so`` (declared in ``include/kla.h``),
whose CUDA kernels do all of the arithmetic.
"""
from .api import (chunk_fwd, decode_step, chunk_fwd_workspace_size,  # noqa: F401
                  KLAError)

__all__ = ["chunk_fwd", "decode_step", "chunk_fwd_workspace_size", "KLAError"]
