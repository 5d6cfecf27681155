"""KLA (Kaczmarz Linear Attention) hot path for NVIDIA B200 (sm_100a).

The public calls live in :mod:`delta_rule_linear_kla_b200.api`; they marshal
torch tensors into the C ABI of ``libkla.so`` (declared in ``include/kla.h``),
whose CUDA kernels do all of the arithmetic.
"""
from .autograd import kla_prefill  # noqa: F401
from .api import (KLAError, check_device_error, chunk_fwd, chunk_fwd_host,  # noqa: F401
                  chunk_fwd_states,
                  chunk_fwd_segments, chunk_fwd_workspace_size, chunk_state_fwd,
                  chunk_ut_transform, decode_step, gdn_chunk_fwd, gdn_decode_step,
                  kda_chunk_fwd, kda_chunk_fwd_beta, kda_decode_step, kda_decode_step_beta,
                  kda_fwd, kda_fwd_beta, kda_recurrent_bwd, kda_recurrent_bwd_beta,
                  kda_recurrent_bwd_workspace_size, gdn_recurrent_bwd, chunk_bwd,
                  gdn_chunk_bwd, chunk_bwd_workspace_size,
                  recurrent_bwd, recurrent_bwd_workspace_size, recurrent_fwd)

__all__ = ["kla_prefill", "chunk_fwd", "chunk_fwd_states", "chunk_fwd_host", "chunk_ut_transform", "chunk_state_fwd", "recurrent_fwd",
           "decode_step", "gdn_chunk_fwd", "gdn_decode_step", "chunk_fwd_workspace_size",
           "chunk_fwd_segments", "kda_fwd", "kda_fwd_beta", "kda_chunk_fwd", "kda_chunk_fwd_beta",
           "kda_decode_step",
           "kda_decode_step_beta", "recurrent_bwd", "gdn_recurrent_bwd",
           "recurrent_bwd_workspace_size", "kda_recurrent_bwd", "kda_recurrent_bwd_beta",
           "kda_recurrent_bwd_workspace_size", "chunk_bwd", "gdn_chunk_bwd",
           "chunk_bwd_workspace_size", "check_device_error", "KLAError"]
