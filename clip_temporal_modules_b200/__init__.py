"""B200 (sm_100a) kernels for the clip-parallel temporal modules of Video-Infinity.

The latent video [P positions][F frames][C channels] is cut into N clips along
the frame axis, and CUDA kernels, reached through the C ABI in include/vi.h,
compute the temporal modules with the clip partition inside the kernel grid:

  dual_attn           dual-domain temporal attention (own clip + neighbour
                      context + uniformly sampled global frames)
  temporal_conv       temporal conv1d with neighbour padding, zeros at the ends
  groupnorm_global    GroupNorm with statistics aggregated over every clip
  groupnorm_conv      GroupNorm followed by the conv, fused (no normalised
                      tensor in memory)
  temporal_attention  q/k/v projections + dual_attn + output projection

For a video cut along frames over several GPUs, the *_shard calls compute one
shard from its neighbourhood, and clip_parallel.ClipParallel does the exchange
between ranks.  HostPipeline runs the three modules on pinned host tensors with
the copies overlapped with the kernels.

Python here only marshals arguments; see _binding.py.
"""
from ._binding import (LIB_PATH, ViError, dual_attn, dual_attn_shard,  # noqa: F401
                       groupnorm_conv, groupnorm_global, groupnorm_shard_apply,
                       groupnorm_shard_stats, launch_count, lib, take_device_errors,
                       temporal_attention, temporal_conv, temporal_conv_shard)
from .host_pipeline import HostPipeline, StepShape  # noqa: F401

__all__ = ["dual_attn", "temporal_conv", "groupnorm_global", "groupnorm_conv",
           "temporal_attention", "dual_attn_shard", "temporal_conv_shard",
           "groupnorm_shard_stats", "groupnorm_shard_apply", "take_device_errors",
           "launch_count", "lib", "HostPipeline", "StepShape",
           "ViError", "LIB_PATH"]
