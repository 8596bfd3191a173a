"""B200-native packed joint text+image attention (Mage-Flow NR-MMDiT hot path):
forward, and the backward for training.

The compute lives in ``libmfattn.so`` (hand-written sm_100a CUDA behind the C ABI
in ``include/mf_attn.h``); this package marshals torch tensors into it.
Importing the package does not load the library; the first call does, and
raises if the library has not been built.
"""
from ._native import (MfError, MF_TILE_M, MF_TILE_N, pack_plan, schedule_work,  # noqa: F401
                      workspace_bytes)

__all__ = ["MfError", "MF_TILE_M", "MF_TILE_N", "pack_plan", "schedule_work", "workspace_bytes",
           "PackedPlan", "joint_attention", "joint_attention_host", "qk_prologue",
           "packed_attention", "workspace_views", "device_error", "joint_attention_fwd_lse",
           "joint_attention_bwd", "joint_attention_autograd", "bwd_workspace_bytes",
           "attn_block_fwd", "block_workspace_bytes", "block_workspace_views", "HostPipeline"]


def __getattr__(name):
    if name in ("PackedPlan", "joint_attention", "joint_attention_host", "qk_prologue",
                "packed_attention", "workspace_views", "device_error", "GAMMA_NAMES",
                "joint_attention_fwd_lse", "joint_attention_bwd", "joint_attention_autograd",
                "bwd_workspace_bytes", "JointAttentionFunction", "attn_block_fwd",
                "block_workspace_bytes", "block_workspace_views", "BLOCK_PARAMS",
                "HostPipeline"):
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
