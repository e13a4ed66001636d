"""B200-native (sm_100a) linear-memory relation-KL distillation loss.

The hot path of LinearARD's relation distillation: per-row KL between the
row-softmaxed Q/Q, K/K and V/V self-relations of a frozen teacher and a
RoPE-scaled student, and its gradient dL/dX_s, without an N x N matrix.
Compute runs in librelkl.so (tcgen05/TMA kernels); this package only marshals
PyTorch tensors into its C ABI (include/relkl.h).
"""
from .ops import (RelationKL, make_desc, relation_kl, relkl_bwd, relkl_bwd_qkv, relkl_fwd,
                  relkl_fwd_noalloc, relkl_fwd_qkv, relkl_get_device_error, relkl_path_for, relkl_set_wait_timeout_ns,
                  relkl_workspace_bytes, relkl_workspace_init, workspace, relkl_rope_bwd,
                  relkl_weight_grad, student_weight_grads, relkl_cast_bf16)

__all__ = ["RelationKL", "make_desc", "relation_kl", "relkl_bwd", "relkl_bwd_qkv", "relkl_fwd",
           "relkl_fwd_noalloc", "relkl_fwd_qkv", "relkl_get_device_error", "relkl_path_for",
           "relkl_set_wait_timeout_ns", "relkl_workspace_bytes", "relkl_workspace_init",
           "workspace", "relkl_rope_bwd", "relkl_weight_grad", "student_weight_grads",
           "relkl_cast_bf16"]
