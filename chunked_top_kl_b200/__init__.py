"""B200-native fused chunked top-K KL distillation loss.

The compute path is libkdtopkl.so (hand-written sm_100a CUDA); this package
is its thin binding: ``_abi`` exposes the C entry points under their own
names, ``api`` wraps them for torch tensors (memory and streams only).
Importing fails loudly if the library has not been built.
"""

from ._abi import (EXPORTS, KDError, kd_status_string, kd_topk_kl_backward, kd_topk_kl_check,
                   kd_topk_kl_forward, kd_topk_kl_workspace_size, load)
from .api import (KDTopKKLFunction, alloc_workspace, backward, check, forward, kd_topk_kl_loss,
                  workspace_bytes)

load()

__all__ = [
    "EXPORTS", "KDError", "kd_status_string", "kd_topk_kl_backward", "kd_topk_kl_check",
    "kd_topk_kl_forward", "kd_topk_kl_workspace_size", "KDTopKKLFunction", "alloc_workspace",
    "backward", "check", "forward", "kd_topk_kl_loss", "workspace_bytes",
]
