"""B200-native fused chunked top-K KL distillation loss.

The compute path is libkdtopkl.so (hand-written sm_100a CUDA); this package
is its thin binding: ``_abi`` exposes the C entry points under their own
names, ``api`` wraps them for torch tensors (memory and streams only).
The first call into the library fails loudly (ImportError) if it has not
been built; there is no fallback path.
"""

from ._abi import (EXPORTS, KDError, kd_status_string, kd_teacher_topk, kd_teacher_topk_workspace_size,
                   kd_topk_kl_backward, kd_topk_kl_backward_ex, kd_topk_kl_backward_profiled, kd_topk_kl_check,
                   kd_topk_kl_forward, kd_topk_kl_forward_backward, kd_topk_kl_forward_backward_ex,
                   kd_topk_kl_forward_ex, kd_topk_kl_forward_noalloc, kd_topk_kl_workspace_size, load,
                   kd_selftest_wait_timeout, make_options)
from .api import (KDTopKKLFunction, alloc_workspace, backward, backward_launches, check, forward,
                  forward_backward, forward_backward_launches, kd_topk_kl_loss, teacher_topk, workspace_bytes)

__all__ = [
    "EXPORTS", "KDError", "kd_status_string", "kd_teacher_topk", "kd_teacher_topk_workspace_size",
    "kd_topk_kl_backward", "kd_topk_kl_backward_ex", "kd_topk_kl_backward_profiled", "kd_topk_kl_check",
    "kd_topk_kl_forward", "kd_topk_kl_forward_backward", "kd_topk_kl_forward_backward_ex", "kd_topk_kl_forward_ex",
    "kd_topk_kl_forward_noalloc", "kd_topk_kl_workspace_size", "kd_selftest_wait_timeout", "load", "make_options",
    "KDTopKKLFunction", "alloc_workspace", "backward", "backward_launches", "check", "forward",
    "forward_backward", "forward_backward_launches", "kd_topk_kl_loss", "teacher_topk", "workspace_bytes",
]
