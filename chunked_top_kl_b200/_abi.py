"""ctypes binding of libkdtopkl.so: the C entry points under the same names.

Argument marshalling only.  Pointers are passed as Python ints (device
addresses), sizes as ints, the stream as an int (cudaStream_t).  Loading
fails loudly when the library has not been built: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

from .build import LIB

KD_OK = 0
KD_ERR_INVALID_ARG = 1
KD_ERR_UNSUPPORTED = 2
KD_ERR_WORKSPACE = 3
KD_ERR_CUDA = 4
KD_ERR_BAD_INDEX = 5
KD_ERR_TIMEOUT = 6

EXPORTS = (
    "kd_status_string",
    "kd_topk_kl_workspace_size",
    "kd_topk_kl_forward",
    "kd_topk_kl_backward",
    "kd_topk_kl_check",
    "kd_topk_kl_forward_noalloc",
    "kd_topk_kl_backward_profiled",
    "kd_topk_kl_forward_backward",
    "kd_topk_kl_forward_ex",
    "kd_topk_kl_backward_ex",
    "kd_topk_kl_forward_backward_ex",
    "kd_teacher_topk_workspace_size",
    "kd_teacher_topk",
    "kd_selftest_wait_timeout",
)


class KDOptions(ctypes.Structure):
    """kd_topk_kl_options (see the C header)."""
    _fields_ = [("logit_bf16", ctypes.c_int32), ("student_temperature", ctypes.c_int32),
                ("skip_masked_rows", ctypes.c_int32), ("reserved", ctypes.c_int32 * 5)]


def make_options(logit_bf16: bool = False, student_temperature: bool = False,
                 skip_masked_rows: bool = False) -> KDOptions:
    o = KDOptions()
    o.logit_bf16 = int(bool(logit_bf16))
    o.student_temperature = int(bool(student_temperature))
    o.skip_masked_rows = int(bool(skip_masked_rows))
    return o


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError(
                f"libkdtopkl.so not found at {LIB}; build it with "
                "`python -m chunked_top_kl_b200.build` (CUDA sm_100a)")
        lib = ctypes.CDLL(LIB)
        p, i64, f32, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_size_t
        lib.kd_status_string.argtypes = [i32]
        lib.kd_status_string.restype = ctypes.c_char_p
        lib.kd_topk_kl_workspace_size.argtypes = [i64, i64, i64, i64, i64]
        lib.kd_topk_kl_workspace_size.restype = sz
        lib.kd_topk_kl_forward.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, i64, p, p, p, sz, p]
        lib.kd_topk_kl_forward.restype = i32
        lib.kd_topk_kl_backward.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, i64, p, p, p, p, i32,
                                            p, sz, p]
        lib.kd_topk_kl_backward.restype = i32
        lib.kd_topk_kl_check.argtypes = [p, p, ctypes.POINTER(i64)]
        lib.kd_topk_kl_check.restype = i32
        lib.kd_topk_kl_backward_profiled.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, i64, p, p, p,
                                                     p, i32, p, sz, p, ctypes.POINTER(ctypes.c_void_p), i64]
        lib.kd_topk_kl_backward_profiled.restype = i32
        lib.kd_topk_kl_forward_backward.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, i64, p, p, p, p, p,
                                                    i32, p, sz, p, ctypes.POINTER(ctypes.c_void_p), i64]
        lib.kd_topk_kl_forward_backward.restype = i32
        lib.kd_topk_kl_forward_noalloc.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, p, p, p]
        lib.kd_topk_kl_forward_noalloc.restype = i32
        opt = ctypes.POINTER(KDOptions)
        evp = ctypes.POINTER(ctypes.c_void_p)
        lib.kd_topk_kl_forward_ex.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, i64, p, p, p, sz, p, opt]
        lib.kd_topk_kl_forward_ex.restype = i32
        lib.kd_topk_kl_backward_ex.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, i64, p, p, p, p, i32,
                                               p, sz, p, evp, i64, opt]
        lib.kd_topk_kl_backward_ex.restype = i32
        lib.kd_topk_kl_forward_backward_ex.argtypes = [p, p, p, p, p, i64, i64, i64, i64, f32, i64, p, p, p,
                                                       p, p, i32, p, sz, p, evp, i64, opt]
        lib.kd_topk_kl_forward_backward_ex.restype = i32
        lib.kd_teacher_topk_workspace_size.argtypes = [i64, i64, i64, i64, i64]
        lib.kd_teacher_topk_workspace_size.restype = sz
        lib.kd_teacher_topk.argtypes = [p, p, i64, i64, i64, i64, i64, p, p, p, sz, p]
        lib.kd_teacher_topk.restype = i32
        lib.kd_selftest_wait_timeout.argtypes = [p, sz, i64, p]
        lib.kd_selftest_wait_timeout.restype = i32
        _lib = lib
    return _lib


class KDError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {kd_status_string(status)}")


def kd_status_string(status: int) -> str:
    return load().kd_status_string(int(status)).decode()


def kd_topk_kl_workspace_size(N: int, d: int, V: int, K: int, chunk: int) -> int:
    return int(load().kd_topk_kl_workspace_size(N, d, V, K, chunk))


def kd_topk_kl_forward(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, loss, lse,
                       workspace, workspace_bytes, stream) -> int:
    return int(load().kd_topk_kl_forward(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk,
                                         loss, lse, workspace, workspace_bytes, stream))


def kd_topk_kl_backward(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, lse, grad_loss,
                        dH, dW, accumulate_dW, workspace, workspace_bytes, stream) -> int:
    return int(load().kd_topk_kl_backward(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk,
                                          lse, grad_loss, dH, dW, int(accumulate_dW), workspace,
                                          workspace_bytes, stream))


def kd_topk_kl_backward_profiled(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, lse,
                                 grad_loss, dH, dW, accumulate_dW, workspace, workspace_bytes, stream,
                                 events) -> int:
    """``events``: a sequence of cudaEvent_t handles (ints), one more than
    the backward pass's launches (2 + 2 * ceil(N / chunk))."""
    arr = (ctypes.c_void_p * len(events))(*events)
    return int(load().kd_topk_kl_backward_profiled(H, W, topk_idx, topk_logit, mask, N, d, V, K, T,
                                                   chunk, lse, grad_loss, dH, dW, int(accumulate_dW),
                                                   workspace, workspace_bytes, stream, arr, len(events)))


def kd_topk_kl_forward_backward(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, loss, lse,
                                grad_loss, dH, dW, accumulate_dW, workspace, workspace_bytes, stream,
                                events=None) -> int:
    """``events``: None, or cudaEvent_t handles (ints), one more than the
    call's launches (5 + 2 * ceil(N / chunk))."""
    if events:
        arr = (ctypes.c_void_p * len(events))(*events)
        n = len(events)
    else:
        arr, n = None, 0
    return int(load().kd_topk_kl_forward_backward(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk,
                                                  loss, lse, grad_loss, dH, dW, int(accumulate_dW),
                                                  workspace, workspace_bytes, stream, arr, n))


def kd_topk_kl_check(workspace, stream) -> tuple[int, int]:
    n = ctypes.c_int64(0)
    st = int(load().kd_topk_kl_check(workspace, stream, ctypes.byref(n)))
    return st, int(n.value)


def kd_topk_kl_forward_noalloc(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, loss, lse,
                               stream) -> int:
    """Forward pass on the library's built-in 16 MiB scratch array, for
    callers that cannot allocate device memory (see the C header)."""
    return int(load().kd_topk_kl_forward_noalloc(H, W, topk_idx, topk_logit, mask, N, d, V, K, T,
                                                 loss, lse, stream))


def _events(events):
    if events:
        return (ctypes.c_void_p * len(events))(*events), len(events)
    return None, 0


def _opt(options):
    return None if options is None else ctypes.byref(options)


def kd_topk_kl_forward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, loss, lse,
                          workspace, workspace_bytes, stream, options=None) -> int:
    return int(load().kd_topk_kl_forward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk,
                                            loss, lse, workspace, workspace_bytes, stream, _opt(options)))


def kd_topk_kl_backward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, lse, grad_loss,
                           dH, dW, accumulate_dW, workspace, workspace_bytes, stream, events=None,
                           options=None) -> int:
    arr, n = _events(events)
    return int(load().kd_topk_kl_backward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk,
                                             lse, grad_loss, dH, dW, int(accumulate_dW), workspace,
                                             workspace_bytes, stream, arr, n, _opt(options)))


def kd_topk_kl_forward_backward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T, chunk, loss, lse,
                                   grad_loss, dH, dW, accumulate_dW, workspace, workspace_bytes, stream,
                                   events=None, options=None) -> int:
    arr, n = _events(events)
    return int(load().kd_topk_kl_forward_backward_ex(H, W, topk_idx, topk_logit, mask, N, d, V, K, T,
                                                     chunk, loss, lse, grad_loss, dH, dW,
                                                     int(accumulate_dW), workspace, workspace_bytes,
                                                     stream, arr, n, _opt(options)))


def kd_teacher_topk_workspace_size(N: int, d: int, V: int, K: int, chunk: int) -> int:
    return int(load().kd_teacher_topk_workspace_size(N, d, V, K, chunk))


def kd_teacher_topk(Ht, Wt, N, d, V, K, chunk, topk_idx, topk_logit, workspace, workspace_bytes, stream) -> int:
    return int(load().kd_teacher_topk(Ht, Wt, N, d, V, K, chunk, topk_idx, topk_logit, workspace,
                                      workspace_bytes, stream))


def kd_selftest_wait_timeout(workspace, workspace_bytes, limit_us, stream) -> int:
    """Launch the failure-detection self-test (see the C header)."""
    return int(load().kd_selftest_wait_timeout(workspace, workspace_bytes, int(limit_us), stream))
