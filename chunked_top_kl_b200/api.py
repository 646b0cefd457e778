"""Torch-facing wrappers over the C ABI: allocate outputs and workspace with
torch on the tensors' device, pass raw pointers and the current stream, and
raise on a non-zero status.  No arithmetic of the loss happens here."""

from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _abi


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_buffer(t, name: str, shape, dtype, dev) -> None:
    """A caller-supplied tensor the library reads or writes through a raw
    pointer: it must be on ``dev`` with exactly this shape and dtype, and
    contiguous, or the kernels would address memory outside it."""
    if t.device != dev:
        raise ValueError(f"kd_topk_kl: {name} is on {t.device}, the inputs on {dev}")
    if t.dtype != dtype:
        raise TypeError(f"kd_topk_kl: {name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"kd_topk_kl: {name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"kd_topk_kl: {name} must be contiguous")


def _check_workspace(ws, dev) -> None:
    if ws.device != dev or ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous():
        raise ValueError(f"kd_topk_kl: workspace must be a contiguous 1-D uint8 tensor on {dev}")


def _grad_scalar(grad_loss, dev):
    if grad_loss is None:
        return None
    if grad_loss.numel() != 1:
        raise ValueError("kd_topk_kl: grad_loss must hold one value")
    return grad_loss.reshape(()).to(device=dev, dtype=torch.float32).contiguous()


def _check_inputs(H, W, topk_idx, topk_logit, mask):
    if not (H.is_cuda and W.is_cuda and topk_idx.is_cuda and topk_logit.is_cuda):
        raise ValueError("kd_topk_kl: all inputs must be CUDA tensors")
    for t in (W, topk_idx, topk_logit) + ((mask,) if mask is not None else ()):
        if t.device != H.device:
            raise ValueError(f"kd_topk_kl: inputs on {t.device} and {H.device}; all must be on one device")
    if H.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("kd_topk_kl: H and W must be bfloat16")
    if topk_idx.dtype != torch.int32 or topk_logit.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("kd_topk_kl: topk_idx must be int32 and topk_logit float32 or bfloat16")
    if mask is not None and (mask.dtype != torch.float32 or not mask.is_cuda):
        raise TypeError("kd_topk_kl: mask must be a float32 CUDA tensor")
    for t in (H, W, topk_idx, topk_logit) + ((mask,) if mask is not None else ()):
        if not t.is_contiguous():
            raise ValueError("kd_topk_kl: inputs must be contiguous")
    N, d = H.shape
    V = W.shape[0]
    K = topk_idx.shape[1]
    if W.shape[1] != d or topk_idx.shape != (N, K) or topk_logit.shape != (N, K):
        raise ValueError("kd_topk_kl: shape mismatch")
    if mask is not None and mask.shape != (N,):
        raise ValueError("kd_topk_kl: mask must have shape [N]")
    return N, d, V, K


def workspace_bytes(N: int, d: int, V: int, K: int, chunk: int) -> int:
    n = _abi.kd_topk_kl_workspace_size(N, d, V, K, chunk)
    if n == 0:
        raise ValueError("kd_topk_kl: unsupported sizes")
    return n


def alloc_workspace(N, d, V, K, chunk, device) -> torch.Tensor:
    return torch.empty(workspace_bytes(N, d, V, K, chunk), dtype=torch.uint8, device=device)


def _on(dev):
    """The library works on the calling thread's current CUDA device (its
    occupancy figures, tensor maps and the no-allocation scratch address
    come from cudaGetDevice), so every call is made with the inputs' device
    current."""
    return torch.cuda.device(dev)


def _raise(st: int, where: str):
    if st != _abi.KD_OK:
        raise _abi.KDError(st, where)


def _event_handles(events):
    """cudaEvent_t handles of torch.cuda.Event objects; an Event creates its
    CUDA event on first record, so a fresh one is recorded once here."""
    if events is None:
        return None
    for e in events:
        if not e.cuda_event:
            e.record()
    return [e.cuda_event for e in events]


def _options(topk_logit, student_temperature: bool, skip_masked_rows: bool = False):
    """kd_topk_kl_options for these inputs, or None for the default loss
    (fp32 logits, T on the teacher only, every row): the plain entry points
    then run."""
    bf16 = topk_logit.dtype == torch.bfloat16
    if not bf16 and not student_temperature and not skip_masked_rows:
        return None
    return _abi.make_options(logit_bf16=bf16, student_temperature=student_temperature,
                             skip_masked_rows=skip_masked_rows)


def forward(H, W, topk_idx, topk_logit, mask=None, T: float = 1.0, chunk: int = 4096,
            workspace: Optional[torch.Tensor] = None,
            student_temperature: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Returns (loss [] fp32, lse [N] fp32).  ``topk_logit`` may be fp32 or
    bf16; ``student_temperature`` selects the variant with the student
    logits divided by T too and the loss multiplied by T^2."""
    N, d, V, K = _check_inputs(H, W, topk_idx, topk_logit, mask)
    dev = H.device
    if workspace is None:
        workspace = alloc_workspace(N, d, V, K, chunk, dev)
    _check_workspace(workspace, dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = torch.empty(N, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    opt = _options(topk_logit, student_temperature)
    with _on(dev):
        if opt is None:
            st = _abi.kd_topk_kl_forward(_ptr(H), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask),
                                         N, d, V, K, float(T), int(chunk), _ptr(loss), _ptr(lse),
                                         _ptr(workspace), workspace.numel(), stream)
            where = "kd_topk_kl_forward"
        else:
            st = _abi.kd_topk_kl_forward_ex(_ptr(H), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask),
                                            N, d, V, K, float(T), int(chunk), _ptr(loss), _ptr(lse),
                                            _ptr(workspace), workspace.numel(), stream, opt)
            where = "kd_topk_kl_forward_ex"
    _raise(st, where)
    return loss, lse


def backward_launches(N: int, chunk: int, skip_masked_rows: bool = False) -> int:
    """Kernel launches of one backward call (see kd_topk_kl_backward_profiled)."""
    c = (N + chunk - 1) // chunk
    return 0 if N == 0 else (3 + 4 * c if skip_masked_rows else 2 + 2 * c)


def backward(H, W, topk_idx, topk_logit, mask, T: float, chunk: int, lse: torch.Tensor,
             grad_loss: Optional[torch.Tensor] = None, dW: Optional[torch.Tensor] = None,
             accumulate_dW: bool = False, workspace: Optional[torch.Tensor] = None,
             dH: Optional[torch.Tensor] = None, events=None,
             student_temperature: bool = False,
             skip_masked_rows: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Returns (dH [N,d] bf16, dW [V,d] fp32).  With ``events`` (a list of
    backward_launches(N, chunk) + 1 created torch.cuda.Event objects) the
    library records them around each of its kernel launches.
    ``student_temperature`` must match the forward call that made ``lse``;
    ``skip_masked_rows`` skips the rows of tokens with a zero dZ row."""
    N, d, V, K = _check_inputs(H, W, topk_idx, topk_logit, mask)
    dev = H.device
    if workspace is None:
        workspace = alloc_workspace(N, d, V, K, chunk, dev)
    _check_workspace(workspace, dev)
    _check_buffer(lse, "lse", (N,), torch.float32, dev)
    if dH is None:
        dH = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
    _check_buffer(dH, "dH", (N, d), torch.bfloat16, dev)
    if dW is None:
        dW = torch.empty((V, d), dtype=torch.float32, device=dev)
        accumulate_dW = False
    _check_buffer(dW, "dW", (V, d), torch.float32, dev)
    grad_loss = _grad_scalar(grad_loss, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    opt = _options(topk_logit, student_temperature, skip_masked_rows)
    evs = _event_handles(events)
    with _on(dev):
        if opt is not None:
            st = _abi.kd_topk_kl_backward_ex(
                _ptr(H), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), N, d, V, K, float(T),
                int(chunk), _ptr(lse), _ptr(grad_loss), _ptr(dH), _ptr(dW), int(bool(accumulate_dW)),
                _ptr(workspace), workspace.numel(), stream, evs, opt)
            where = "kd_topk_kl_backward_ex"
        elif events is None:
            st = _abi.kd_topk_kl_backward(_ptr(H), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask),
                                          N, d, V, K, float(T), int(chunk), _ptr(lse), _ptr(grad_loss),
                                          _ptr(dH), _ptr(dW), int(bool(accumulate_dW)), _ptr(workspace),
                                          workspace.numel(), stream)
            where = "kd_topk_kl_backward"
        else:
            st = _abi.kd_topk_kl_backward_profiled(
                _ptr(H), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), N, d, V, K, float(T),
                int(chunk), _ptr(lse), _ptr(grad_loss), _ptr(dH), _ptr(dW), int(bool(accumulate_dW)),
                _ptr(workspace), workspace.numel(), stream, evs)
            where = "kd_topk_kl_backward_profiled"
    _raise(st, where)
    return dH, dW


def forward_backward_launches(N: int, chunk: int, skip_masked_rows: bool = False) -> int:
    """Kernel launches of one fused forward + backward call."""
    c = (N + chunk - 1) // chunk
    return 0 if N == 0 else (6 + 4 * c if skip_masked_rows else 5 + 2 * c)


def forward_backward(H, W, topk_idx, topk_logit, mask=None, T: float = 1.0, chunk: int = 4096,
                     grad_loss: Optional[torch.Tensor] = None, dW: Optional[torch.Tensor] = None,
                     accumulate_dW: bool = False, workspace: Optional[torch.Tensor] = None,
                     dH: Optional[torch.Tensor] = None, events=None, student_temperature: bool = False,
                     skip_masked_rows: bool = False):
    """One call for a training step: returns (loss, lse, dH, dW)."""
    N, d, V, K = _check_inputs(H, W, topk_idx, topk_logit, mask)
    dev = H.device
    if workspace is None:
        workspace = alloc_workspace(N, d, V, K, chunk, dev)
    _check_workspace(workspace, dev)
    loss = torch.empty((), dtype=torch.float32, device=dev)
    lse = torch.empty(N, dtype=torch.float32, device=dev)
    if dH is None:
        dH = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
    _check_buffer(dH, "dH", (N, d), torch.bfloat16, dev)
    if dW is None:
        dW = torch.empty((V, d), dtype=torch.float32, device=dev)
        accumulate_dW = False
    _check_buffer(dW, "dW", (V, d), torch.float32, dev)
    grad_loss = _grad_scalar(grad_loss, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    evs = _event_handles(events)
    opt = _options(topk_logit, student_temperature, skip_masked_rows)
    args = (_ptr(H), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), N, d, V, K, float(T), int(chunk),
            _ptr(loss), _ptr(lse), _ptr(grad_loss), _ptr(dH), _ptr(dW), int(bool(accumulate_dW)),
            _ptr(workspace), workspace.numel(), stream)
    with _on(dev):
        if opt is None:
            st, where = _abi.kd_topk_kl_forward_backward(*args, evs), "kd_topk_kl_forward_backward"
        else:
            st, where = _abi.kd_topk_kl_forward_backward_ex(*args, evs, opt), "kd_topk_kl_forward_backward_ex"
    _raise(st, where)
    return loss, lse, dH, dW


def teacher_topk(Ht, Wt, K: int, chunk: int = 1024,
                 workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The teacher top-K cache of hidden states Ht [N,d] under head Wt [V,d]
    (both bf16): returns (topk_idx [N,K] int32, topk_logit [N,K] fp32), each
    row's K largest logits largest first, ties in increasing column order."""
    if not (Ht.is_cuda and Wt.is_cuda) or Ht.dtype != torch.bfloat16 or Wt.dtype != torch.bfloat16:
        raise TypeError("teacher_topk: Ht and Wt must be bfloat16 CUDA tensors")
    if not (Ht.is_contiguous() and Wt.is_contiguous()) or Ht.shape[1] != Wt.shape[1]:
        raise ValueError("teacher_topk: contiguous Ht [N,d] and Wt [V,d] expected")
    if Wt.device != Ht.device:
        raise ValueError("teacher_topk: Ht and Wt must be on one device")
    N, d = Ht.shape
    V = Wt.shape[0]
    dev = Ht.device
    if workspace is None:
        n = _abi.kd_teacher_topk_workspace_size(N, d, V, K, chunk)
        if n == 0:
            raise ValueError("teacher_topk: unsupported sizes")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    _check_workspace(workspace, dev)
    idx = torch.empty((N, K), dtype=torch.int32, device=dev)
    val = torch.empty((N, K), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    with _on(dev):
        st = _abi.kd_teacher_topk(_ptr(Ht), _ptr(Wt), N, d, V, int(K), int(chunk), _ptr(idx), _ptr(val),
                                  _ptr(workspace), workspace.numel(), stream)
    _raise(st, "kd_teacher_topk")
    return idx, val


def check(workspace: torch.Tensor) -> Tuple[int, int]:
    """Synchronise the current stream and read the device status words:
    returns (status, bad_index_count)."""
    stream = torch.cuda.current_stream(workspace.device).cuda_stream
    with _on(workspace.device):
        return _abi.kd_topk_kl_check(_ptr(workspace), stream)


class KDTopKKLFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, topk_idx, topk_logit, mask, T, chunk, student_temperature=False):
        loss, lse = forward(H, W, topk_idx, topk_logit, mask, T, chunk,
                            student_temperature=student_temperature)
        ctx.save_for_backward(H, W, topk_idx, topk_logit, mask, lse)
        ctx.T, ctx.chunk, ctx.student_temperature = T, chunk, student_temperature
        return loss

    @staticmethod
    def backward(ctx, grad):
        H, W, topk_idx, topk_logit, mask, lse = ctx.saved_tensors
        dH, dW = backward(H, W, topk_idx, topk_logit, mask, ctx.T, ctx.chunk, lse,
                          grad_loss=grad.reshape(()), student_temperature=ctx.student_temperature)
        return dH, dW.to(W.dtype), None, None, None, None, None, None


def kd_topk_kl_loss(H, W, topk_idx, topk_logit, mask=None, T: float = 1.0, chunk: int = 4096,
                    student_temperature: bool = False):
    """Differentiable loss (autograd).  dW is accumulated in fp32 inside the
    library and cast to W's dtype for autograd; call ``backward`` directly to
    keep an fp32 gradient."""
    return KDTopKKLFunction.apply(H, W, topk_idx, topk_logit, mask, T, chunk, student_temperature)
