"""The C-ABI library loads, exports every entry point the header declares,
and rejects bad arguments synchronously (no GPU needed: argument checks
return before any CUDA call)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kd_topk_kl.h")


@pytest.fixture(scope="module")
def lib():
    from chunked_top_kl_b200 import build
    build.build()
    import chunked_top_kl_b200 as k
    return k


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kd_[a-z_0-9]+)\s*\(", src)))


def test_exports_match_header(lib):
    declared = _declared_functions()
    assert declared, "no declarations found"
    raw = ctypes.CDLL(lib.build.LIB if hasattr(lib, "build") else None)
    for name in declared:
        assert hasattr(raw, name), f"{name} declared in the header but not exported"
    assert set(declared) == set(lib.EXPORTS)


def test_status_strings(lib):
    for code, name in [(0, "KD_OK"), (1, "KD_ERR_INVALID_ARG"), (2, "KD_ERR_UNSUPPORTED"),
                       (3, "KD_ERR_WORKSPACE"), (4, "KD_ERR_CUDA"), (5, "KD_ERR_BAD_INDEX"),
                       (6, "KD_ERR_TIMEOUT")]:
        assert lib.kd_status_string(code) == name
    assert lib.kd_status_string(99) == "KD_ERR_UNKNOWN"


def test_workspace_size(lib):
    ws = lib.kd_topk_kl_workspace_size
    assert ws(512, 256, 4096, 16, 128) > 0
    assert ws(0, 256, 4096, 16, 128) > 0
    assert ws(512, 250, 4096, 16, 128) == 0          # d % 8
    assert ws(512, 256, 4096, 513, 128) == 0         # K > 512
    assert ws(512, 256, 4096, 16, 0) == 0            # chunk
    assert ws(-1, 256, 4096, 16, 128) == 0
    assert ws(512, 256, 0, 16, 128) == 0
    # linear in N for fixed chunk; the dZ chunk buffer is chunk x round_up(V, 8) bf16
    a, b, c = ws(1 << 14, 2048, 128256, 100, 4096), ws(1 << 15, 2048, 128256, 100, 4096), ws(1 << 16, 2048, 128256, 100, 4096)
    assert abs((c - b) - 2 * (b - a)) <= 4096
    assert ws(4096, 2048, 128256, 100, 1024) < ws(4096, 2048, 128256, 100, 4096)


def test_argument_errors_are_synchronous(lib):
    from chunked_top_kl_b200 import _abi
    F = _abi.kd_topk_kl_forward
    B = _abi.kd_topk_kl_backward
    P = 1 << 20          # a 256-aligned fake device address; never dereferenced on these paths
    N, d, V, K = 512, 256, 4096, 16
    nb = lib.kd_topk_kl_workspace_size(N, d, V, K, 128)
    ok = dict(H=P, W=P, topk_idx=P, topk_logit=P, mask=None, N=N, d=d, V=V, K=K, T=1.0, chunk=128,
              loss=P, lse=P, workspace=P, workspace_bytes=nb, stream=None)

    def fwd(**kw):
        a = dict(ok, **kw)
        return F(a["H"], a["W"], a["topk_idx"], a["topk_logit"], a["mask"], a["N"], a["d"], a["V"],
                 a["K"], a["T"], a["chunk"], a["loss"], a["lse"], a["workspace"], a["workspace_bytes"],
                 a["stream"])

    assert fwd(W=None) == _abi.KD_ERR_INVALID_ARG
    assert fwd(H=None) == _abi.KD_ERR_INVALID_ARG
    assert fwd(H=P + 8) == _abi.KD_ERR_INVALID_ARG            # 16-byte alignment
    assert fwd(workspace=P + 16) == _abi.KD_ERR_INVALID_ARG    # 256-byte alignment
    assert fwd(T=0.0) == _abi.KD_ERR_INVALID_ARG
    assert fwd(T=float("nan")) == _abi.KD_ERR_INVALID_ARG
    assert fwd(T=float("inf")) == _abi.KD_ERR_INVALID_ARG
    assert fwd(N=-3) == _abi.KD_ERR_INVALID_ARG
    assert fwd(chunk=0) == _abi.KD_ERR_INVALID_ARG
    assert fwd(d=100) == _abi.KD_ERR_UNSUPPORTED
    assert fwd(K=600) == _abi.KD_ERR_UNSUPPORTED
    assert fwd(workspace_bytes=nb - 1) == _abi.KD_ERR_WORKSPACE
    assert fwd(loss=None) == _abi.KD_ERR_INVALID_ARG
    assert B(P, P, P, P, None, N, d, V, K, 1.0, 128, P, None, P, None, 0, P, nb, None) == _abi.KD_ERR_INVALID_ARG
    assert B(P, P, P, P, None, N, d, V, K, 1.0, 128, P, None, P + 4, P, 0, P, nb, None) == _abi.KD_ERR_INVALID_ARG
    assert B(P, P, P, P, None, N, d, V, K, 1.0, 128, None, None, P, P, 0, P, nb, None) == _abi.KD_ERR_INVALID_ARG


def test_options_are_validated_first(lib):
    from chunked_top_kl_b200 import _abi
    P = 1 << 20          # never dereferenced: the options are rejected before any other check
    N, d, V, K = 512, 256, 4096, 16
    nb = lib.kd_topk_kl_workspace_size(N, d, V, K, 128)

    def fwd(opt, logit=P):
        return _abi.kd_topk_kl_forward_ex(P, P, P, logit, None, N, d, V, K, 1.0, 128, P, P, P, nb, None, opt)

    bad = _abi.make_options()
    bad.reserved[3] = 1
    assert fwd(bad) == _abi.KD_ERR_INVALID_ARG
    bad = _abi.make_options()
    bad.student_temperature = 2
    assert fwd(bad) == _abi.KD_ERR_INVALID_ARG
    assert _abi.kd_topk_kl_backward_ex(P, P, P, P, None, N, d, V, K, 1.0, 128, P, None, P, P, 0, P, nb,
                                       None, None, bad) == _abi.KD_ERR_INVALID_ARG
    assert _abi.kd_topk_kl_forward_backward_ex(P, P, P, P, None, N, d, V, K, 1.0, 128, P, P, None, P, P, 0,
                                               P, nb, None, None, bad) == _abi.KD_ERR_INVALID_ARG
    # fp32 logits need 4-byte alignment (rejected before anything is enqueued)
    assert fwd(_abi.make_options(), logit=P + 2) == _abi.KD_ERR_INVALID_ARG


def test_binding_checks_caller_buffers(lib):
    """Buffers the caller hands in (dH, dW, lse, workspace, grad_loss) are
    written or read through raw pointers, so the binding checks device, shape,
    dtype and contiguity before any call (host logic, CPU tensors here)."""
    import torch
    from chunked_top_kl_b200 import api
    cpu = torch.device("cpu")
    api._check_buffer(torch.empty(4, 8, dtype=torch.bfloat16), "dH", (4, 8), torch.bfloat16, cpu)
    with pytest.raises(ValueError, match="shape"):
        api._check_buffer(torch.empty(4, 9, dtype=torch.bfloat16), "dH", (4, 8), torch.bfloat16, cpu)
    with pytest.raises(TypeError):
        api._check_buffer(torch.empty(4, 8, dtype=torch.float32), "dH", (4, 8), torch.bfloat16, cpu)
    with pytest.raises(ValueError, match="contiguous"):
        api._check_buffer(torch.empty(8, 4, dtype=torch.bfloat16).t(), "dH", (4, 8), torch.bfloat16, cpu)
    with pytest.raises(ValueError, match="is on"):
        api._check_buffer(torch.empty(4, 8, dtype=torch.bfloat16), "dH", (4, 8), torch.bfloat16,
                          torch.device("meta"))
    api._check_workspace(torch.empty(64, dtype=torch.uint8), cpu)
    for bad in (torch.empty(64, dtype=torch.int8), torch.empty(8, 8, dtype=torch.uint8),
                torch.empty(128, dtype=torch.uint8)[::2]):
        with pytest.raises(ValueError):
            api._check_workspace(bad, cpu)
    assert api._grad_scalar(None, cpu) is None
    g = api._grad_scalar(torch.tensor([2.5], dtype=torch.float64), cpu)
    assert g.shape == () and g.dtype == torch.float32 and float(g) == 2.5
    with pytest.raises(ValueError):
        api._grad_scalar(torch.ones(2), cpu)


def test_noalloc_size_limit(lib):
    """kd_topk_kl_forward_noalloc holds the forward pass's state in a 16 MiB
    array: the header promises every N with (8 Kp + 199) N + 4096 <= 16 MiB
    and rejects every N with (8 Kp + 198) N > 16 MiB (Kp = round_up(K+1, 4)),
    whatever d and V.  Rejection is synchronous, before any CUDA call.  The
    accepted side is checked only on a machine without a CUDA device, where
    the call gets past the size check and then fails at cudaGetDevice (with
    a device it would launch on these fake pointers)."""
    import math
    import torch
    from chunked_top_kl_b200 import _abi
    P = 1 << 20
    F = _abi.kd_topk_kl_forward_noalloc
    no_device = not torch.cuda.is_available()
    for K in (1, 16, 100, 512):
        Kp = 4 * math.ceil((K + 1) / 4)
        n_bad = (16 << 20) // (8 * Kp + 198) + 1
        n_ok = ((16 << 20) - 4096) // (8 * Kp + 199)
        for d, V in ((2880, 201088), (8, 64)):
            assert F(P, P, P, P, None, n_bad, d, V, K, 1.0, P, P, None) == _abi.KD_ERR_WORKSPACE
            if no_device:
                assert F(P, P, P, P, None, n_ok, d, V, K, 1.0, P, P, None) == _abi.KD_ERR_CUDA
    assert F(P, P, P, P, None, 100, 8, 64, 16, 1.0, None, P, None) == _abi.KD_ERR_INVALID_ARG
    assert F(P, P + 8, P, P, None, 100, 8, 64, 16, 1.0, P, P, None) == _abi.KD_ERR_INVALID_ARG
