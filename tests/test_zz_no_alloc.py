"""The forward pass for callers that cannot allocate device memory.

kd_topk_kl_forward_noalloc runs the forward pass on a fixed scratch array
built into the library instead of a caller workspace, for callers such as a
runtime that owns all device memory or a plug-in called under its host's
allocator lock.  Here it is called through the C ABI twice in a row, on
different inputs, and each result is compared with kd_topk_kl_forward's on
a caller-allocated workspace.  This file sorts last so that a run stopping
at the first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import workloads
from workloads.configs import Config

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
LSE_ATOL = 2e-3


@pytest.fixture(scope="module")
def kd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from chunked_top_kl_b200 import build
    build.build()
    import chunked_top_kl_b200 as k
    k.load()
    return k


def _inputs(N, d, V, K, T, seed, mask):
    cfg = Config(f"noalloc_N{N}", N, d, V, K, T, 128, w_std=d ** -0.5, teacher="uniform", mask=mask, seed=seed)
    return {k: v.cuda() for k, v in workloads.make_inputs(cfg).items()}


def _noalloc(kd, g, T):
    N, d = g["H"].shape
    V, K = g["W"].shape[0], g["topk_idx"].shape[1]
    loss = torch.full((), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    st = kd.kd_topk_kl_forward_noalloc(g["H"].data_ptr(), g["W"].data_ptr(), g["topk_idx"].data_ptr(),
                                       g["topk_logit"].data_ptr(), g["mask"].data_ptr(), N, d, V, K,
                                       float(T), loss.data_ptr(), lse.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == 0, kd.kd_status_string(st)
    return loss, lse


def test_noalloc_matches_workspace_forward_twice(kd):
    cases = [(512, 256, 4096, 16, 1.0, 1, "ones"), (300, 72, 1000, 7, 0.7, 2, "drop5")]
    for N, d, V, K, T, seed, mask in cases:           # two calls in a row
        g = _inputs(N, d, V, K, T, seed, mask)
        loss_n, lse_n = _noalloc(kd, g, T)
        loss_w, lse_w = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, 128)
        torch.cuda.synchronize()
        a, b = float(loss_n.item()), float(loss_w.item())
        assert np.isfinite(a) and abs(a - b) <= LOSS_RTOL * abs(b), (N, a, b)
        err = float((lse_n - lse_w).abs().max().item())
        assert err <= LSE_ATOL, (N, err)


def test_noalloc_rejects_sizes_beyond_its_scratch(kd):
    from chunked_top_kl_b200 import _abi
    N, d, V, K = 100_000, 8, 64, 100                   # about 100 MB of state, over the 16 MiB limit
    H = torch.zeros(N, d, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(V, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(N, K, dtype=torch.int32, device="cuda")
    lg = torch.zeros(N, K, dtype=torch.float32, device="cuda")
    loss = torch.zeros((), dtype=torch.float32, device="cuda")
    lse = torch.zeros(N, dtype=torch.float32, device="cuda")
    st = kd.kd_topk_kl_forward_noalloc(H.data_ptr(), W.data_ptr(), idx.data_ptr(), lg.data_ptr(), 0,
                                       N, d, V, K, 1.0, loss.data_ptr(), lse.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == _abi.KD_ERR_WORKSPACE
