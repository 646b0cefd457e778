"""The forward pass for callers that cannot allocate device memory.

kd_topk_kl_forward_noalloc runs the forward pass on a fixed scratch array
built into the library instead of a caller workspace, for callers such as a
runtime that owns all device memory or a plug-in called under its host's
allocator lock.  It runs the same kernels as kd_topk_kl_forward, so its
results must equal that entry point's bit for bit.  Here it is called
through the C ABI twice in a row on different inputs, at a GPT-OSS-shaped
head (d = 2880, V = 201088) with the largest token count its scratch holds
(checked against the fp64 oracle on sampled tokens too), and with a bad
teacher index, which it reports as NaN (its caller has no workspace to read
the status words from), and on an empty batch.  This file sorts last so that a run stopping at the
first failure has already run every other test.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads.configs import Config

pytestmark = pytest.mark.gpu

LSE_ATOL = 2e-3
SCRATCH_BYTES = 16 << 20


def noalloc_max_tokens(K: int) -> int:
    """The largest N the header promises to accept at this K."""
    Kp = 4 * math.ceil((K + 1) / 4)
    return (SCRATCH_BYTES - 4096) // (8 * Kp + 199)


@pytest.fixture(scope="module")
def kd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from chunked_top_kl_b200 import build
    build.build()
    import chunked_top_kl_b200 as k
    k.load()
    return k


def _cfg(N, d, V, K, T, seed, mask, w_std=None):
    return Config(f"noalloc_N{N}_d{d}_V{V}", N, d, V, K, T, 128, w_std=w_std or d ** -0.5,
                  teacher="uniform", mask=mask, seed=seed)


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


def _same_as_workspace_forward(kd, g, T):
    loss_n, lse_n = _noalloc(kd, g, T)
    loss_w, lse_w = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, 128)
    torch.cuda.synchronize()
    assert math.isfinite(loss_n.item())
    assert torch.equal(loss_n, loss_w), (loss_n.item(), loss_w.item())
    assert torch.equal(lse_n, lse_w)
    return lse_n


def test_noalloc_matches_workspace_forward_twice(kd):
    cases = [(512, 256, 4096, 16, 1.0, 1, "ones"), (300, 72, 1000, 7, 0.7, 2, "drop5")]
    for N, d, V, K, T, seed, mask in cases:           # two calls in a row
        g = {k: v.cuda() for k, v in workloads.make_inputs(_cfg(N, d, V, K, T, seed, mask)).items()}
        _same_as_workspace_forward(kd, g, T)


def test_noalloc_at_its_limit_gptoss_head(kd):
    """The largest token count the scratch holds at K = 100, on a
    GPT-OSS-shaped head; the lse of sampled tokens against the oracle."""
    N = noalloc_max_tokens(100)
    cfg = _cfg(N, 2880, 201088, 100, 1.0, 7, "drop5", w_std=0.02)
    x = workloads.make_inputs(cfg)
    g = {k: v.cuda() for k, v in x.items()}
    lse = _same_as_workspace_forward(kd, g, cfg.T)
    rows = np.array(sorted({0, N - 1} | set(np.random.default_rng(7).choice(N, 30, replace=False).tolist())))
    ref = oracle.lse_rows(x["H"], x["W"], rows)
    err = np.abs(lse[torch.from_numpy(rows).cuda()].double().cpu().numpy() - ref)
    assert float(err.max()) <= LSE_ATOL, float(err.max())


def test_noalloc_reports_bad_index_as_nan(kd):
    g = {k: v.cuda() for k, v in workloads.make_inputs(_cfg(256, 64, 1000, 8, 1.0, 3, "ones")).items()}
    bad = dict(g)
    bad["topk_idx"] = g["topk_idx"].clone()
    bad["topk_idx"][5, 2] = 1000                        # == V: outside [0, V)
    loss, lse = _noalloc(kd, bad, 1.0)
    torch.cuda.synchronize()
    assert math.isnan(loss.item())
    assert bool(torch.isnan(lse).all())
    loss, lse = _noalloc(kd, g, 1.0)                   # the next good call is clean again
    torch.cuda.synchronize()
    assert math.isfinite(loss.item()) and bool(torch.isfinite(lse).all())


def test_noalloc_rejects_sizes_beyond_its_scratch(kd):
    from chunked_top_kl_b200 import _abi
    K = 100
    N = 16 * 1024 * 1024 // (8 * 104 + 198) + 1       # first size the header says is rejected
    d, V = 8, 64
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


def test_noalloc_forward_on_an_empty_batch(kd):
    """N = 0: nothing to read, the loss is written as 0 (an empty mask sum)."""
    W = torch.randn(100, 64, device="cuda").to(torch.bfloat16)
    H = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(0, 4, dtype=torch.int32, device="cuda")
    lg = torch.empty(0, 4, dtype=torch.float32, device="cuda")
    loss = torch.full((), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.empty(0, dtype=torch.float32, device="cuda")
    st = kd.kd_topk_kl_forward_noalloc(H.data_ptr() or 256, W.data_ptr(), idx.data_ptr() or 256,
                                       lg.data_ptr() or 256, 0, 0, 64, 100, 4, 1.0, loss.data_ptr(),
                                       lse.data_ptr() or 256, torch.cuda.current_stream().cuda_stream)
    assert st == 0, kd.kd_status_string(st)
    torch.cuda.synchronize()
    assert loss.item() == 0.0
