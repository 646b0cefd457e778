"""Failure detection on the GPU without a fault: the library's pipeline waits
are bounded, and a wait that gives up is reported through the workspace's
status words.  kd_selftest_wait_timeout runs a kernel that waits on a barrier
nothing ever arrives on; the wait must give up within its limit, the host
must read KD_ERR_TIMEOUT, and the device must stay usable (the next loss call
on the same workspace succeeds and reports KD_OK)."""

from __future__ import annotations

import time

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from chunked_top_kl_b200 import build
    build.build()
    import chunked_top_kl_b200 as k
    return k


def test_wait_timeout_is_reported_and_recovered(kd):
    from chunked_top_kl_b200 import _abi
    cfg = workloads.get_config(0)
    x = {k: v.cuda() for k, v in workloads.make_inputs(cfg).items()}
    ws = kd.alloc_workspace(cfg.N, cfg.d, cfg.V, cfg.K, cfg.chunk, "cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    assert kd.kd_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 50_000, stream) == _abi.KD_OK
    st, _ = kd.check(ws)
    waited = time.perf_counter() - t0
    assert st == _abi.KD_ERR_TIMEOUT, kd.kd_status_string(st)
    assert waited < 5.0, waited                      # the 50 ms limit, not a hang
    # the context is still usable and the next call clears the status
    loss, lse = kd.forward(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"], cfg.T, cfg.chunk,
                           workspace=ws)
    st, _ = kd.check(ws)
    assert st == _abi.KD_OK and torch.isfinite(loss).item()


def test_selftest_arguments(kd):
    from chunked_top_kl_b200 import _abi
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    assert kd.kd_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 0, None) == _abi.KD_ERR_INVALID_ARG
    assert kd.kd_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 3_000_000, None) == _abi.KD_ERR_INVALID_ARG
    assert kd.kd_selftest_wait_timeout(ws.data_ptr(), 16, 1000, None) == _abi.KD_ERR_INVALID_ARG
