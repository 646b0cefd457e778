"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element.

Tolerances: loss relative error <= 1e-3, per-token lse absolute error
<= 2e-3, relative Frobenius error <= 1e-2 for dH and dW.  Small and ragged
shapes are compared in full; the large workloads on sampled rows (the oracle
computes those one by one) and on identities that hold at any size.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads.configs import Config

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
LSE_ATOL = 2e-3
GRAD_RFRO = 1e-2


@pytest.fixture(scope="module")
def kd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from chunked_top_kl_b200 import build
    build.build()
    import chunked_top_kl_b200 as k
    return k


def _cfg(N, d, V, K, T=1.0, chunk=128, seed=0, mask="ones", teacher="uniform", w_std=None):
    return Config(f"case_N{N}_d{d}_V{V}_K{K}", N, d, V, K, T, chunk,
                  w_std=(w_std if w_std is not None else d ** -0.5), teacher=teacher, mask=mask, seed=seed)


def _to_dev(x):
    return {k: v.cuda() for k, v in x.items()}


def _gpu(kd, x, T, chunk, grad=None, mask=True):
    g = _to_dev(x)
    m = g["mask"] if mask else None
    ws = kd.alloc_workspace(g["H"].shape[0], g["H"].shape[1], g["W"].shape[0], g["topk_idx"].shape[1],
                            chunk, g["H"].device)
    loss, lse = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], m, T, chunk, workspace=ws)
    st, nbad = kd.check(ws)
    assert st == 0, kd.kd_status_string(st)
    gl = None if grad is None else torch.tensor(grad, dtype=torch.float32, device="cuda")
    dH, dW = kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], m, T, chunk, lse,
                         grad_loss=gl, workspace=ws)
    st, nbad = kd.check(ws)
    assert st == 0, kd.kd_status_string(st)
    torch.cuda.synchronize()
    return {"loss": float(loss.item()), "lse": lse.cpu().double().numpy(),
            "dH": dH.float().cpu().double().numpy(), "dW": dW.cpu().double().numpy()}


def _rfro(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def _assert_parity(got, ref, what=""):
    rel = abs(got["loss"] - ref["loss"]) / max(abs(ref["loss"]), 1e-30)
    assert rel <= LOSS_RTOL, f"{what} loss {got['loss']} vs {ref['loss']} (rel {rel:.2e})"
    lse_err = np.max(np.abs(got["lse"] - ref["lse"]))
    assert lse_err <= LSE_ATOL, f"{what} lse max abs err {lse_err:.2e}"
    for k in ("dH", "dW"):
        e = _rfro(got[k], ref[k])
        assert e <= GRAD_RFRO, f"{what} {k} rel Frobenius err {e:.2e}"


def _oracle(x, T, grad=1.0, mask=True):
    return oracle.kd_topk_kl(x["H"], x["W"], x["topk_idx"], x["topk_logit"],
                             x["mask"] if mask else None, T, grad=grad)


SMALL_CASES = [
    # (N, d, V, K, T, chunk, mask)   ragged in every dimension somewhere
    (512, 256, 4096, 16, 1.0, 128, "ones"),          # the small parity workload's shape
    (300, 72, 1000, 7, 0.7, 100, "drop5"),            # ragged N, d, V; 3 chunks + tail
    (129, 128, 257, 1, 1.0, 64, "ones"),              # K = 1, one column past a tile
    (1, 64, 24, 5, 2.0, 4096, "ones"),                # single token, V < one tile
    (700, 512, 5000, 100, 1.3, 256, "drop5"),         # K = 100, many tiles
    (256, 8, 300, 300, 1.0, 128, "ones"),             # K = V (whole vocabulary), d = 8
    (300, 320, 2000, 12, 1.1, 128, "drop5"),          # d = 2 x 160: dH / dW tiles narrower than 256, dH tail of 32
    (260, 384, 1500, 9, 1.0, 128, "ones"),            # d = 2 x 192: narrow tiles, whole 64-column boxes
    (300, 240, 2000, 12, 1.0, 96, "drop5"),           # d = 240: one tile, dH tail of 48 and dW tail of 16 columns
    (520, 480, 3000, 20, 0.9, 256, "ones"),           # d = 2 x 240 (the 2880 = 12 x 240 split in small)
    (200, 136, 900, 10, 1.0, 64, "ones"),             # d = 136: no equal split, a 256 tile clipped at d
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: "N{}_d{}_V{}_K{}".format(*c[:4]))
def test_parity_small(kd, case):
    N, d, V, K, T, chunk, mask = case
    x = workloads.make_inputs(_cfg(N, d, V, K, T=T, chunk=chunk, mask=mask, seed=N + V))
    ref = _oracle(x, T, grad=1.0)
    got = _gpu(kd, x, T, chunk)
    _assert_parity(got, ref, str(case))


def test_parity_config0_with_grad_and_no_mask(kd):
    cfg = workloads.get_config(0)
    x = workloads.make_inputs(cfg)
    ref = _oracle(x, cfg.T, grad=2.5, mask=False)
    got = _gpu(kd, x, cfg.T, cfg.chunk, grad=2.5, mask=False)
    _assert_parity(got, ref, "config0 grad=2.5")


def test_parity_packed_head_config1(kd):
    cfg = workloads.get_config(1)
    x = workloads.make_inputs(cfg)
    ref = _oracle(x, cfg.T)
    got = _gpu(kd, x, cfg.T, cfg.chunk)
    _assert_parity(got, ref, "config1")
    # masked tokens have exactly zero gradient rows
    masked = (x["mask"].numpy() == 0)
    assert np.all(got["dH"][masked] == 0.0)


def test_negative_upstream_gradient(kd):
    x = workloads.make_inputs(_cfg(300, 72, 1000, 7, T=0.8, mask="drop5", seed=12))
    ref = _oracle(x, 0.8, grad=-1.7)
    got = _gpu(kd, x, 0.8, 100, grad=-1.7)
    _assert_parity(got, ref, "grad=-1.7")


def test_chunk_invariance_and_determinism(kd):
    x = workloads.make_inputs(_cfg(300, 72, 1000, 7, T=0.9, mask="drop5", seed=11))
    base = _gpu(kd, x, 0.9, 300)
    again = _gpu(kd, x, 0.9, 300)
    for k in ("lse", "dH", "dW"):
        assert np.array_equal(base[k], again[k]), f"rerun changed {k}"
    assert base["loss"] == again["loss"]
    for chunk in (1, 64, 128, 299):
        r = _gpu(kd, x, 0.9, chunk)
        assert r["loss"] == base["loss"] and np.array_equal(r["lse"], base["lse"])
        assert np.array_equal(r["dH"], base["dH"]), f"dH depends on chunk={chunk}"
        assert _rfro(r["dW"], base["dW"]) <= 1e-5, f"dW chunk={chunk}"


def test_duplicate_teacher_indices(kd):
    x = workloads.make_inputs(_cfg(200, 64, 700, 6, seed=5))
    x["topk_idx"][:, 3] = x["topk_idx"][:, 0]
    x["topk_idx"][::7, 5] = x["topk_idx"][::7, 0]
    ref = _oracle(x, 1.0)
    got = _gpu(kd, x, 1.0, 64)
    _assert_parity(got, ref, "duplicates")


def test_zero_mask_sum(kd):
    x = workloads.make_inputs(_cfg(130, 64, 600, 4, seed=6))
    x["mask"].zero_()
    ref = _oracle(x, 1.0)
    got = _gpu(kd, x, 1.0, 64)
    assert got["loss"] == 0.0 and ref["loss"] == 0.0
    assert np.all(got["dH"] == 0.0) and np.all(got["dW"] == 0.0)
    assert np.max(np.abs(got["lse"] - ref["lse"])) <= LSE_ATOL


def test_neg_inf_teacher_logit(kd):
    x = workloads.make_inputs(_cfg(140, 64, 900, 8, seed=7))
    x["topk_logit"][::3, -1] = -math.inf
    ref = _oracle(x, 1.0)
    got = _gpu(kd, x, 1.0, 64)
    _assert_parity(got, ref, "-inf logits")


@pytest.mark.parametrize("d", [64, 240])
def test_accumulate_dW(kd, d):
    # d = 240: the last 16 columns of each dW tile are added from registers
    x = workloads.make_inputs(_cfg(200, d, 700, 6, seed=8))
    g = _to_dev(x)
    ws = kd.alloc_workspace(200, d, 700, 6, 64, "cuda")
    _, lse = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, workspace=ws)
    dW0 = torch.randn(700, d, device="cuda")
    _, dW = kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, lse,
                        dW=dW0.clone(), accumulate_dW=True, workspace=ws)
    _, dW1 = kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, lse,
                         workspace=ws)
    torch.cuda.synchronize()
    assert torch.allclose(dW, dW0 + dW1, rtol=0, atol=1e-6)


def test_empty_input(kd):
    H = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.randn(100, 64, device="cuda").to(torch.bfloat16)
    idx = torch.empty(0, 4, dtype=torch.int32, device="cuda")
    lg = torch.empty(0, 4, dtype=torch.float32, device="cuda")
    loss, lse = kd.forward(H, W, idx, lg, None, 1.0, 64)
    dH, dW = kd.backward(H, W, idx, lg, None, 1.0, 64, lse)
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and lse.numel() == 0 and dH.numel() == 0
    assert torch.count_nonzero(dW).item() == 0


def test_bad_index_is_reported(kd):
    x = workloads.make_inputs(_cfg(64, 64, 500, 4, seed=9))
    x["topk_idx"][3, 1] = 500
    x["topk_idx"][9, 0] = -2
    g = _to_dev(x)
    ws = kd.alloc_workspace(64, 64, 500, 4, 64, "cuda")
    kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, workspace=ws)
    st, nbad = kd.check(ws)
    assert st == 5 and nbad == 2
    # the workspace status is per call: a clean call clears it
    g["topk_idx"][3, 1] = 1
    g["topk_idx"][9, 0] = 2
    kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, workspace=ws)
    assert kd.check(ws) == (0, 0)


def test_autograd_wrapper(kd):
    x = workloads.make_inputs(_cfg(256, 128, 1000, 8, seed=10))
    g = _to_dev(x)
    H = g["H"].clone().requires_grad_(True)
    W = g["W"].clone().requires_grad_(True)
    loss = kd.kd_topk_kl_loss(H, W, g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 128)
    (3.0 * loss).backward()
    ref = _oracle(x, 1.0, grad=3.0)
    assert abs(loss.item() - ref["loss"]) / ref["loss"] <= LOSS_RTOL
    assert _rfro(H.grad.float().cpu().double().numpy(), ref["dH"]) <= GRAD_RFRO
    assert _rfro(W.grad.float().cpu().double().numpy(), ref["dW"]) <= GRAD_RFRO


def test_fused_forward_backward_matches_separate_calls(kd):
    for (N, d, V, K, T, chunk) in [(300, 72, 1000, 7, 0.7, 100), (512, 256, 4096, 16, 1.0, 128)]:
        x = workloads.make_inputs(_cfg(N, d, V, K, T=T, mask="drop5", seed=13))
        g = _to_dev(x)
        ws = kd.alloc_workspace(N, d, V, K, chunk, "cuda")
        gl = torch.tensor(1.3, device="cuda")
        loss_a, lse_a = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, chunk, workspace=ws)
        dH_a, dW_a = kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, chunk, lse_a,
                                 grad_loss=gl, workspace=ws)
        n = kd.forward_backward_launches(N, chunk)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        for e in ev:
            e.record()
        loss_b, lse_b, dH_b, dW_b = kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"],
                                                         g["mask"], T, chunk, grad_loss=gl, workspace=ws,
                                                         events=ev)
        torch.cuda.synchronize()
        assert kd.check(ws) == (0, 0)
        assert loss_a.item() == loss_b.item()
        assert torch.equal(lse_a, lse_b) and torch.equal(dH_a, dH_b) and torch.equal(dW_a, dW_b)
        times = [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
        assert all(t >= 0 for t in times)
        ref = _oracle(x, T, grad=1.3)
        _assert_parity({"loss": loss_b.item(), "lse": lse_b.cpu().double().numpy(),
                        "dH": dH_b.float().cpu().double().numpy(), "dW": dW_b.cpu().double().numpy()},
                       ref, f"fused {N}")


def test_event_count_is_checked(kd):
    x = workloads.make_inputs(_cfg(200, 64, 700, 6, seed=14))
    g = _to_dev(x)
    ws = kd.alloc_workspace(200, 64, 700, 6, 64, "cuda")
    _, lse = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, workspace=ws)
    n = kd.backward_launches(200, 64)
    too_few = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in too_few:
        e.record()
    with pytest.raises(kd.KDError):
        kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, lse, workspace=ws,
                    events=too_few)
    with pytest.raises(kd.KDError):
        kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, workspace=ws,
                            events=too_few)


def test_caller_buffers_are_checked(kd):
    """A dH, dW or lse of the wrong shape or dtype is refused before any launch."""
    x = workloads.make_inputs(_cfg(130, 64, 600, 4, seed=15))
    g = _to_dev(x)
    ws = kd.alloc_workspace(130, 64, 600, 4, 64, "cuda")
    _, lse = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64, workspace=ws)
    args = (g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 64)
    with pytest.raises(ValueError):
        kd.backward(*args, lse, workspace=ws, dH=torch.empty(129, 64, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(TypeError):
        kd.backward(*args, lse, workspace=ws, dW=torch.empty(600, 64, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        kd.backward(*args, lse[:-1], workspace=ws)
    with pytest.raises(ValueError):
        kd.forward_backward(*args, workspace=ws, dW=torch.empty(600, 64, device="cpu"))
    torch.cuda.synchronize()
    dH, dW = kd.backward(*args, lse, workspace=ws)     # the same call with valid buffers still runs
    assert kd.check(ws) == (0, 0) and torch.isfinite(dW).all()


def test_calls_run_with_the_inputs_device_current(kd, monkeypatch):
    """The library reads the device from cudaGetDevice, so the binding makes
    the inputs' device current around every call."""
    from chunked_top_kl_b200 import api
    seen = []
    real = api._on

    def spy(dev):
        seen.append(torch.device(dev))
        return real(dev)

    monkeypatch.setattr(api, "_on", spy)
    x = workloads.make_inputs(_cfg(64, 64, 500, 8, seed=11))
    g = _to_dev(x)
    ws = kd.alloc_workspace(64, 64, 500, 8, 32, g["H"].device)
    loss, lse = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 32, workspace=ws)
    kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 32, lse, workspace=ws)
    kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 32, workspace=ws)
    kd.teacher_topk(g["H"], g["W"], 8, chunk=32)
    st, _ = kd.check(ws)
    assert st == 0
    assert len(seen) == 5 and all(d == g["H"].device for d in seen), seen


@pytest.mark.parametrize("skip", [False, True], ids=["all_rows", "skip_masked_rows"])
def test_fused_call_replays_in_a_cuda_graph(kd, skip):
    """The fused call enqueues only stream work on the current stream
    (memsets and kernel launches; skipped rows are counted on the device), so
    a training loop can capture a step in a CUDA graph and replay it.  Each
    replay must give the eager call's results bit for bit."""
    N, d, V, K, chunk = 700, 512, 5000, 100, 256
    g = _to_dev(workloads.make_inputs(_cfg(N, d, V, K, mask="drop5", seed=21)))
    ws = kd.alloc_workspace(N, d, V, K, chunk, "cuda")
    dH = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(V, d, dtype=torch.float32, device="cuda")

    def step():
        return kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, chunk,
                                   workspace=ws, dH=dH, dW=dW, skip_masked_rows=skip)

    loss0, lse0, _, _ = step()
    ref = (loss0.clone(), lse0.clone(), dH.clone(), dW.clone())
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                                   # first calls on the capture stream happen before capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        loss, lse, _, _ = step()
    for _ in range(2):
        dH.fill_(1.0)
        dW.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(loss, ref[0]) and torch.equal(lse, ref[1])
        assert torch.equal(dH, ref[2]) and torch.equal(dW, ref[3])
    st, _ = kd.check(ws)
    assert st == 0
    del graph
