"""GPU parity of the loss variants (options of the library; none is on the
pages) against the fp64 oracle, through the C ABI's *_ex entry points:

* empty teacher slots (index -1), including tokens with no entry at all;
* a bf16 teacher cache (topk_logit in bf16);
* the student at temperature T with the T^2 factor;
* skipping the rows of masked tokens in the backward pass (the same loss
  and gradients, less work).

Same tolerances as the main parity tests: loss relative error <= 1e-3,
lse absolute error <= 2e-3, relative Frobenius error <= 1e-2 for dH, dW.
"""

from __future__ import annotations

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


def _inputs(N, d, V, K, seed, mask="drop5"):
    cfg = Config(f"variant_N{N}_d{d}_V{V}_K{K}", N, d, V, K, 1.0, 128, w_std=d ** -0.5,
                 teacher="uniform", mask=mask, seed=seed)
    return workloads.make_inputs(cfg)


def _empty_slots(idx, seed, frac=0.3, empty_rows=(5, 17)):
    g = torch.Generator().manual_seed(500 + seed)
    idx = idx.clone()
    idx[torch.rand(idx.shape, generator=g) < frac] = -1
    for r in empty_rows:
        if r < idx.shape[0]:
            idx[r] = -1
    return idx


def _run(kd, x, T, chunk, grad, student_temperature=False, fused=False):
    g = {k: v.cuda() for k, v in x.items()}
    N, d = g["H"].shape
    V, K = g["W"].shape[0], g["topk_idx"].shape[1]
    ws = kd.alloc_workspace(N, d, V, K, chunk, "cuda")
    gl = torch.tensor(grad, dtype=torch.float32, device="cuda")
    if fused:
        loss, lse, dH, dW = kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T,
                                                chunk, grad_loss=gl, workspace=ws,
                                                student_temperature=student_temperature)
    else:
        loss, lse = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, chunk,
                               workspace=ws, student_temperature=student_temperature)
        dH, dW = kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, chunk, lse,
                             grad_loss=gl, workspace=ws, student_temperature=student_temperature)
    st, nbad = kd.check(ws)
    assert st == 0 and nbad == 0, (kd.kd_status_string(st), nbad)
    return {"loss": float(loss.item()), "lse": lse.cpu(), "dH": dH.cpu(), "dW": dW.cpu()}


def _numpy(r):
    return {"loss": r["loss"], "lse": r["lse"].double().numpy(), "dH": r["dH"].double().numpy(),
            "dW": r["dW"].double().numpy()}


def _rfro(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def _assert_parity(got, ref, what):
    got = _numpy(got)
    rel = abs(got["loss"] - ref["loss"]) / max(abs(ref["loss"]), 1e-30)
    assert rel <= LOSS_RTOL, f"{what} loss {got['loss']} vs {ref['loss']} (rel {rel:.2e})"
    err = np.max(np.abs(got["lse"] - ref["lse"]))
    assert err <= LSE_ATOL, f"{what} lse max abs err {err:.2e}"
    for k in ("dH", "dW"):
        e = _rfro(got[k], ref[k])
        assert e <= GRAD_RFRO, f"{what} {k} rel Frobenius err {e:.2e}"


def _oracle(x, T, grad, student_T=False):
    return oracle.kd_topk_kl(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"], T, grad=grad,
                             student_T=student_T)


@pytest.mark.parametrize("shape", [(300, 128, 3000, 16, 64), (700, 512, 5000, 100, 256)],
                         ids=lambda s: "N{}_d{}_V{}_K{}".format(*s[:4]))
def test_empty_teacher_slots(kd, shape):
    N, d, V, K, chunk = shape
    x = _inputs(N, d, V, K, seed=40)
    x["topk_idx"] = _empty_slots(x["topk_idx"], 40)
    got = _run(kd, x, 1.0, chunk, grad=1.3)
    ref = _oracle(x, 1.0, grad=1.3)
    _assert_parity(got, ref, "empty slots")
    # tokens with no entry: zero dH rows (exactly), and no bad-index report
    assert torch.count_nonzero(got["dH"][[5, 17]]) == 0


def test_bf16_teacher_cache(kd):
    x = _inputs(400, 256, 4096, 32, seed=41)
    x["topk_logit"] = x["topk_logit"].to(torch.bfloat16)
    got = _run(kd, x, 1.2, 128, grad=0.8)
    ref = _oracle(x, 1.2, grad=0.8)              # the oracle reads the bf16 values exactly
    _assert_parity(got, ref, "bf16 cache")
    # the kernels widen bf16 exactly: same bits as fp32 logits holding those values
    y = dict(x, topk_logit=x["topk_logit"].float())
    same = _run(kd, y, 1.2, 128, grad=0.8)
    assert got["loss"] == same["loss"]
    for k in ("lse", "dH", "dW"):
        assert torch.equal(got[k], same[k]), k


@pytest.mark.parametrize("T", [2.0, 0.5])
def test_student_temperature(kd, T):
    x = _inputs(500, 192, 3000, 20, seed=42)
    got = _run(kd, x, T, 128, grad=1.1, student_temperature=True)
    ref = _oracle(x, T, grad=1.1, student_T=True)
    _assert_parity(got, ref, f"student T={T}")


def test_variants_combined_fused(kd):
    # empty slots + bf16 cache + student temperature, through the fused call,
    # bitwise equal to the separate calls
    x = _inputs(333, 136, 2049, 24, seed=43)
    x["topk_idx"] = _empty_slots(x["topk_idx"], 43)
    x["topk_logit"] = x["topk_logit"].to(torch.bfloat16)
    a = _run(kd, x, 1.5, 100, grad=0.6, student_temperature=True, fused=True)
    b = _run(kd, x, 1.5, 100, grad=0.6, student_temperature=True, fused=False)
    assert a["loss"] == b["loss"]
    for k in ("lse", "dH", "dW"):
        assert torch.equal(a[k], b[k]), k
    ref = _oracle(x, 1.5, grad=0.6, student_T=True)
    _assert_parity(a, ref, "combined")


def _masked_inputs(N, d, V, K, seed, frac):
    x = _inputs(N, d, V, K, seed=seed, mask="ones")
    g = torch.Generator().manual_seed(900 + seed)
    x["mask"] = (torch.rand(N, generator=g) >= frac).float()
    return x


@pytest.mark.parametrize("frac,chunk,d", [(0.05, 128, 136), (0.6, 64, 136), (1.0, 96, 136), (0.05, 128, 240),
                                          (1.0, 96, 240)],
                         ids=["drop5", "drop60", "all", "drop5_d240", "all_d240"])
def test_skip_masked_rows(kd, frac, chunk, d):
    # the backward over the kept tokens only: the forward is untouched, dH
    # equal bit for bit (every dZ row is computed the same way), dW equal up
    # to the fp32 order of the chunk sums; with 60 % dropped the trailing
    # chunks have no live row, with everything dropped dW must still be zeroed
    x = _masked_inputs(700, d, 3000, 24, seed=44, frac=frac)
    x["topk_idx"] = _empty_slots(x["topk_idx"], 44, frac=0.1, empty_rows=(3,))
    a = _run(kd, x, 1.0, chunk, grad=1.4, student_temperature=False)
    g = {k: v.cuda() for k, v in x.items()}
    ws = kd.alloc_workspace(700, d, 3000, 24, chunk, "cuda")
    dW = torch.full((3000, d), float("nan"), device="cuda")       # overwritten, never read
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(kd.forward_backward_launches(700, chunk, True) + 1)]
    for e in evs:
        e.record()                       # creates the CUDA event behind each object
    loss, lse, dH, dW = kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, chunk,
                                            grad_loss=torch.tensor(1.4, device="cuda"), dW=dW, workspace=ws,
                                            events=evs, skip_masked_rows=True)
    st, nbad = kd.check(ws)
    assert st == 0 and nbad == 0
    b = {"loss": float(loss.item()), "lse": lse.cpu(), "dH": dH.cpu(), "dW": dW.cpu()}
    assert a["loss"] == b["loss"] and torch.equal(a["lse"], b["lse"])
    assert torch.equal(a["dH"], b["dH"])
    assert torch.isfinite(b["dW"]).all()
    if frac < 1.0:
        assert _rfro(b["dW"].double().numpy(), a["dW"].double().numpy()) <= 1e-5
        _assert_parity(b, _oracle(x, 1.0, grad=1.4), "skip rows")
    else:
        assert torch.count_nonzero(b["dW"]) == 0 and torch.count_nonzero(b["dH"]) == 0
    for e in evs:
        e.synchronize()


def test_skip_masked_rows_accumulates(kd):
    x = _masked_inputs(500, 64, 2000, 16, seed=45, frac=0.3)
    g = {k: v.cuda() for k, v in x.items()}
    ws = kd.alloc_workspace(500, 64, 2000, 16, 128, "cuda")
    loss, lse = kd.forward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 128, workspace=ws)
    base = torch.randn(2000, 64, device="cuda") * 1e-4       # the gradient's scale: no cancellation
    dW = base.clone()
    dH, dW = kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 128, lse, dW=dW,
                         accumulate_dW=True, workspace=ws, skip_masked_rows=True)
    _, ref = kd.backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], 1.0, 128, lse, workspace=ws)
    assert kd.check(ws)[0] == 0
    assert _rfro((dW - base).double().cpu().numpy(), ref.double().cpu().numpy()) <= 1e-5
