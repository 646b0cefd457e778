"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each pin is a function of the oracle module so that ``test_oracle_mutants``
can run the same pins against copies of the oracle with a planted mistake
and show that every planted mistake is caught.

* brute-force dense KL on tiny V (the pages state that the dense, the
  forward-chunked and the fused chunked losses are mathematically
  equivalent: blog post "Two systems changes"; the dense variant rebuilds the
  whole teacher probability grid from the cached top-K: Japanese summary,
  method paragraph), through ``torch.nn.functional.kl_div`` and autograd;
* K = 1 reduces to cross-entropy (``torch.nn.functional.cross_entropy``);
* W = 0 gives lse = ln V and loss = ln V - mean teacher entropy
  (``scipy.stats.entropy``);
* teacher logits equal to student logits over the whole vocabulary give a
  zero loss and zero gradients;
* KL >= 0; invariances; central finite differences;
* hand-derived worked examples under ``tests/golden/``;
* the library's variants (empty slots marked by index -1, the student at
  temperature T with the T^2 factor): dense torch references with autograd,
  compaction of empty slots, finite differences.
"""

from __future__ import annotations

import json
import math
import os
import types

import numpy as np
import pytest
import scipy.stats
import torch
import torch.nn.functional as F

import oracle as ORACLE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


# ----------------------------------------------------------------- helpers

def _rand_case(seed, N=7, d=5, V=11, K=4, T=1.0, masked=True, dup=False, neg_inf=False):
    g = torch.Generator().manual_seed(seed)
    H = torch.randn(N, d, generator=g, dtype=torch.float64)
    W = torch.randn(V, d, generator=g, dtype=torch.float64) * 0.7
    idx = torch.stack([torch.randperm(V, generator=g)[:K] for _ in range(N)])
    if dup:
        idx[:, -1] = idx[:, 0]
    logit = torch.randn(N, K, generator=g, dtype=torch.float64) * 2.0
    if neg_inf:
        logit[0, -1] = -math.inf
    mask = (torch.rand(N, generator=g, dtype=torch.float64) > 0.3).double() if masked else torch.ones(N, dtype=torch.float64)
    mask[0] = 1.0
    return H, W, idx, logit, mask, T


def _torch_dense(H, W, idx, logit, mask, T, grad=1.0):
    """Dense reference: full teacher grid + full student log-softmax + kl_div."""
    H = H.clone().requires_grad_(True)
    W = W.clone().requires_grad_(True)
    z = H @ W.T
    logq = torch.log_softmax(z, dim=1)
    p = torch.softmax(logit / T, dim=1)
    P = torch.zeros_like(z).scatter_add(1, idx, p)
    kl = F.kl_div(logq, P, reduction="none").sum(dim=1)
    loss = (mask * kl).sum() / mask.sum()
    (grad * loss).backward()
    return (loss.item(), torch.logsumexp(z, 1).detach().numpy(), H.grad.numpy(), W.grad.numpy())


def _run(orc, H, W, idx, logit, mask, T, grad=1.0, **kw):
    return orc.kd_topk_kl(H.numpy(), W.numpy(), idx.numpy(), logit.numpy(), mask.numpy(), T, grad=grad, **kw)


def _torch_dense_variant(H, W, idx, logit, mask, T, grad=1.0, student_T=False):
    """Dense reference of the library's variants: slots with index -1 hold no
    entry (the teacher softmax runs over the filled slots only; a row with
    none has an all-zero teacher grid), and with ``student_T`` the student
    log-softmax is taken of z / T and the loss multiplied by T^2."""
    H = H.clone().requires_grad_(True)
    W = W.clone().requires_grad_(True)
    z = H @ W.T
    logq = torch.log_softmax(z / T if student_T else z, dim=1)
    filled = idx != -1
    t = torch.where(filled, logit / T, torch.full_like(logit, -math.inf))
    any_filled = filled.any(dim=1, keepdim=True)
    p = torch.where(any_filled, torch.softmax(torch.where(any_filled, t, torch.zeros_like(t)), dim=1),
                    torch.zeros_like(t))
    p = torch.where(filled, p, torch.zeros_like(p))
    P = torch.zeros_like(z).scatter_add(1, torch.where(filled, idx, torch.zeros_like(idx)), p)
    kl = F.kl_div(logq, P, reduction="none").sum(dim=1)
    loss = (T * T if student_T else 1.0) * (mask * kl).sum() / mask.sum()
    (grad * loss).backward()
    lse = torch.logsumexp(z / T if student_T else z, 1)
    return (loss.item(), lse.detach().numpy(), H.grad.numpy(), W.grad.numpy())


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} (scale {scale:.3e})"


# ----------------------------------------------------------------- pins

def pin_bruteforce_dense(orc):
    for seed, kw in [(0, {}), (1, {"T": 0.5}), (2, {"T": 3.0, "K": 11}), (3, {"N": 1, "K": 1}),
                     (4, {"neg_inf": True}), (5, {"masked": False, "V": 64, "K": 9, "N": 16})]:
        H, W, idx, logit, mask, T = _rand_case(seed, **kw)
        r = _run(orc, H, W, idx, logit, mask, T, grad=1.7)
        loss, lse, dH, dW = _torch_dense(H, W, idx, logit, mask, T, grad=1.7)
        _close(r["loss"], loss, 1e-12, f"loss seed {seed}")
        _close(r["lse"], lse, 1e-12, f"lse seed {seed}")
        _close(r["dH"], dH, 1e-12, f"dH seed {seed}")
        _close(r["dW"], dW, 1e-12, f"dW seed {seed}")


def pin_duplicate_gradient(orc):
    # Duplicate indices: the gradient is the dense one with scatter-added p.
    H, W, idx, logit, mask, T = _rand_case(6, dup=True)
    r = _run(orc, H, W, idx, logit, mask, T)
    _, _, dH, dW = _torch_dense(H, W, idx, logit, mask, T)
    _close(r["dH"], dH, 1e-12, "dH dup")
    _close(r["dW"], dW, 1e-12, "dW dup")


def pin_cross_entropy_k1(orc):
    H, W, idx, logit, mask, T = _rand_case(7, K=1, N=9)
    r = _run(orc, H, W, idx, logit, mask, T)
    Hg = H.clone().requires_grad_(True)
    Wg = W.clone().requires_grad_(True)
    ce = F.cross_entropy(Hg @ Wg.T, idx[:, 0], reduction="none")
    loss = (mask * ce).sum() / mask.sum()
    loss.backward()
    _close(r["loss"], loss.item(), 1e-12, "K=1 loss vs cross_entropy")
    _close(r["dH"], Hg.grad.numpy(), 1e-12, "K=1 dH")
    _close(r["dW"], Wg.grad.numpy(), 1e-12, "K=1 dW")


def pin_w_zero(orc):
    H, W, idx, logit, mask, T = _rand_case(8, V=13, K=5, T=1.3)
    W = torch.zeros_like(W)
    r = _run(orc, H, W, idx, logit, mask, T)
    V = W.shape[0]
    _close(r["lse"], np.full(H.shape[0], math.log(V)), 1e-14, "lse = ln V")
    p = torch.softmax(logit / T, dim=1).numpy()
    ent = scipy.stats.entropy(p, axis=1)
    m = mask.numpy()
    expect = float(np.sum(m * (math.log(V) - ent)) / np.sum(m))
    _close(r["loss"], expect, 1e-13, "loss = ln V - H(p)")


def pin_equal_teacher(orc):
    # Integer-valued H, W: z is exact in fp32, so cached fp32 teacher logits
    # can equal the student logits exactly.  K = V covers the whole vocabulary.
    g = torch.Generator().manual_seed(9)
    N, d, V = 6, 4, 10
    H = torch.randint(-2, 3, (N, d), generator=g).double()
    W = torch.randint(-2, 3, (V, d), generator=g).double()
    z = (H @ W.T)
    idx = torch.stack([torch.randperm(V, generator=g) for _ in range(N)])
    logit = torch.gather(z, 1, idx).float().double()
    mask = torch.ones(N, dtype=torch.float64)
    r = _run(orc, H, W, idx, logit, mask, 1.0)
    _close(r["loss"], 0.0, 1e-14, "loss zero")
    _close(r["dH"], np.zeros((N, d)), 1e-14, "dH zero")
    _close(r["dW"], np.zeros((V, d)), 1e-14, "dW zero")


def pin_kl_nonneg(orc):
    for seed in range(10, 14):
        H, W, idx, logit, mask, T = _rand_case(seed, N=12, V=17, K=6)
        r = _run(orc, H, W, idx, logit, mask, T)
        assert np.all(r["term"] > 0.0), "per-token KL must be positive off the equality case"
        assert r["loss"] > 0.0


def pin_invariances(orc):
    H, W, idx, logit, mask, T = _rand_case(15, N=8, V=19, K=7, T=0.8)
    base = _run(orc, H, W, idx, logit, mask, T)
    g = torch.Generator().manual_seed(16)
    perm = torch.randperm(W.shape[0], generator=g)          # new row r holds old row perm[r]
    inv = torch.argsort(perm)
    r = _run(orc, H, W[perm], inv[idx], logit, mask, T)
    _close(r["loss"], base["loss"], 1e-13, "perm loss")
    _close(r["lse"], base["lse"], 1e-13, "perm lse")
    _close(r["dH"], base["dH"], 1e-13, "perm dH")
    _close(r["dW"], base["dW"][perm.numpy()], 1e-13, "perm dW")
    shift = torch.randn(H.shape[0], 1, generator=g, dtype=torch.float64) * 5
    r = _run(orc, H, W, idx, logit + shift, mask, T)
    _close(r["loss"], base["loss"], 1e-12, "teacher shift loss")
    _close(r["dW"], base["dW"], 1e-12, "teacher shift dW")
    r = _run(orc, H, W, idx, logit, mask * 3.5, T)
    _close(r["loss"], base["loss"], 1e-13, "mask scale loss")
    _close(r["dH"], base["dH"], 1e-13, "mask scale dH")


def pin_finite_differences(orc):
    H, W, idx, logit, mask, T = _rand_case(17, N=3, d=8, V=24, K=5, T=1.4)
    grad = 0.9
    r = _run(orc, H, W, idx, logit, mask, T, grad=grad)
    h = 1e-6

    def L(Hx, Wx):
        return grad * orc.kd_topk_kl(Hx, Wx, idx.numpy(), logit.numpy(), mask.numpy(), T, backward=False)["loss"]

    Hn, Wn = H.numpy().copy(), W.numpy().copy()
    for (i, j) in [(0, 0), (1, 3), (2, 7)]:
        Hp, Hm = Hn.copy(), Hn.copy()
        Hp[i, j] += h
        Hm[i, j] -= h
        fd = (L(Hp, Wn) - L(Hm, Wn)) / (2 * h)
        assert abs(fd - r["dH"][i, j]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-9, ("dH", i, j, fd, r["dH"][i, j])
    for (v, j) in [(0, 0), (int(idx[0, 0]), 2), (int(idx[2, 1]), 5), (23, 7)]:
        Wp, Wm = Wn.copy(), Wn.copy()
        Wp[v, j] += h
        Wm[v, j] -= h
        fd = (L(Hn, Wp) - L(Hn, Wm)) / (2 * h)
        assert abs(fd - r["dW"][v, j]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-9, ("dW", v, j, fd, r["dW"][v, j])


def pin_golden(orc):
    data = json.load(open(GOLDEN))
    env = {"math": math, "E": math.e}
    for case in data["cases"]:
        r = orc.kd_topk_kl(np.array(case["H"]), np.array(case["W"]), np.array(case["idx"]),
                           np.array(case["logit"]), np.array(case["mask"]), case["T"])
        ex = case["expect"]
        _close(r["loss"], eval(ex["loss"], env), 1e-14, case["name"] + " loss")
        _close(r["lse"], [eval(e, env) for e in ex["lse"]], 1e-14, case["name"] + " lse")
        _close(r["dH"], [[eval(e, env) for e in row] for row in ex["dH"]], 1e-14, case["name"] + " dH")
        _close(r["dW"], [[eval(e, env) for e in row] for row in ex["dW"]], 1e-14, case["name"] + " dW")


def _empty_slots(idx, seed, frac=0.4, empty_row=True):
    g = torch.Generator().manual_seed(1000 + seed)
    idx = idx.clone()
    idx[torch.rand(idx.shape, generator=g) < frac] = -1
    if empty_row and idx.shape[0] > 2:
        idx[2] = -1
    return idx


def pin_empty_slots_dense(orc):
    # variant: index -1 marks an empty slot; a row without entries adds nothing
    for seed, kw in [(30, {}), (31, {"T": 2.0, "K": 6}), (32, {"V": 40, "K": 12, "N": 9, "masked": False})]:
        H, W, idx, logit, mask, T = _rand_case(seed, **kw)
        idx = _empty_slots(idx, seed)
        r = _run(orc, H, W, idx, logit, mask, T, grad=1.3)
        loss, lse, dH, dW = _torch_dense_variant(H, W, idx, logit, mask, T, grad=1.3)
        _close(r["loss"], loss, 1e-12, f"loss seed {seed}")
        _close(r["lse"], lse, 1e-12, f"lse seed {seed}")
        _close(r["dH"], dH, 1e-12, f"dH seed {seed}")
        _close(r["dW"], dW, 1e-12, f"dW seed {seed}")
        assert r["term"][2] == 0.0 and np.all(r["dH"][2] == 0.0)


def pin_empty_slots_compaction(orc):
    # every row with the same number of filled slots == the cache without them
    H, W, idx, logit, mask, T = _rand_case(33, N=6, V=15, K=7, T=1.4)
    g = torch.Generator().manual_seed(33)
    keep = torch.stack([torch.randperm(7, generator=g)[:4].sort().values for _ in range(6)])
    padded = torch.full_like(idx, -1)
    padded.scatter_(1, keep, idx.gather(1, keep))
    r = _run(orc, H, W, padded, logit, mask, T, grad=0.8)
    c = _run(orc, H, W, idx.gather(1, keep), logit.gather(1, keep), mask, T, grad=0.8)
    for k in ("loss", "lse", "term", "dH", "dW"):
        _close(r[k], c[k], 1e-13, "compaction " + k)


def pin_student_temperature_dense(orc):
    # variant: the student at temperature T too, loss times T^2
    for seed, kw, empty in [(34, {"T": 2.0}, False), (35, {"T": 0.5, "K": 6}, False),
                            (36, {"T": 3.0, "V": 30, "K": 8, "N": 8}, True)]:
        H, W, idx, logit, mask, T = _rand_case(seed, **kw)
        if empty:
            idx = _empty_slots(idx, seed)
        r = _run(orc, H, W, idx, logit, mask, T, grad=0.9, student_T=True)
        loss, lse, dH, dW = _torch_dense_variant(H, W, idx, logit, mask, T, grad=0.9, student_T=True)
        _close(r["loss"], loss, 1e-12, f"loss seed {seed}")
        _close(r["lse"], lse, 1e-12, f"lse seed {seed}")
        _close(r["dH"], dH, 1e-12, f"dH seed {seed}")
        _close(r["dW"], dW, 1e-12, f"dW seed {seed}")


def pin_student_temperature_fd(orc):
    # central finite differences of the variant's loss
    H, W, idx, logit, mask, T = _rand_case(37, N=3, d=4, V=9, K=3, T=1.7)
    Hn, Wn, In, Ln, Mn = H.numpy(), W.numpy(), idx.numpy(), logit.numpy(), mask.numpy()
    r = orc.kd_topk_kl(Hn, Wn, In, Ln, Mn, T, grad=1.0, student_T=True)
    L = lambda a, b: orc.kd_topk_kl(a, b, In, Ln, Mn, T, backward=False, student_T=True)["loss"]
    h = 1e-6
    for (i, j) in [(0, 0), (1, 2), (2, 3)]:
        Hp, Hm = Hn.copy(), Hn.copy()
        Hp[i, j] += h
        Hm[i, j] -= h
        fd = (L(Hp, Wn) - L(Hm, Wn)) / (2 * h)
        assert abs(fd - r["dH"][i, j]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-9, ("dH", i, j, fd, r["dH"][i, j])
    for (v, j) in [(0, 1), (4, 0), (8, 3)]:
        Wp, Wm = Wn.copy(), Wn.copy()
        Wp[v, j] += h
        Wm[v, j] -= h
        fd = (L(Hn, Wp) - L(Hn, Wm)) / (2 * h)
        assert abs(fd - r["dW"][v, j]) <= 1e-6 * max(1e-3, abs(fd)) + 1e-9, ("dW", v, j, fd, r["dW"][v, j])


PINS = [pin_bruteforce_dense, pin_duplicate_gradient, pin_cross_entropy_k1, pin_w_zero,
        pin_equal_teacher, pin_kl_nonneg, pin_invariances, pin_finite_differences, pin_golden,
        pin_empty_slots_dense, pin_empty_slots_compaction, pin_student_temperature_dense,
        pin_student_temperature_fd]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(ORACLE)


# ----------------------------------------------------------------- other oracle behaviour

def test_sum_mask_zero():
    H, W, idx, logit, mask, T = _rand_case(18)
    r = _run(ORACLE, H, W, idx, logit, torch.zeros_like(mask), T)
    assert r["loss"] == 0.0
    assert np.all(r["dH"] == 0.0) and np.all(r["dW"] == 0.0)
    assert np.all(np.isfinite(r["lse"]))


def test_bad_index_rejected():
    H, W, idx, logit, mask, T = _rand_case(19)
    idx[0, 0] = W.shape[0]
    with pytest.raises(ValueError):
        _run(ORACLE, H, W, idx, logit, mask, T)
    idx[0, 0] = -2          # -1 is an empty slot, any other negative index an error
    with pytest.raises(ValueError):
        _run(ORACLE, H, W, idx, logit, mask, T)


def test_row_helpers_match_full():
    H, W, idx, logit, mask, T = _rand_case(20, N=10, V=23, K=6, T=1.1)
    r = _run(ORACLE, H, W, idx, logit, mask, T, grad=0.7)
    rows = [0, 3, 9]
    lse, term = ORACLE.term_rows(H.numpy(), W.numpy(), idx.numpy(), logit.numpy(), rows, T)
    _close(lse, r["lse"][rows], 1e-14, "lse rows")
    _close(ORACLE.lse_rows(H.numpy(), W.numpy(), rows), r["lse"][rows], 1e-14, "lse_rows")
    _close(term, r["term"][rows], 1e-14, "term rows")
    dH = ORACLE.dH_rows(H.numpy(), W.numpy(), idx.numpy(), logit.numpy(), mask.numpy(), rows, T, grad=0.7)
    _close(dH, r["dH"][rows], 1e-14, "dH rows")
    vrows = [0, int(idx[1, 2]), 22]
    dW = ORACLE.dW_rows(H.numpy(), W.numpy(), idx.numpy(), logit.numpy(), mask.numpy(), r["lse"], vrows, T, grad=0.7)
    _close(dW, r["dW"][vrows], 1e-14, "dW rows")


def test_row_blocks_do_not_change_result(monkeypatch):
    H, W, idx, logit, mask, T = _rand_case(21, N=13, V=9, K=3)
    a = _run(ORACLE, H, W, idx, logit, mask, T)
    import oracle.kd_oracle as mod
    monkeypatch.setattr(mod, "_BLOCK_ELEMS", 2 * 9)      # two tokens per block
    b = _run(ORACLE, H, W, idx, logit, mask, T)
    for k in ("lse", "term", "dH", "dW"):
        _close(b[k], a[k], 1e-14, k)


# ----------------------------------------------------------------- planted mistakes

MUTANTS = {
    "lse_drops_max": ("(zmax + np.log(np.sum(np.exp(z - zmax)", "(np.log(np.sum(np.exp(z - zmax)"),
    "term_sign": ("inner = logp - (z_at - lse[:, None])", "inner = logp - (z_at + lse[:, None])"),
    "term_drops_entropy": ("inner = logp - (z_at - lse[:, None])", "inner = -(z_at - lse[:, None])"),
    "teacher_not_normalised": ("logp = t - lse_t", "logp = t - tmax"),
    "temperature_multiplies": ("t = as_f64(logit) / float(T)", "t = as_f64(logit) * float(T)"),
    "scatter_wrong_pairing": ("np.add.at(scat, (rows, idx.reshape(-1)), p.reshape(-1))",
                              "np.add.at(scat, (rows, np.sort(idx, axis=1).reshape(-1)), p.reshape(-1))"),
    "dz_sign": ("return c[:, None] * (q - scat)", "return c[:, None] * (scat - q)"),
    "grad_scale_dropped": ("c = (grad * m / sum_mask)", "c = (m / sum_mask)"),
    "mask_not_normalised": ("loss = float(np.sum(m * term) / sum_mask)", "loss = float(np.sum(m * term) / len(m))"),
    "dW_uses_wrong_operand": ("dW += dz.T @ Hf[s:e]", "dW += dz.T @ Hf[s:e] * 0.5"),
    "dH_dropped_term": ("dH[s:e] = dz @ Wf", "dH[s:e] = (dz * (dz > 0)) @ Wf"),
    "empty_slot_in_softmax": ("t = np.where(filled, t, -np.inf)", "t = np.where(filled, t, t)"),
    "empty_row_keeps_softmax": ("q = np.exp(z - lse[:, None]) * np.sum(p, axis=1, keepdims=True)",
                                "q = np.exp(z - lse[:, None])"),
    "student_T_not_squared": ("tfac = float(T) ** 2 if student_T else 1.0", "tfac = float(T) if student_T else 1.0"),
    "student_T_student_unscaled": ("zs = 1.0 / float(T) if student_T else 1.0", "zs = 1.0"),
    "student_T_grad_scale": ("c[s:e] * (tfac * zs)", "c[s:e] * tfac"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_oracle_mutants(name):
    src_path = os.path.join(os.path.dirname(ORACLE.__file__), "kd_oracle.py")
    src = open(src_path).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutant anchor not found once: {old!r}"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"
