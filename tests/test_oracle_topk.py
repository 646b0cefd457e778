"""Pins of the teacher top-K cache oracle (``oracle/topk_cache.py``) to facts
that do not come from it: ``torch.topk`` on tie-free logits, closed forms for
ties, a vocabulary permutation, and the loss oracle (a student distilled
from its own full cache has zero loss).  Planted mistakes in a copy of the
oracle must each fail a pin."""

from __future__ import annotations

import os
import types

import numpy as np
import pytest
import torch

import oracle
import oracle.topk_cache as TOPK


def _case(seed, N=9, d=6, V=40):
    g = torch.Generator().manual_seed(seed)
    H = torch.randn(N, d, generator=g, dtype=torch.float64)
    W = torch.randn(V, d, generator=g, dtype=torch.float64)
    return H.numpy(), W.numpy()


def pin_torch_topk(mod):
    for seed, K in [(0, 1), (1, 7), (2, 40)]:
        H, W = _case(seed)
        idx, val = mod.teacher_topk(H, W, K)
        tv, ti = torch.topk(torch.from_numpy(H @ W.T), K, dim=1, largest=True, sorted=True)
        assert np.array_equal(idx, ti.numpy()), seed
        assert np.allclose(val, tv.numpy(), rtol=0, atol=1e-12), seed


def pin_ties_lower_index_first(mod):
    # W = 0: every logit ties at 0, so the cache is columns 0..K-1
    H, W = _case(3)
    idx, val = mod.teacher_topk(H, np.zeros_like(W), 5)
    assert np.array_equal(idx, np.tile(np.arange(5), (H.shape[0], 1))) and np.all(val == 0.0)
    # two equal columns: the lower one comes first, and both precede smaller logits
    W = np.zeros((6, 2))
    W[1] = W[4] = [1.0, 0.0]
    W[2] = [0.5, 0.0]
    H = np.array([[2.0, 1.0]])
    idx, val = mod.teacher_topk(H, W, 3)
    assert idx.tolist() == [[1, 4, 2]] and val.tolist() == [[2.0, 2.0, 1.0]]


def pin_vocab_permutation(mod):
    H, W = _case(4)
    perm = np.random.default_rng(4).permutation(W.shape[0])
    idx, val = mod.teacher_topk(H, W, 6)
    idx_p, val_p = mod.teacher_topk(H, W[perm], 6)        # row r of W[perm] is row perm[r] of W
    assert np.array_equal(perm[idx_p], idx) and np.array_equal(val_p, val)


def pin_self_distillation(mod):
    # the student's own full cache (K = V) as the teacher: the KD loss is 0
    H, W = _case(5, N=4, d=5, V=12)
    idx, val = mod.teacher_topk(H, W, 12)
    r = oracle.kd_topk_kl(H, W, idx, val, None, 1.0)
    assert abs(r["loss"]) < 1e-12 and np.max(np.abs(r["dH"])) < 1e-12


PINS = [pin_torch_topk, pin_ties_lower_index_first, pin_vocab_permutation, pin_self_distillation]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_topk_oracle_pin(pin):
    pin(TOPK)


def test_topk_oracle_rejects_bad_K():
    H, W = _case(6)
    with pytest.raises(ValueError):
        TOPK.teacher_topk(H, W, 0)
    with pytest.raises(ValueError):
        TOPK.teacher_topk(H, W, W.shape[0] + 1)


MUTANTS = {
    "ascending": ("order = np.argsort(-z, axis=1, kind=\"stable\")[:, :K]",
                  "order = np.argsort(z, axis=1, kind=\"stable\")[:, :K]"),
    "ties_higher_index_first": ("order = np.argsort(-z, axis=1, kind=\"stable\")[:, :K]",
                                "order = (z.shape[1] - 1 - np.argsort(-z[:, ::-1], axis=1, kind=\"stable\"))[:, :K]"),
    "values_not_paired": ("val[s:s + rows] = np.take_along_axis(z, order, axis=1)",
                          "val[s:s + rows] = np.take_along_axis(z, np.sort(order, axis=1), axis=1)"),
    "transposed_head": ("z = H[s:s + rows] @ W.T", "z = (H[s:s + rows] @ W.T)[:, ::-1]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_topk_oracle_mutants(name):
    path = TOPK.__file__
    src = open(path).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, old
    mod = types.ModuleType(f"topk_mutant_{name}")
    mod.__dict__["__package__"] = "oracle"
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"
