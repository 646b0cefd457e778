"""The seeded input generator: determinism and the stated recipe."""

import math

import torch

import workloads
from workloads.configs import CONFIGS


def test_deterministic_and_shapes():
    cfg = workloads.get_config(0)
    a = workloads.make_inputs(cfg)
    b = workloads.make_inputs(cfg)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert a["H"].shape == (cfg.N, cfg.d) and a["H"].dtype == torch.bfloat16
    assert a["W"].shape == (cfg.V, cfg.d) and a["W"].dtype == torch.bfloat16
    assert a["topk_idx"].shape == (cfg.N, cfg.K) and a["topk_idx"].dtype == torch.int32
    assert a["topk_logit"].shape == (cfg.N, cfg.K) and a["topk_logit"].dtype == torch.float32
    assert a["mask"].shape == (cfg.N,)


def test_teacher_recipe():
    cfg = workloads.get_config(0)
    x = workloads.make_inputs(cfg)
    idx = x["topk_idx"].long()
    srt, _ = idx.sort(1)
    assert (srt[:, 1:] != srt[:, :-1]).all(), "indices distinct per token"
    assert idx.min() >= 0 and idx.max() < cfg.V
    lg = x["topk_logit"]
    assert (lg[:, 1:] <= lg[:, :-1]).all(), "sorted descending"
    base = 6.0 - 1.5 * torch.log(torch.arange(1, cfg.K + 1, dtype=torch.float64))
    # Sorting permutes each row, so row sums and sums of squares keep the
    # recipe's moments: mean offset 0 and noise variance 0.1 per entry.
    L = lg.double()
    assert abs(float((L.sum(1) - base.sum()).mean()) / cfg.K) < 0.01
    extra = float((L.pow(2).sum(1) - base.pow(2).sum()).mean()) / cfg.K
    assert abs(extra - 0.1) < 0.03


def test_mask_recipes():
    cfg = CONFIGS[3].with_N(2000)
    m = workloads.make_inputs(cfg.__class__(**{**cfg.__dict__, "d": 8, "V": 300}))["mask"]
    assert int((m == 0).sum()) == round(0.05 * 2000)
    cfg1 = CONFIGS[1]
    small = cfg1.__class__(**{**cfg1.__dict__, "N": 2048, "d": 16, "V": 512})
    x = workloads.make_inputs(small)
    m = x["mask"]
    assert m[0] == 0 and m[1024] == 0
    assert int((m == 0).sum()) == 2 + round(0.10 * 2048)


def test_overlap_recipe():
    cfg1 = CONFIGS[1]
    small = cfg1.__class__(**{**cfg1.__dict__, "N": 64, "d": 32, "V": 1000})
    x = workloads.make_inputs(small)
    z = x["H"].float() @ x["W"].float().T
    top = torch.sort(z, dim=1, descending=True, stable=True)[1][:, :small.K]
    idx = x["topk_idx"].long()
    for n in range(small.N):
        s = set(top[n].tolist())
        assert sum(int(i) in s for i in idx[n].tolist()) == 30
    srt, _ = idx.sort(1)
    assert (srt[:, 1:] != srt[:, :-1]).all()


def test_sample_distinct_exclude():
    g = torch.Generator().manual_seed(0)
    ex = torch.arange(10).repeat(5, 1)
    out = workloads.sample_distinct(g, 5, 8, 20, exclude=ex)
    assert (out >= 10).all()
    assert all(len(set(r.tolist())) == 8 for r in out)
