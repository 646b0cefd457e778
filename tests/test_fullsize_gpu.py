"""Parity at the full workload sizes, in the launch configuration bench.py
times (same chunk, the same fused forward + backward entry point).

Expected values come from ``tests/golden/fullsize_*.npz``, written by
``tests/golden/make_fullsize_expected.py`` with the fp64 oracle only: the
loss, every token's lse (a 4096-token sample above 32768 tokens), dH for
sampled tokens and dW for sampled vocabulary rows.  The generated inputs are
checked against the SHA-256 stored with them.  On top of that, identities
that hold at any size are checked on the full GPU outputs:

* masked tokens have exactly zero dH rows;
* every row of dZ sums to zero (softmax and the teacher distribution both
  sum to one), so the column sums of dW vanish up to the bf16 rounding of
  dZ: |sum_v dW[v,j]| <= 2^-8 sum_n c_n |H[n,j]| (+ fp32 slack);
* <dH, H> = <dW, W> (both equal sum dZ * z), up to the bf16 rounding of dH.
"""

from __future__ import annotations

import glob
import os

import numpy as np
import pytest
import torch

import workloads
from workloads.configs import CONFIGS

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = sorted(glob.glob(os.path.join(HERE, "golden", "fullsize_*.npz")))

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


def _input_sha(x):
    import hashlib
    h = hashlib.sha256()
    for k in ("H", "W", "topk_idx", "topk_logit", "mask"):
        t = x[k].contiguous()
        h.update(t.view(torch.int16).numpy().tobytes() if t.dtype == torch.bfloat16 else t.numpy().tobytes())
    return h.hexdigest()


def _rfro(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("path", CASES, ids=lambda p: os.path.basename(p)[9:-4])
def test_fullsize_parity(kd, path):
    z = np.load(path)
    name, N = str(z["workload"]), int(z["N"])
    index = [c.name for c in CONFIGS].index(name)
    cfg = workloads.get_config(index, N)
    x = workloads.make_inputs(cfg)
    assert _input_sha(x) == str(z["input_sha256"]), "generated inputs differ from the stored ones"

    g = {k: v.cuda() for k, v in x.items()}
    ws = kd.alloc_workspace(cfg.N, cfg.d, cfg.V, cfg.K, cfg.chunk, "cuda")
    loss, lse, dH, dW = kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], cfg.T,
                                            cfg.chunk, workspace=ws)
    st, nbad = kd.check(ws)
    assert st == 0, kd.kd_status_string(st)

    ref_loss = float(z["loss"])
    assert abs(loss.item() - ref_loss) <= LOSS_RTOL * abs(ref_loss), (loss.item(), ref_loss)
    lse_rows = torch.from_numpy(z["lse_rows"]).cuda()
    err = (lse[lse_rows].double().cpu().numpy() - z["lse"].astype(np.float64))
    assert np.max(np.abs(err)) <= LSE_ATOL, np.max(np.abs(err))
    rows = torch.from_numpy(z["rows"]).cuda()
    assert _rfro(dH[rows].double().cpu().numpy(), z["dH_rows"].astype(np.float64)) <= GRAD_RFRO
    vrows = torch.from_numpy(z["vrows"]).cuda()
    assert _rfro(dW[vrows].double().cpu().numpy(), z["dW_rows"].astype(np.float64)) <= GRAD_RFRO

    # identities on the full outputs
    masked = g["mask"] == 0
    if bool(masked.any()):
        assert int(torch.count_nonzero(dH[masked])) == 0
    c = (g["mask"].double() / g["mask"].double().sum())
    colsum = dW.double().sum(0)
    bound = (c[:, None] * g["H"].double().abs()).sum(0) * (2.0 ** -8 + 2e-5)
    assert bool((colsum.abs() <= bound).all()), float((colsum.abs() / bound).max())
    Hd, Wd = g["H"].double(), g["W"].double()
    a = float((dH.double() * Hd).sum())
    b = float((dW.double() * Wd).sum())
    scale = float((dH.double() * Hd).abs().sum() + (dW.double() * Wd).abs().sum())
    assert abs(a - b) <= 2.0 ** -8 * scale, (a, b, scale)
