"""Parity at the full workload sizes, in the launch configuration bench.py
times: the same chunk, the same fused forward + backward entry point, and
the same choice of backward rows (bench.py skips the rows of masked tokens
when some token is masked and N >= AUTO_SKIP_MIN_N; the GPT-OSS-shaped 32K
head is timed that way).  A masked workload runs both ways and the two must
agree: loss, lse and dH bit for bit, dW up to the fp32 order of its chunk
sums (skipping rows changes which tokens share a chunk).

Expected values: ``tests/golden/fullsize_*.npz``, written by
``tests/golden/make_fullsize_expected.py`` with the fp64 oracle only, hold
the loss and every token's lse.  dH of 512 sampled tokens and dW of 512
sampled vocabulary rows come from the oracle here (``oracle.dH_rows``;
``oracle.dW_rows`` with the stored lse of every token).  The token sample
always includes tokens of the last, partial chunk of the kept-token list,
the chunk boundaries and masked tokens.  The generated inputs are checked
against the SHA-256 stored with them.  On top of that, identities that hold
at any size are checked on the full GPU outputs:

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

import bench
import oracle
import workloads
from workloads.configs import CONFIGS

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = sorted(glob.glob(os.path.join(HERE, "golden", "fullsize_*.npz")))

LOSS_RTOL = 1e-3
LSE_ATOL = 2e-3
GRAD_RFRO = 1e-2
SKIP_DW_RFRO = 1e-5     # dW with and without skipped rows: fp32 summation order only
N_SAMPLE = 512          # sampled dH tokens and dW vocabulary rows


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


def _kept_tokens(x):
    """Tokens whose dZ row can be non-zero (mask != 0 and a teacher entry),
    in order: the rows the backward runs over when masked rows are skipped."""
    keep = (x["mask"] != 0) & (x["topk_idx"] != -1).any(dim=1)
    return torch.nonzero(keep).flatten().numpy()


def _token_sample(cfg, x, index):
    """N_SAMPLE distinct tokens: the first and last token, masked tokens, the
    kept tokens at every chunk boundary of the kept list, 64 tokens of its
    last (partial) chunk, and uniform draws for the rest."""
    rng = np.random.default_rng(100 + index)
    kept = _kept_tokens(x)
    must = {0, cfg.N - 1}
    must.update(int(i) for i in np.nonzero(x["mask"].numpy() == 0)[0][:4])
    for b in range(cfg.chunk, len(kept), cfg.chunk):
        must.update((int(kept[b - 1]), int(kept[b])))
    tail = kept[(len(kept) // cfg.chunk) * cfg.chunk:] if len(kept) % cfg.chunk else kept[-cfg.chunk:]
    must.update(int(i) for i in rng.choice(tail, size=min(64, len(tail)), replace=False))
    must.add(int(kept[-1]))
    rest = np.setdiff1d(np.arange(cfg.N), np.fromiter(must, dtype=np.int64))
    n_more = max(0, min(N_SAMPLE - len(must), len(rest)))
    must.update(int(i) for i in rng.choice(rest, size=n_more, replace=False))
    return np.array(sorted(must), dtype=np.int64)


def _vocab_sample(cfg, x, index):
    """N_SAMPLE distinct vocabulary rows: the first and last, the teacher
    columns of token 0 (rows that get a scattered p) and uniform draws."""
    rng = np.random.default_rng(200 + index)
    must = {0, cfg.V - 1}
    must.update(int(v) for v in x["topk_idx"][0].numpy()[:16] if v >= 0)
    rest = np.setdiff1d(np.arange(cfg.V), np.fromiter(must, dtype=np.int64))
    must.update(int(v) for v in rng.choice(rest, size=N_SAMPLE - len(must), replace=False))
    return np.array(sorted(must), dtype=np.int64)


def _run(kd, cfg, g, skip):
    ws = kd.alloc_workspace(cfg.N, cfg.d, cfg.V, cfg.K, cfg.chunk, "cuda")
    loss, lse, dH, dW = kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], cfg.T,
                                            cfg.chunk, workspace=ws, skip_masked_rows=skip)
    st, nbad = kd.check(ws)
    assert st == 0, kd.kd_status_string(st)
    return loss, lse, dH, dW


@pytest.mark.parametrize("path", CASES, ids=lambda p: os.path.basename(p)[9:-4])
def test_fullsize_parity(kd, path):
    z = np.load(path)
    name, N = str(z["workload"]), int(z["N"])
    index = [c.name for c in CONFIGS].index(name)
    cfg = workloads.get_config(index, N)
    x = workloads.make_inputs(cfg)
    assert _input_sha(x) == str(z["input_sha256"]), "generated inputs differ from the stored ones"
    assert z["lse"].shape == (cfg.N,)

    n_kept = len(_kept_tokens(x))
    bench_skips = n_kept < cfg.N and cfg.N >= bench.AUTO_SKIP_MIN_N
    g = {k: v.cuda() for k, v in x.items()}
    runs = {False: _run(kd, cfg, g, False)}
    if n_kept < cfg.N:
        runs[True] = _run(kd, cfg, g, True)
        a, b = runs[False], runs[True]
        assert torch.equal(a[0], b[0]), (a[0].item(), b[0].item())
        assert torch.equal(a[1], b[1])
        assert torch.equal(a[2], b[2])
        assert float(torch.linalg.norm(a[3] - b[3]) / torch.linalg.norm(a[3])) <= SKIP_DW_RFRO

    # the oracle's values for the samples
    rows = _token_sample(cfg, x, index)
    vrows = _vocab_sample(cfg, x, index)
    ref_dH = oracle.dH_rows(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"], rows, cfg.T)
    ref_dW = oracle.dW_rows(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"],
                            z["lse"].astype(np.float64), vrows, cfg.T)
    ref_loss = float(z["loss"])
    ref_lse = z["lse"].astype(np.float64)

    for skip, (loss, lse, dH, dW) in runs.items():
        where = f"skip_masked_rows={skip}"
        assert abs(loss.item() - ref_loss) <= LOSS_RTOL * abs(ref_loss), (where, loss.item(), ref_loss)
        err = lse.double().cpu().numpy() - ref_lse
        assert np.max(np.abs(err)) <= LSE_ATOL, (where, np.max(np.abs(err)))
        rows_t = torch.from_numpy(rows).cuda()
        e_dH = _rfro(dH[rows_t].double().cpu().numpy(), ref_dH)
        assert e_dH <= GRAD_RFRO, (where, e_dH)
        vrows_t = torch.from_numpy(vrows).cuda()
        e_dW = _rfro(dW[vrows_t].double().cpu().numpy(), ref_dW)
        assert e_dW <= GRAD_RFRO, (where, e_dW)

    # identities on the full outputs of the launch configuration bench.py times
    loss, lse, dH, dW = runs[bench_skips]
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
