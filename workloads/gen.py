"""Seeded generator for the synthetic workloads.

Draw order inside one torch CPU generator seeded with ``cfg.seed`` is fixed:
H, W, teacher indices, teacher noise, mask.  The same seed therefore gives
the same bytes on every machine, and every consumer (oracle, CUDA path,
benchmark) sees identical inputs.

Recipe (stated readings of the workload descriptions):

* ``H ~ N(0, 1)`` and ``W ~ N(0, w_std^2)``, drawn in fp32 and rounded to
  bf16 (round to nearest even).
* Teacher logits: for rank ``k = 0..K-1``, ``6 - 1.5 ln(k+1) + eps`` with
  ``eps`` of variance 0.1 (standard deviation sqrt(0.1)), then sorted
  descending, fp32.  This is a Zipf-shaped top-K list.
* Teacher indices, ``uniform``: K distinct uniform draws from ``[0, V)``.
  ``overlap30``: 30 of the K come from the student's own top-K logits (fp32
  ``H @ W^T`` of the bf16 values, ties to the lower index), chosen
  uniformly without replacement; the rest are uniform distinct draws from
  outside that set; the K indices are then randomly permuted before being
  paired with the sorted teacher logits.
* Mask, ``ones``: all ones.  ``packed10``: zero at the first token of each
  packed 1024-token sequence plus ``round(0.10 N)`` further distinct
  positions.  ``drop5``: ``round(0.05 N)`` distinct zero positions.
"""

from __future__ import annotations

import math
from typing import Dict

import torch

from .configs import Config

SEQ_LEN_PACKED = 1024
OVERLAP = 30


def sample_distinct(gen: torch.Generator, rows: int, k: int, n: int,
                    exclude: torch.Tensor | None = None) -> torch.Tensor:
    """``rows`` x ``k`` int64 draws, distinct within each row, uniform over
    ``[0, n)`` minus ``exclude[row]`` (if given).  Draws that repeat an
    earlier slot of their row, or hit an excluded value, are redrawn until
    none is left; the result depends only on the generator."""
    if k > n - (0 if exclude is None else exclude.shape[1]):
        raise ValueError("not enough distinct values to draw from")
    out = torch.randint(0, n, (rows, k), generator=gen, dtype=torch.int64)
    while True:
        srt, order = out.sort(dim=1, stable=True)
        bad = torch.zeros_like(out, dtype=torch.bool)
        if k > 1:
            rep = torch.zeros_like(out, dtype=torch.bool)
            rep[:, 1:] = srt[:, 1:] == srt[:, :-1]          # later slot of a repeated value
            bad.scatter_(1, order, rep)
        if exclude is not None:
            bad |= (out[:, :, None] == exclude[:, None, :]).any(dim=2)
        nbad = int(bad.sum())
        if nbad == 0:
            return out
        out[bad] = torch.randint(0, n, (nbad,), generator=gen, dtype=torch.int64)


def _student_topk(H: torch.Tensor, W: torch.Tensor, k: int, rows_per_block: int = 512) -> torch.Tensor:
    """Indices of each token's k largest fp32 student logits (ties: lower index)."""
    Wf = W.float()
    outs = []
    for s in range(0, H.shape[0], rows_per_block):
        z = H[s:s + rows_per_block].float() @ Wf.T
        _, order = torch.sort(z, dim=1, descending=True, stable=True)
        outs.append(order[:, :k])
    return torch.cat(outs, 0)


def make_inputs(cfg: Config) -> Dict[str, torch.Tensor]:
    """Return CPU tensors H bf16[N,d], W bf16[V,d], topk_idx int32[N,K],
    topk_logit fp32[N,K], mask fp32[N] for ``cfg`` (seeded by ``cfg.seed``)."""
    N, d, V, K = cfg.N, cfg.d, cfg.V, cfg.K
    if K > V:
        raise ValueError("K must not exceed V")
    gen = torch.Generator().manual_seed(cfg.seed)

    H = torch.randn((N, d), generator=gen, dtype=torch.float32).to(torch.bfloat16)
    W = (torch.randn((V, d), generator=gen, dtype=torch.float32) * cfg.w_std).to(torch.bfloat16)

    if cfg.teacher == "uniform":
        idx = sample_distinct(gen, N, K, V)
    elif cfg.teacher == "overlap30":
        n_ov = min(OVERLAP, K)
        top = _student_topk(H, W, K)                                   # [N, K]
        pick = torch.rand((N, K), generator=gen).argsort(dim=1)[:, :n_ov]
        ov = torch.gather(top, 1, pick)
        rest = sample_distinct(gen, N, K - n_ov, V, exclude=top)
        idx = torch.cat([ov, rest], dim=1)
        perm = torch.rand((N, K), generator=gen).argsort(dim=1)
        idx = torch.gather(idx, 1, perm)
    else:
        raise ValueError(f"unknown teacher recipe {cfg.teacher!r}")

    base = 6.0 - 1.5 * torch.log(torch.arange(1, K + 1, dtype=torch.float64))
    noise = torch.randn((N, K), generator=gen, dtype=torch.float64) * math.sqrt(0.1)
    logit, _ = (base[None, :] + noise).to(torch.float32).sort(dim=1, descending=True)

    mask = torch.ones(N, dtype=torch.float32)
    if cfg.mask == "ones":
        pass
    elif cfg.mask == "packed10":
        starts = torch.arange(0, N, SEQ_LEN_PACKED)
        mask[starts] = 0.0
        others = torch.ones(N, dtype=torch.bool)
        others[starts] = False
        cand = torch.nonzero(others).flatten()
        n_drop = int(round(0.10 * N))
        mask[cand[torch.randperm(cand.numel(), generator=gen)[:n_drop]]] = 0.0
    elif cfg.mask == "drop5":
        n_drop = int(round(0.05 * N))
        mask[torch.randperm(N, generator=gen)[:n_drop]] = 0.0
    else:
        raise ValueError(f"unknown mask recipe {cfg.mask!r}")

    return {
        "H": H.contiguous(),
        "W": W.contiguous(),
        "topk_idx": idx.to(torch.int32).contiguous(),
        "topk_logit": logit.contiguous(),
        "mask": mask,
    }
