"""fp64 CPU oracle of the teacher top-K cache writer.

TEST INFRASTRUCTURE ONLY (like ``kd_oracle``): used by ``tests/`` alone; the
CUDA library never imports it and shares no code with it.

What it computes
----------------
The offline distillation set-up of "Efficient Knowledge Distillation for
LLMs: Offline Top-K Logits and a Fused Chunked KL Loss" (blog post, "Two
systems changes", offline distillation paragraph) runs the teacher once
over the data and stores, for every position, the indices and logits of the
teacher's K largest output logits; the loss later renormalises them with a
softmax.  The pages do not say how the cache is written.  The plain reading
for a teacher head with hidden states ``Ht[N,d]`` and weight ``Wt[V,d]``:

  1. ``z[n,v] = sum_j Ht[n,j] Wt[v,j]`` (fp64 from the exact bf16 values);
  2. per token, the K columns with the largest ``z``, ties broken towards the
     lower column index;
  3. written in that order (largest first): ``idx[n,k]`` int32 and
     ``logit[n,k] = z[n, idx[n,k]]``.

A library primitive (numpy's stable sort) does step 2.
"""

from __future__ import annotations

import numpy as np

from .kd_oracle import as_f64

__all__ = ["teacher_topk"]


def teacher_topk(Ht, Wt, K: int):
    """Steps 1-3 for every token: ``(idx [N,K] int64, logit [N,K] fp64)``."""
    H = as_f64(Ht)
    W = as_f64(Wt)
    V = W.shape[0]
    if not 1 <= K <= V:
        raise ValueError("K must be in [1, V]")
    N = H.shape[0]
    idx = np.empty((N, K), dtype=np.int64)
    val = np.empty((N, K), dtype=np.float64)
    rows = max(1, (1 << 24) // V)
    for s in range(0, N, rows):
        z = H[s:s + rows] @ W.T
        # stable sort of -z: equal logits keep increasing column order
        order = np.argsort(-z, axis=1, kind="stable")[:, :K]
        idx[s:s + rows] = order
        val[s:s + rows] = np.take_along_axis(z, order, axis=1)
    return idx, val
