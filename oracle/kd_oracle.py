"""fp64 CPU oracle of the fused chunked top-K KL distillation loss.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
module: it is used by ``tests/``, by ``__graft_entry__.smoke()`` (to check
one small GPU call) and by the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py``.  It shares no code with the CUDA library; the two only
consume the same seeded inputs from ``workloads``.

What it computes
----------------
"Efficient Knowledge Distillation for LLMs: Offline Top-K Logits and a
Fused Chunked KL Loss" trains a student against an offline cache of the
teacher's top-K logits per position (blog post, "Two systems changes",
paragraph on offline distillation) with a KL loss (blog post, the online
baseline paragraph, which links torch's ``KLDivLoss``).  The three loss
implementations it compares (dense, forward-chunked, fused chunked; listed
in the Japanese summary's method paragraph) are stated to compute the same
mathematical quantity (blog post, "Two systems changes": "mathematically
equivalent"), so the oracle computes that quantity directly, without
chunking.  The concrete reading, for student hidden states ``H[N,d]``,
LM-head weight ``W[V,d]``, teacher cache ``(idx[N,K], logit[N,K])``, mask
``m[N]`` and temperature ``T``:

For each token n:
  1. ``z[v] = sum_j H[n,j] W[v,j]`` for every v in ``[0, V)``, in fp64 from
     the exact bf16 values.
  2. ``lse_n = M + log sum_v exp(z[v] - M)``, ``M = max_v z[v]``.
  3. Teacher: ``t_k = logit[n,k] / T``; ``lseT = logsumexp_k t_k``;
     ``logp_k = t_k - lseT``; ``p_k = exp(logp_k)``; ``0 log 0 = 0``.
  4. ``term_n = sum_k p_k (logp_k - (z[idx_k] - lse_n))``, the forward KL of
     the teacher's renormalised top-K distribution from the student's
     full-vocabulary softmax (teacher zero outside its top-K).
  5. ``L = sum_n m_n term_n / sum_n m_n`` (``L = 0`` when ``sum m = 0``).

Backward, for an upstream scalar gradient ``g``:
  6. ``c_n = g m_n / sum m``.
  7. ``dZ[n,v] = c_n (exp(z[v] - lse_n) - sum_{k: idx_k = v} p_k)``.  Because
     ``sum_k p_k = 1`` the derivative of ``term_n`` with respect to ``z`` is
     the student softmax minus the scattered teacher distribution; the blog
     post's closing paragraph mentions a closed-form gradient without
     printing it, and this is that derivative.
  8. ``dH[n,:] = sum_v dZ[n,v] W[v,:]``.
  9. ``dW[v,:] = sum_n dZ[n,v] H[n,:]``.

Readings where the pages are silent: T divides the teacher logits only (no
T^2 factor); duplicate teacher indices add their probabilities at that
column; an index outside ``[0, V)`` is an error; masked tokens still get an
lse; a teacher logit of ``-inf`` gives ``p = 0`` and contributes nothing.

Variants (not on the pages; options of the library, defaults off):
  * An index of ``-1`` marks an empty teacher slot (a cache with fewer than
    K entries for some tokens).  Empty slots take no part in step 3's
    softmax, so ``p`` is renormalised over the filled slots.  A token with no
    filled slot has an empty teacher distribution: ``P_n = sum_k p_k = 0``,
    ``term_n = 0`` and, since ``d term_n / dz = P_n softmax(z) - scatter(p)``,
    a zero dZ row.  Its mask still counts in ``sum m``.
  * ``student_T``: the usual distillation temperature, applied to the
    student too: steps 2 and 4 use ``z / T`` in place of ``z`` (``lse`` is
    then ``logsumexp(z / T)``) and ``term_n`` is multiplied by ``T^2``, so
    step 7 becomes ``dZ = c_n T (softmax(z / T) - scatter(p))``.
  * A bf16 teacher cache needs nothing here: the oracle takes the logits'
    values, whatever type held them.

Tokens are processed in row blocks only to bound memory; every quantity
above is per token except the sums over n in steps 5 and 9, which are
accumulated block by block in fp64.  Matrix products use numpy's fp64
``@`` (a library primitive).
"""

from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

__all__ = [
    "as_f64",
    "teacher_distribution",
    "student_lse",
    "kd_topk_kl",
    "forward",
    "backward",
    "lse_rows",
    "term_rows",
    "dH_rows",
    "dW_rows",
]

_BLOCK_ELEMS = 1 << 24   # fp64 elements of one [rows, V] logit block


def as_f64(x) -> np.ndarray:
    """Exact fp64 copy of a numpy array or a CPU torch tensor (bf16 included)."""
    if hasattr(x, "detach"):                     # torch tensor, bf16 has no numpy dtype
        x = x.detach().cpu()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _as_i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.int64)


def _rows_per_block(V: int) -> int:
    return max(1, _BLOCK_ELEMS // max(1, V))


def teacher_distribution(logit: np.ndarray, T: float, filled: Optional[np.ndarray] = None):
    """Step 3: ``p`` and ``log p`` of the temperature softmax over each row's K
    cached teacher logits.  Rows of ``logit`` are tokens.  ``filled`` (bool,
    same shape) marks the slots that hold an entry; the others get ``p = 0``
    and take no part in the normalisation.  A row without a finite filled
    logit gets ``p = 0`` throughout."""
    t = as_f64(logit) / float(T)
    if filled is not None:
        t = np.where(filled, t, -np.inf)
    tmax = np.max(t, axis=1, keepdims=True) if t.shape[1] else np.full((t.shape[0], 1), -np.inf)
    empty = ~np.isfinite(tmax[:, 0])
    tmax = np.where(np.isfinite(tmax), tmax, 0.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        lse_t = tmax + np.log(np.sum(np.exp(t - tmax), axis=1, keepdims=True))
        logp = t - lse_t
    logp[empty] = -np.inf
    p = np.exp(logp)
    return p, logp


def student_lse(z: np.ndarray) -> np.ndarray:
    """Step 2: log-sum-exp of each row of the student logits ``z``."""
    zmax = np.max(z, axis=1, keepdims=True)
    return (zmax + np.log(np.sum(np.exp(z - zmax), axis=1, keepdims=True)))[:, 0]


EMPTY_SLOT = -1   # teacher index of an empty cache slot


def _check_idx(idx: np.ndarray, V: int) -> None:
    if idx.size and (idx.min() < EMPTY_SLOT or idx.max() >= V or np.any((idx < 0) & (idx != EMPTY_SLOT))):
        raise ValueError("teacher index outside [0, V)")


def _slots(idx: np.ndarray):
    """Filled-slot mask, and indices with empty slots pointed at column 0
    (their p is 0, so they add nothing there)."""
    filled = idx != EMPTY_SLOT
    return filled, np.where(filled, idx, 0)


def _token_terms(z: np.ndarray, lse: np.ndarray, idx: np.ndarray,
                 p: np.ndarray, logp: np.ndarray) -> np.ndarray:
    """Step 4 for a block of tokens: sum_k p_k (logp_k - (z[idx_k] - lse))."""
    z_at = np.take_along_axis(z, idx, axis=1)
    inner = logp - (z_at - lse[:, None])
    with np.errstate(invalid="ignore"):          # p = 0 with logp = -inf: 0 log 0 = 0
        return np.sum(np.where(p > 0.0, p * inner, 0.0), axis=1)


def _dz_block(z: np.ndarray, lse: np.ndarray, idx: np.ndarray, p: np.ndarray,
              c: np.ndarray) -> np.ndarray:
    """Step 7 for a block of tokens: ``c_n (P_n softmax(z) - scatter(p))`` with
    ``P_n = sum_k p_k`` (1, or 0 for a token without teacher entries)."""
    q = np.exp(z - lse[:, None]) * np.sum(p, axis=1, keepdims=True)
    scat = np.zeros_like(q)
    rows = np.repeat(np.arange(z.shape[0]), idx.shape[1])
    np.add.at(scat, (rows, idx.reshape(-1)), p.reshape(-1))
    return c[:, None] * (q - scat)


def kd_topk_kl(H, W, topk_idx, topk_logit, mask=None, T: float = 1.0,
               grad: float = 1.0, backward: bool = True, student_T: bool = False) -> Dict[str, object]:
    """Steps 1-9 for all tokens.  Returns ``loss`` (float), ``lse`` [N],
    ``term`` [N], ``sum_mask`` and, if ``backward``, ``dH`` [N,d] and
    ``dW`` [V,d]; all fp64.  ``student_T`` selects the variant with the
    student at temperature T and the T^2 factor."""
    Hf = as_f64(H)
    Wf = as_f64(W)
    idx = _as_i64(topk_idx)
    N, d = Hf.shape
    V = Wf.shape[0]
    _check_idx(idx, V)
    filled, idx = _slots(idx)
    m = np.ones(N) if mask is None else as_f64(mask)
    p, logp = teacher_distribution(topk_logit, T, filled)
    sum_mask = float(np.sum(m))
    c = (grad * m / sum_mask) if sum_mask != 0.0 else np.zeros(N)
    zs = 1.0 / float(T) if student_T else 1.0            # student logits used: z * zs
    tfac = float(T) ** 2 if student_T else 1.0           # factor on term_n

    lse = np.empty(N)
    term = np.empty(N)
    dH = np.zeros((N, d)) if backward else None
    dW = np.zeros((V, d)) if backward else None
    B = _rows_per_block(V)
    for s in range(0, N, B):
        e = min(N, s + B)
        z = (Hf[s:e] @ Wf.T) * zs                            # step 1
        lse[s:e] = student_lse(z)                            # step 2
        term[s:e] = tfac * _token_terms(z, lse[s:e], idx[s:e], p[s:e], logp[s:e])  # step 4
        if backward:
            dz = _dz_block(z, lse[s:e], idx[s:e], p[s:e], c[s:e] * (tfac * zs))  # step 7
            dH[s:e] = dz @ Wf                                # step 8
            dW += dz.T @ Hf[s:e]                             # step 9
    loss = float(np.sum(m * term) / sum_mask) if sum_mask != 0.0 else 0.0   # step 5
    out = {"loss": loss, "lse": lse, "term": term, "sum_mask": sum_mask}
    if backward:
        out["dH"] = dH
        out["dW"] = dW
    return out


def forward(H, W, topk_idx, topk_logit, mask=None, T: float = 1.0, student_T: bool = False):
    """Steps 1-5: ``(loss, lse)``."""
    r = kd_topk_kl(H, W, topk_idx, topk_logit, mask, T, backward=False, student_T=student_T)
    return r["loss"], r["lse"]


def backward(H, W, topk_idx, topk_logit, mask=None, T: float = 1.0, grad: float = 1.0,
             student_T: bool = False):
    """Steps 6-9: ``(dH, dW)``."""
    r = kd_topk_kl(H, W, topk_idx, topk_logit, mask, T, grad=grad, student_T=student_T)
    return r["dH"], r["dW"]


# ---- per-row evaluation for spot checks at sizes where the full oracle is too slow

def lse_rows(H, W, rows: Sequence[int]) -> np.ndarray:
    """Steps 1-2 for the tokens ``rows`` only."""
    rows = np.asarray(rows, dtype=np.int64)
    Hf = as_f64(H[rows]) if hasattr(H, "detach") else as_f64(H)[rows]
    Wf = as_f64(W)
    return student_lse(Hf @ Wf.T)


def term_rows(H, W, topk_idx, topk_logit, rows: Sequence[int], T: float = 1.0):
    """Steps 1-4 for the tokens ``rows`` only: ``(lse, term)``."""
    rows = np.asarray(rows, dtype=np.int64)
    Hf = as_f64(H[rows]) if hasattr(H, "detach") else as_f64(H)[rows]
    Wf = as_f64(W)
    idx = _as_i64(topk_idx)[rows]
    _check_idx(idx, Wf.shape[0])
    filled, idx = _slots(idx)
    p, logp = teacher_distribution(as_f64(topk_logit)[rows], T, filled)
    z = Hf @ Wf.T
    lse = student_lse(z)
    return lse, _token_terms(z, lse, idx, p, logp)


def dH_rows(H, W, topk_idx, topk_logit, mask, rows: Sequence[int], T: float = 1.0,
            grad: float = 1.0) -> np.ndarray:
    """Steps 1-3 and 6-8 for the tokens ``rows`` only (``sum m`` over all N)."""
    rows = np.asarray(rows, dtype=np.int64)
    Hf = as_f64(H[rows]) if hasattr(H, "detach") else as_f64(H)[rows]
    Wf = as_f64(W)
    idx = _as_i64(topk_idx)[rows]
    _check_idx(idx, Wf.shape[0])
    m_all = np.ones(as_f64(topk_logit).shape[0]) if mask is None else as_f64(mask)
    sum_mask = float(np.sum(m_all))
    c = grad * m_all[rows] / sum_mask if sum_mask != 0.0 else np.zeros(len(rows))
    filled, idx = _slots(idx)
    p, _ = teacher_distribution(as_f64(topk_logit)[rows], T, filled)
    z = Hf @ Wf.T
    lse = student_lse(z)
    return _dz_block(z, lse, idx, p, c) @ Wf


def dW_rows(H, W, topk_idx, topk_logit, mask, lse: np.ndarray, vrows: Sequence[int],
            T: float = 1.0, grad: float = 1.0) -> np.ndarray:
    """Steps 6-7 and 9 for the vocabulary rows ``vrows`` only.  Needs every
    token's ``lse``, which the caller takes from this oracle."""
    vrows = np.asarray(vrows, dtype=np.int64)
    Hf = as_f64(H)
    Wv = as_f64(W[vrows]) if hasattr(W, "detach") else as_f64(W)[vrows]
    V = W.shape[0]
    idx = _as_i64(topk_idx)
    _check_idx(idx, V)
    N = Hf.shape[0]
    m = np.ones(N) if mask is None else as_f64(mask)
    sum_mask = float(np.sum(m))
    c = grad * m / sum_mask if sum_mask != 0.0 else np.zeros(N)
    filled, idx = _slots(idx)
    p, _ = teacher_distribution(topk_logit, T, filled)
    psum = np.sum(p, axis=1)
    lse = np.asarray(lse, dtype=np.float64)
    out = np.zeros((len(vrows), Hf.shape[1]))
    B = _rows_per_block(len(vrows))
    for s in range(0, N, B):
        e = min(N, s + B)
        z = Hf[s:e] @ Wv.T                                   # z[n, vrows]
        q = np.exp(z - lse[s:e, None]) * psum[s:e, None]
        scat = np.zeros_like(q)
        for j, v in enumerate(vrows):
            scat[:, j] = np.sum(np.where(idx[s:e] == v, p[s:e], 0.0), axis=1)
        dz = c[s:e, None] * (q - scat)
        out += dz.T @ Hf[s:e]
    return out
