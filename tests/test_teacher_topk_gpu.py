"""GPU parity of the teacher top-K cache writer (``kd_teacher_topk``) with the
fp64 oracle ``oracle.teacher_topk``.

* Integer-valued H and W (exact in bf16, and every logit an integer well
  inside fp32's exact range): the GPU logits equal the oracle's exactly, so
  indices and logits must match bit for bit, ties (many of them) included.
  With at least K tiles of 256 columns the selection reads only the tiles
  whose maximum reaches the K-th largest tile maximum, otherwise the whole
  row; the cases cover both, K equal to the number of tiles (every tile
  read) and one past it.
* Gaussian H and W at a few shapes (ragged N, V and chunk): the logits match
  within fp32 accumulation error, and the index sets match except where the
  oracle's K-th and (K+1)-th logits are closer than that error.
* The cache, fed to the loss with the teacher equal to the student and K = V,
  gives a zero loss.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from chunked_top_kl_b200 import build
    build.build()
    import chunked_top_kl_b200 as k
    return k


def _gpu_topk(kd, Ht, Wt, K, chunk):
    idx, val = kd.teacher_topk(Ht.cuda(), Wt.cuda(), K, chunk=chunk)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy()


@pytest.mark.parametrize("N,d,V,K,chunk", [(300, 64, 5000, 100, 128), (77, 16, 700, 7, 32), (40, 8, 300, 300, 64),
                                           (128, 64, 4096, 16, 64), (128, 64, 4096, 17, 64), (100, 32, 3001, 5, 64)],
                         ids=["N300_V5000_K100", "N77_V700_K7", "K_equals_V",
                              "K_equals_tiles", "K_one_past_tiles", "V3001_K5_tiles"])
def test_integer_logits_exact(kd, N, d, V, K, chunk):
    g = torch.Generator().manual_seed(N + V)
    Ht = torch.randint(-3, 4, (N, d), generator=g).to(torch.bfloat16)
    Wt = torch.randint(-3, 4, (V, d), generator=g).to(torch.bfloat16)
    idx, val = _gpu_topk(kd, Ht, Wt, K, chunk)
    ridx, rval = oracle.teacher_topk(Ht, Wt, K)
    assert np.array_equal(idx, ridx)
    assert np.array_equal(val.astype(np.float64), rval)


@pytest.mark.parametrize("N,d,V,K,chunk", [(513, 256, 4096, 16, 256), (300, 136, 10007, 100, 128),
                                           (1, 64, 24, 5, 16)],
                         ids=["N513_V4096_K16", "N300_V10007_K100", "N1_V24"])
def test_gaussian_logits(kd, N, d, V, K, chunk):
    g = torch.Generator().manual_seed(7 * N + V)
    Ht = torch.randn(N, d, generator=g).to(torch.bfloat16)
    Wt = (torch.randn(V, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    idx, val = _gpu_topk(kd, Ht, Wt, K, chunk)
    z = Ht.double().numpy() @ Wt.double().numpy().T
    ridx, rval = oracle.teacher_topk(Ht, Wt, K)
    # fp32 accumulation of d bf16 products: |error| <= d * 2^-23 * sum|h w| (a loose bound)
    tol = d * 2.0 ** -23 * (np.abs(Ht.double().numpy()) @ np.abs(Wt.double().numpy()).T).max() + 1e-6
    assert np.max(np.abs(val - np.take_along_axis(z, idx, axis=1))) <= tol      # values are the logits at idx
    assert np.all(np.diff(val, axis=1) <= 0)                                   # largest first
    assert np.max(np.abs(val - rval)) <= 2 * tol
    for n in range(N):
        got, want = set(idx[n].tolist()), set(ridx[n].tolist())
        if got != want:
            # only columns whose logit is within the error of the K-th may differ
            kth = rval[n, K - 1]
            for c in got ^ want:
                assert abs(z[n, c] - kth) <= 2 * tol, (n, c, z[n, c], kth)


def test_cache_feeds_the_loss(kd):
    g = torch.Generator().manual_seed(11)
    N, d, V = 64, 32, 96
    H = torch.randint(-2, 3, (N, d), generator=g).to(torch.bfloat16).cuda()
    W = torch.randint(-2, 3, (V, d), generator=g).to(torch.bfloat16).cuda()
    idx, val = kd.teacher_topk(H, W, V, chunk=32)
    loss, lse = kd.forward(H, W, idx, val, None, 1.0, 32)
    assert abs(loss.item()) < 1e-4


def test_workspace_and_arguments(kd):
    assert kd.kd_teacher_topk_workspace_size(1000, 64, 5000, 100, 256) > 0
    assert kd.kd_teacher_topk_workspace_size(1000, 64, 50, 100, 256) == 0       # K > V
    assert kd.kd_teacher_topk_workspace_size(1000, 60, 5000, 100, 256) == 0     # d % 8
    assert kd.kd_teacher_topk_workspace_size(1000, 64, 5000, 513, 256) == 0     # K > 512


@pytest.mark.parametrize("V,K,n_pos", [(5000, 10, 0), (3000, 512, 0), (3020, 100, 20)],
                         ids=["all_tied_K10", "all_tied_K512", "20_above_3000_tied"])
def test_tied_rows(kd, V, K, n_pos):
    """Rows where more values share the K-th value's 12-bit key bin than the
    select's shared-memory candidate buffer holds (2048): it then finishes as a
    radix select, with the same result (ties in increasing column order)."""
    g = torch.Generator().manual_seed(V + K)
    N, d = 37, 16
    Ht = torch.randint(1, 3, (N, d), generator=g).to(torch.bfloat16)       # positive
    Wt = torch.zeros(V, d, dtype=torch.bfloat16)
    if n_pos:
        # n_pos columns near the end with positive logits; every other logit is 0
        Wt[V - n_pos:] = torch.randint(1, 3, (n_pos, d), generator=g).to(torch.bfloat16)
    idx, val = _gpu_topk(kd, Ht, Wt, K, chunk=16)
    ridx, rval = oracle.teacher_topk(Ht, Wt, K)
    assert np.array_equal(idx, ridx)
    assert np.array_equal(val.astype(np.float64), rval)


def _ordered_head(N, V, descending):
    """A head whose logits are z[n, v] = v (or -v): H rows (4096, 64, 1, 0...)
    and W rows (v // 4096, v // 64 % 64, v % 64, 0...) are exact in bf16, and
    so are the integer logits in fp32."""
    d = 16
    Ht = torch.zeros(N, d)
    Ht[:, 0], Ht[:, 1], Ht[:, 2] = 4096.0, 64.0, 1.0
    if descending:
        Ht = -Ht
    v = torch.arange(V)
    Wt = torch.zeros(V, d)
    Wt[:, 0], Wt[:, 1], Wt[:, 2] = (v // 4096).float(), (v // 64 % 64).float(), (v % 64).float()
    return Ht.to(torch.bfloat16), Wt.to(torch.bfloat16)


@pytest.mark.parametrize("V,K,descending", [(70001, 100, False), (70001, 100, True), (40003, 512, False),
                                            (9, 3, False)],
                         ids=["ascending", "descending", "ascending_K512", "V9"])
def test_ordered_rows(kd, V, K, descending):
    """Rows in increasing column order make every block of the row the new
    top K (the streaming select raises its threshold on each); decreasing
    rows put it all in the first block."""
    Ht, Wt = _ordered_head(5, V, descending)
    idx, val = _gpu_topk(kd, Ht, Wt, K, chunk=4)
    ridx, rval = oracle.teacher_topk(Ht, Wt, K)
    assert np.array_equal(idx, ridx)
    assert np.array_equal(val.astype(np.float64), rval)


@pytest.mark.parametrize("N,d,V,K", [(40, 64, 70001, 100), (24, 32, 40000, 300)],
                         ids=["V70001_K100", "V40000_K300"])
def test_integer_logits_long_rows(kd, N, d, V, K):
    """Rows many times the select's block length, with ties (integer logits)."""
    g = torch.Generator().manual_seed(N * V + K)
    Ht = torch.randint(-3, 4, (N, d), generator=g).to(torch.bfloat16)
    Wt = torch.randint(-3, 4, (V, d), generator=g).to(torch.bfloat16)
    idx, val = _gpu_topk(kd, Ht, Wt, K, chunk=16)
    ridx, rval = oracle.teacher_topk(Ht, Wt, K)
    assert np.array_equal(idx, ridx)
    assert np.array_equal(val.astype(np.float64), rval)


def test_infinite_logits(kd):
    """+inf and -inf logits in a long row: +inf ranks above every finite
    logit (and first in the cache), -inf below them."""
    N, V, K = 4, 50001, 64
    Ht, Wt = _ordered_head(N, V, descending=False)          # z[n, v] = v, exactly
    W2 = Wt.clone().float()
    W2[7, 0] = float("inf")                                  # z = +inf
    W2[40000, 0] = float("-inf")                             # z = -inf
    W2 = W2.to(torch.bfloat16)
    idx, val = _gpu_topk(kd, Ht, W2, K, chunk=4)
    ridx, rval = oracle.teacher_topk(Ht, W2, K)
    assert np.isposinf(rval[:, 0]).all() and (ridx[:, 0] == 7).all()
    assert np.array_equal(idx, ridx)
    assert np.array_equal(val.astype(np.float64), rval)
