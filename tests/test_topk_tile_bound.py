"""The bound the teacher top-K select's tile route rests on, checked on the CPU
with numpy on random and adversarial rows (no GPU, no oracle code).

For a row of V logits cut into 256-column tiles, with at least K tiles: let
tau be the K-th largest of the tiles' maxima.  Then (1) at least K values of
the row are >= tau, so the row's K-th largest value is >= tau; (2) every value
that is >= the row's K-th largest (ties included) lies in a tile whose maximum
is >= tau.  Reading only those tiles and keeping the values >= tau therefore
keeps all of the row's top K, ties at the K-th value included.  Values are
compared through an order-preserving integer key with -0 mapped to +0, as the
kernel compares them.
"""

from __future__ import annotations

import numpy as np
import pytest

TILE = 256


def order_key(x: np.ndarray) -> np.ndarray:
    """Order-preserving uint32 key of float32 values (-0 taken as +0)."""
    x = np.where(x == 0, np.float32(0), x).astype(np.float32)
    u = x.view(np.uint32)
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def check_row(row: np.ndarray, K: int) -> None:
    V = row.size
    keys = order_key(row)
    ntiles = -(-V // TILE)
    assert ntiles >= K
    tile_max = np.array([keys[i * TILE:(i + 1) * TILE].max() for i in range(ntiles)], dtype=np.uint32)
    tau = np.sort(tile_max)[::-1][K - 1]
    kth = np.sort(keys)[::-1][K - 1]
    assert (keys >= tau).sum() >= K          # (1)
    assert kth >= tau
    selected = np.repeat(tile_max >= tau, TILE)[:V]
    assert np.all(selected[keys >= kth])     # (2): every value >= the K-th largest sits in a selected tile
    # the kept candidates hold the exact top K with its ties, and their K-th largest is the row's
    cand = keys[selected & (keys >= tau)]
    assert np.sort(cand)[::-1][K - 1] == kth
    assert (cand >= kth).sum() == (keys >= kth).sum()


@pytest.mark.parametrize("seed", range(6))
def test_gaussian_rows(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(256 * 100, 201088))
    check_row((rng.standard_normal(V) * 1.07).astype(np.float32), 100)


@pytest.mark.parametrize("K", [1, 5, 100, 274])
def test_tied_integer_rows(K):
    rng = np.random.default_rng(K)
    check_row(rng.integers(-3, 4, 70001).astype(np.float32), K)


@pytest.mark.parametrize("descending", [False, True])
def test_ordered_rows(descending):
    row = np.arange(70001, dtype=np.float32)
    check_row(row[::-1].copy() if descending else row, 100)


def test_infinities_and_signed_zeros():
    rng = np.random.default_rng(7)
    row = rng.standard_normal(30000).astype(np.float32)
    row[rng.choice(30000, 500, replace=False)] = -np.inf
    row[rng.choice(30000, 40, replace=False)] = np.inf
    row[rng.choice(30000, 300, replace=False)] = np.float32(-0.0)
    row[rng.choice(30000, 300, replace=False)] = np.float32(0.0)
    check_row(row, 100)
    check_row(np.full(5000, np.float32(-0.0)), 19)       # all equal (as keys): every tile kept


def test_exactly_K_tiles_and_a_ragged_tail():
    rng = np.random.default_rng(3)
    check_row(rng.standard_normal(16 * 256).astype(np.float32), 16)          # K = tiles: every tile kept
    check_row(rng.standard_normal(11 * 256 + 3).astype(np.float32), 12)      # last tile 3 columns wide
