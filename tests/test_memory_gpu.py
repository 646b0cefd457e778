"""Peak device memory of forward + backward is linear in the number of tokens.

The pages' point of the fused chunked loss is that peak memory grows only
linearly with sequence length (abstract; blog post, long-context section).
For the long-context sweep's shape (d = 2048, V = 128256, K = 100, chunk
4096) the peak of the torch allocator over inputs, outputs and workspace is
measured at N = 4K ... 256K tokens, fitted by least squares, and compared
with the analytic per-token bytes:
  H and dH (2 x 2d), teacher cache (8K), mask and lse (8), prepared teacher
  (8 Kp + 4), forward partials (16 splits x 12), the kept-token list for
  skipping masked rows (4) and per-block sums.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

D, V, K, CHUNK = 2048, 128256, 100, 4096
SWEEP = (4096, 16384, 32768, 65536, 131072, 262144)


@pytest.fixture(scope="module")
def kd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from chunked_top_kl_b200 import build
    build.build()
    import chunked_top_kl_b200 as k
    return k


def _peak_bytes(kd, N, W, gen):
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    # drawn in their final dtypes so that no temporary inflates the peak
    H = torch.randn(N, D, device="cuda", generator=gen, dtype=torch.bfloat16)
    idx = torch.randint(0, V, (N, K), device="cuda", generator=gen, dtype=torch.int32)
    lg = torch.randn(N, K, device="cuda", generator=gen)
    mask = torch.ones(N, device="cuda")
    ws = kd.alloc_workspace(N, D, V, K, CHUNK, "cuda")
    loss, lse = kd.forward(H, W, idx, lg, mask, 1.0, CHUNK, workspace=ws)
    dH, dW = kd.backward(H, W, idx, lg, mask, 1.0, CHUNK, lse, workspace=ws)
    st, _ = kd.check(ws)
    assert st == 0
    peak = torch.cuda.max_memory_allocated() - base
    del H, idx, lg, mask, ws, loss, lse, dH, dW
    return peak


def test_peak_memory_linear_in_tokens(kd):
    gen = torch.Generator(device="cuda").manual_seed(4)
    W = torch.randn(V, D, device="cuda", generator=gen, dtype=torch.bfloat16) * 0.02
    peaks = np.array([_peak_bytes(kd, N, W, gen) for N in SWEEP], dtype=np.float64)
    Ns = np.array(SWEEP, dtype=np.float64)
    slope, icpt = np.polyfit(Ns, peaks, 1)
    resid = np.abs(peaks - (slope * Ns + icpt)) / peaks
    Kp = ((K + 1 + 3) // 4) * 4
    per_token = 2 * 2 * D + 8 * K + 8 + 8 * Kp + 4 + 16 * 12 + 4
    print("peaks GiB", peaks / 2**30, "slope B/token", slope, "analytic", per_token)
    assert resid.max() < 0.03, resid
    assert abs(slope - per_token) <= 0.10 * per_token, (slope, per_token)
