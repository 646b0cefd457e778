"""Writes the oracle's expected values for the full-size workloads.

Run on any CPU machine (no GPU); calls only ``oracle`` and the seeded input
generator.  For each workload it stores, in ``tests/golden/fullsize_<name>.npz``:
the fp64 oracle's loss, the lse of every token (of 4096 sampled tokens
above 32768 tokens), dH for 32+ sampled tokens and dW for 32+ sampled
vocabulary rows (exact given the oracle's own lse for all tokens), stored as
fp32 (ample for the tolerances), the sample indices, and a SHA-256
of the generated input bytes so that a change in the generator is detected.

    python tests/golden/make_fullsize_expected.py [workload-index[:N]] ...
"""

from __future__ import annotations

import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

N_SAMPLE = 32          # sampled dH tokens and dW vocabulary rows
LSE_KEEP = 32768       # lse is stored for every token up to this N, else for a sample


def _bf16_bytes(t):
    import torch
    return t.view(torch.int16).numpy().tobytes()


def input_hash_bytes(x) -> str:
    import torch
    h = hashlib.sha256()
    for k in ("H", "W", "topk_idx", "topk_logit", "mask"):
        t = x[k].contiguous()
        h.update(_bf16_bytes(t) if t.dtype == torch.bfloat16 else t.numpy().tobytes())
    return h.hexdigest()


def sample_rows(n: int, count: int, seed: int, must=()) -> np.ndarray:
    rng = np.random.default_rng(seed)
    pick = set(int(i) for i in must if 0 <= i < n)
    pick.update(int(i) for i in rng.choice(n, size=min(n, count), replace=False))
    return np.array(sorted(pick), dtype=np.int64)


def make(index: int, N: int | None = None) -> str:
    cfg = workloads.get_config(index, N)
    t0 = time.time()
    x = workloads.make_inputs(cfg)
    digest = input_hash_bytes(x)
    fwd = oracle.kd_topk_kl(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"], cfg.T,
                            backward=False)
    mask = x["mask"].numpy()
    masked = np.nonzero(mask == 0)[0]
    rows = sample_rows(cfg.N, N_SAMPLE, 100 + index, must=[0, cfg.N - 1] + list(masked[:2]))
    teach = x["topk_idx"][0].numpy()
    vrows = sample_rows(cfg.V, N_SAMPLE, 200 + index, must=[0, cfg.V - 1] + list(teach[:4]))
    dH = oracle.dH_rows(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"], rows, cfg.T)
    dW = oracle.dW_rows(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"], fwd["lse"], vrows, cfg.T)
    name = cfg.name if N is None else f"{cfg.name}_N{cfg.N}"
    out = os.path.join(HERE, f"fullsize_{name}.npz")
    lse_rows = (np.arange(cfg.N, dtype=np.int64) if cfg.N <= LSE_KEEP
                else sample_rows(cfg.N, 4096, 300 + index, must=[0, cfg.N - 1]))
    np.savez_compressed(out, loss=np.float64(fwd["loss"]), lse=fwd["lse"][lse_rows].astype(np.float32),
                        lse_rows=lse_rows, rows=rows, dH_rows=dH.astype(np.float32), vrows=vrows,
                        dW_rows=dW.astype(np.float32),
                        sum_mask=np.float64(fwd["sum_mask"]), input_sha256=np.array(digest),
                        workload=np.array(cfg.name), N=np.int64(cfg.N))
    print(f"{name}: loss {fwd['loss']:.9f}  ({time.time() - t0:.0f} s) -> {out}", flush=True)
    return out


if __name__ == "__main__":
    for arg in sys.argv[1:] or ["2", "3", "4:4096", "4:262144"]:
        i, _, n = arg.partition(":")
        make(int(i), int(n) if n else None)
