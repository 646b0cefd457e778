"""Writes the oracle's expected values for the full-size workloads.

Run on any CPU machine (no GPU); calls only ``oracle`` and the seeded input
generator.  For each workload it stores, in ``tests/golden/fullsize_<name>.npz``,
the fp64 oracle's loss and sum of the mask, the lse of every token (stored as
fp32, ample for the 2e-3 tolerance and for recomputing dZ from it), and a
SHA-256 of the generated input bytes so that a change in the generator is
detected.  The full forward pass (every token's lse) is the expensive part:
the test derives dH of sampled tokens and dW of sampled vocabulary rows from
the oracle at run time (``oracle.dH_rows``, and ``oracle.dW_rows`` with this
stored lse), so the samples can be large without storing them.

    python tests/golden/make_fullsize_expected.py [workload-index[:N]] ...

Default: the Llama-shaped 8K head, the GPT-OSS-shaped 32K head and every
point of the long-context sweep.
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
from workloads.configs import CONFIGS  # noqa: E402


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


def make(index: int, N: int | None = None) -> str:
    cfg = workloads.get_config(index, N)
    t0 = time.time()
    x = workloads.make_inputs(cfg)
    digest = input_hash_bytes(x)
    fwd = oracle.kd_topk_kl(x["H"], x["W"], x["topk_idx"], x["topk_logit"], x["mask"], cfg.T,
                            backward=False)
    name = cfg.name if N is None else f"{cfg.name}_N{cfg.N}"
    out = os.path.join(HERE, f"fullsize_{name}.npz")
    np.savez_compressed(out, loss=np.float64(fwd["loss"]), lse=fwd["lse"].astype(np.float32),
                        sum_mask=np.float64(fwd["sum_mask"]), input_sha256=np.array(digest),
                        workload=np.array(cfg.name), N=np.int64(cfg.N))
    print(f"{name}: loss {fwd['loss']:.9f}  ({time.time() - t0:.0f} s) -> {out}", flush=True)
    return out


if __name__ == "__main__":
    default = ["2", "3"] + [f"4:{n}" for n in CONFIGS[4].sweep]
    for arg in sys.argv[1:] or default:
        i, _, n = arg.partition(":")
        make(int(i), int(n) if n else None)
