"""The five synthetic workloads.

Shapes follow the pages' workloads: the GPT-OSS vocabulary of 201,088 tokens
and 32,768-token context (blog post, "Why distillation recovery is
expensive" and the GPT-OSS 20B result in "Scaling to long context
lengths"), the Llama-3-sized 128,256 vocabulary of the 8K-context
3.2B-student table (Japanese summary, results table), the top-100 teacher
cache (blog post, "Two systems changes") and the 4K to 256K-token
output-head-only sweep (abstract).  The pages give no hidden sizes or value
distributions for the toy head; the ones below are stated choices.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class Config:
    name: str
    N: int                 # tokens
    d: int                 # hidden size
    V: int                 # vocabulary size
    K: int                 # teacher top-K
    T: float               # teacher temperature
    chunk: int             # tokens whose dZ is live at once in backward
    w_std: float           # W ~ N(0, w_std^2); H ~ N(0, 1)
    teacher: str           # "uniform" or "overlap30"
    mask: str              # "ones", "packed10" or "drop5"
    seed: int
    sweep: Tuple[int, ...] = field(default_factory=tuple)

    def with_N(self, N: int) -> "Config":
        return replace(self, N=int(N))


CONFIGS = (
    # 0: small parity case
    Config("small_parity_N512_d256_V4096_K16", 512, 256, 4096, 16, 1.0, 128,
           w_std=256 ** -0.5, teacher="uniform", mask="ones", seed=0),
    # 1: small student head, 4 packed sequences of 1024 tokens
    Config("packed_head_N4096_d2048_V32000_K100", 4096, 2048, 32000, 100, 1.0, 1024,
           w_std=2048 ** -0.5, teacher="overlap30", mask="packed10", seed=1),
    # 2: 3.2B-Llama-shaped student head at 8K context
    Config("llama_head_N8192_d3072_V128256_K100", 8192, 3072, 128256, 100, 1.0, 2048,
           w_std=0.02, teacher="uniform", mask="ones", seed=2),
    # 3: GPT-OSS-20B-shaped head at 32K context
    Config("gptoss_head_N32768_d2880_V201088_K100", 32768, 2880, 201088, 100, 1.0, 4096,
           w_std=0.02, teacher="uniform", mask="drop5", seed=3),
    # 4: long-context output-head-only sweep (N set per point of the sweep)
    Config("sweep_head_d2048_V128256_K100", 4096, 2048, 128256, 100, 1.0, 4096,
           w_std=0.02, teacher="uniform", mask="ones", seed=4,
           sweep=(4096, 16384, 32768, 65536, 131072, 262144)),
)


def get_config(i: int, N: Optional[int] = None) -> Config:
    cfg = CONFIGS[i]
    return cfg.with_N(N) if N is not None else cfg
