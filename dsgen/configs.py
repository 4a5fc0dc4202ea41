"""The decode workloads, each named by what it is and its sizes.

Shapes follow the workloads the Double Sparsity page evaluates on
(Llama-2-7B, Llama-2-70B with grouped KV heads, 256K-token contexts) at its
headline 1/16 token and channel sparsity; the values are synthetic (see
``gen.c`` for the recipe).
"""
from __future__ import annotations

import dataclasses
import math


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    r: int
    k: int
    n_out: int
    n_hh: int = 0
    d: int = 128
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # Algorithmic HBM bytes of one sparse decode step: the label cache, the
    # selected K and V rows, and the query (bf16) and output (fp32).
    def sparse_step_bytes(self) -> int:
        heads = self.B * self.Hq
        return heads * (self.T * self.r * 2 + self.k * 2 * self.d * 2 + self.d * 2 + self.d * 4)

    # The sparse-attention call alone: selected K/V rows, their indices, Q and O.
    def sparse_decode_bytes(self) -> int:
        heads = self.B * self.Hq
        return heads * (self.k * 2 * self.d * 2 + self.k * 4 + self.d * 2 + self.d * 4)

    # Dense decode: every K/V row once per KV head, plus Q and O per query head.
    def dense_bytes(self) -> int:
        return (self.B * self.Hkv * self.T * 2 * self.d * 2
                + self.B * self.Hq * (self.d * 2 + self.d * 4))

    def label_bytes(self) -> int:
        return self.B * self.Hq * self.T * self.r * 2

    # Block-granular selection with kb blocks of bs tokens: every label row, the
    # block scores written and read back, the kept blocks' K/V rows, Q and O.
    def block_step_bytes(self, bs: int, kb: int) -> int:
        nblk = -(-self.T // bs)
        return (self.label_bytes() + self.B * self.Hq * (nblk * 4 * 2 + kb * 4
                + kb * bs * 2 * self.d * 2 + self.d * 2 + self.d * 4))

    # Group-shared selection: every label row, each kept K/V row once per KV
    # group, the group scores written and read back, Q and O per query head.
    def group_step_bytes(self) -> int:
        return (self.label_bytes() + self.B * self.Hkv * self.k * (2 * self.d * 2 + 4)
                + self.B * self.Hkv * self.T * 4 * 2 + self.B * self.Hq * (self.d * 2 + self.d * 4))


_BASE_SEED = 0xD5000000

CONFIGS: dict[str, Workload] = {
    # tiny MHA step, small enough for the oracle in well under a second
    "tiny-B1-H4-T1K": Workload("tiny-B1-H4-T1K", B=1, Hq=4, Hkv=4, T=1024, r=8, k=64,
                               n_out=8, seed=_BASE_SEED + 1),
    # Llama-2-7B-shaped MHA decode, 1/8 channels, 1/16 tokens
    "llama2-7b-B8-H32-T4K": Workload("llama2-7b-B8-H32-T4K", B=8, Hq=32, Hkv=32, T=4096,
                                     r=16, k=256, n_out=16, seed=_BASE_SEED + 2),
    # Llama-2-70B-style grouped-query decode, 64 query heads over 8 KV heads
    "gqa-B16-Hq64-Hkv8-T16K": Workload("gqa-B16-Hq64-Hkv8-T16K", B=16, Hq=64, Hkv=8,
                                       T=16384, r=16, k=1024, n_out=16,
                                       seed=_BASE_SEED + 3),
    # 256K-token single-sequence decode with 0.5% heavy-hitter tokens per head
    "long-B1-H32-T256K": Workload("long-B1-H32-T256K", B=1, Hq=32, Hkv=32, T=262144,
                                  r=8, k=16384, n_out=8, n_hh=round(0.005 * 262144),
                                  seed=_BASE_SEED + 4),
}

# Sparsity / batch sweep at T=32K: one input set, r x k grid, plus the dense
# path and the r=d, k=T invariant cell.
SWEEP_R = (8, 16, 32)
SWEEP_K = (512, 2048, 8192)
for _r in SWEEP_R:
    for _k in SWEEP_K:
        _n = f"sweep-B32-H32-T32K-r{_r}-k{_k}"
        CONFIGS[_n] = Workload(_n, B=32, Hq=32, Hkv=32, T=32768, r=_r, k=_k, n_out=16,
                               seed=_BASE_SEED + 5)

# The order the workloads are listed in (the second one is the headline).
ORDER = ["tiny-B1-H4-T1K", "llama2-7b-B8-H32-T4K", "gqa-B16-Hq64-Hkv8-T16K",
         "long-B1-H32-T256K"] + [f"sweep-B32-H32-T32K-r{r}-k{k}" for r in SWEEP_R
                                 for k in SWEEP_K]


def workload(name: str) -> Workload:
    return CONFIGS[name]
