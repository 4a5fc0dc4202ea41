"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

import dsgen


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (numpy uint16) -> CUDA bfloat16 tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """CUDA bfloat16 tensor -> numpy uint16 bit patterns."""
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


class Inputs:
    """One workload's inputs on the host (bits) and on the device."""

    def __init__(self, w: dsgen.Workload, r: int | None = None, with_v: bool = True):
        self.w = w
        self.r = w.r if r is None else r
        want = ("Q", "K", "V") if with_v else ("Q", "K")
        self.Q, self.K, self.V = dsgen.qkv(w, want=want)
        self.C = dsgen.channels(w, self.r)
        self.dQ = dev_bf16(self.Q)
        self.dK = dev_bf16(self.K)
        self.dV = dev_bf16(self.V) if with_v else None
        self.dC = dev_i32(self.C)

    def free(self):
        for n in ("dQ", "dK", "dV", "dC"):
            setattr(self, n, None)
        torch.cuda.empty_cache()


def sample_heads(B: int, Hq: int, n: int, seed: int = 0):
    """n distinct (b, h) pairs, always including the first and last head."""
    rng = np.random.default_rng(seed)
    total = B * Hq
    pick = {0, total - 1}
    while len(pick) < min(n, total):
        pick.add(int(rng.integers(0, total)))
    return [(p // Hq, p % Hq) for p in sorted(pick)]


def score_error_bound(qc: np.ndarray, lab: np.ndarray) -> np.ndarray:
    """Bound on |fp32 sequential sum - exact sum| of sum_j qc[j]*lab[t,j].

    Every product of two bf16 values is exact in fp32; recursive summation of
    r terms errs by at most (r-1)*u/(1-(r-1)*u) * sum|terms|, u = 2^-24.
    """
    r = qc.shape[-1]
    u = 2.0 ** -24
    gamma = (r - 1) * u / (1 - (r - 1) * u) if r > 1 else 0.0
    return gamma * (np.abs(lab) @ np.abs(qc)) + 1e-30
