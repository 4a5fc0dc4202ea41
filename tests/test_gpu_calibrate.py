"""ds_calibrate against the oracle's calibration (importance and channel choice).

The importance is a float, the channel choice an integer decided from it, so:
  * the GPU's fp32 importance matches the oracle's fp64 value to a relative
    1e-4 (fp32 column sums over at most 512 rows per chunk, then over the
    chunks and the batch, in a fixed order);
  * the GPU's choice is exactly the oracle's rule (largest first, ties to the
    lower channel, ascending) applied to the GPU's own fp32 importance;
  * every chosen channel's exact importance is within the fp32 tolerance of
    the oracle's r-th largest (near-ties may resolve either way).
On the generator's data the choice also equals the seeded outlier channels.
"""
import numpy as np
import pytest
import torch

import dsgen
import oracle
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds

CASES = [
    # name, B, Hq, Hkv, T, T_cap, Nq, r, n_out
    ("tiny", 1, 4, 4, 1000, 1024, 8, 8, 8),
    ("gqa-ragged", 2, 8, 2, 1537, 1600, 5, 16, 16),
    ("one-token", 1, 2, 1, 1, 3, 1, 4, 4),
    ("r-all", 1, 2, 2, 700, 700, 3, 128, 8),
    ("many-chunks", 1, 4, 2, 20000, 20001, 16, 8, 8),
    ("nq-over-chunk", 1, 2, 2, 100, 128, 600, 16, 16),
]


def _check(w, Qc, K, T, r, C, I):
    C_ref, I_ref = oracle.calibrate(Qc, K, T, w.Hq, r)
    Ig = I.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(Ig - I_ref) <= 1e-4 * np.abs(I_ref) + 1e-30)
    Cg = C.cpu().numpy()
    assert np.array_equal(Cg, oracle.calibrate_select(I.cpu().numpy(), r))
    for h in range(w.Hq):
        kth = np.sort(I_ref[h])[::-1][r - 1]
        assert np.all(I_ref[h][Cg[h]] >= kth * (1 - 2e-4))
    return Cg, C_ref


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_calibrate_matches_oracle(case):
    name, B, Hq, Hkv, T, T_cap, Nq, r, n_out = case
    w = dsgen.Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T_cap, r=min(r, 16), k=1, n_out=n_out,
                       seed=0xCA1 + T)
    _, K, _ = dsgen.qkv(w, want=("K",))
    Qc = dsgen.q_calib(w, Nq)
    C = torch.full((Hq, r), -1, dtype=torch.int32, device="cuda")
    I = torch.empty((Hq, 128), dtype=torch.float32, device="cuda")
    ds.calibrate(gu.dev_bf16(Qc), gu.dev_bf16(K), C, T, importance=I)
    torch.cuda.synchronize()
    Cg, C_ref = _check(w, Qc, K, T, r, C, I)
    if r == n_out and T >= 100 and Nq >= 5:
        for h in range(Hq):
            assert np.array_equal(Cg[h], dsgen.outliers(w, h))
    assert ds.device_status() == 0


def test_calibrate_ties_and_without_importance():
    # every value equal: channels 0..r-1 for every head
    B, Hq, Hkv, T, Nq, r = 1, 3, 1, 50, 2, 5
    Qc = torch.ones((B, Hq, Nq, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.full((B, Hkv, T, 128), -2.0, dtype=torch.bfloat16, device="cuda")
    C = torch.empty((Hq, r), dtype=torch.int32, device="cuda")
    ds.calibrate(Qc, K, C, T)
    assert torch.equal(C.cpu(), torch.arange(r, dtype=torch.int32).repeat(Hq, 1))


@pytest.mark.parametrize("name", ["llama2-7b-B8-H32-T4K", "long-B1-H32-T256K"])
def test_calibrate_full_workload(name):
    w = dsgen.workload(name)
    _, K, _ = dsgen.qkv(w, want=("K",))
    Qc = dsgen.q_calib(w, 16)
    C = torch.empty((w.Hq, w.n_out), dtype=torch.int32, device="cuda")
    I = torch.empty((w.Hq, 128), dtype=torch.float32, device="cuda")
    ds.calibrate(gu.dev_bf16(Qc), gu.dev_bf16(K), C, w.T, importance=I)
    torch.cuda.synchronize()
    Cg = C.cpu().numpy()
    Ig = I.cpu().numpy()
    assert np.array_equal(Cg, oracle.calibrate_select(Ig, w.n_out))
    # exact importance of a sample of heads (the oracle on those heads' slabs)
    for h in (0, w.Hq // 2, w.Hq - 1):
        g = h // w.G
        Ks = K[:, g:g + 1]
        Qs = Qc[:, h:h + 1]
        _, Ih = oracle.calibrate(Qs, Ks, w.T, 1, w.n_out)
        assert np.all(np.abs(Ig[h] - Ih[0]) <= 1e-4 * Ih[0])
        assert np.array_equal(Cg[h], dsgen.outliers(w, h))
