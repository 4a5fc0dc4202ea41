"""GPU parity against the C++ oracle (oracle/ds_oracle.cpp, steps O1-O5), with the
acceptance checks of the path on the tiny and the Llama-2-7B-shaped workloads:

  label       bit-exact
  top-k       ds_topk given the oracle's fp32 scores returns the oracle's set
  selection   every index the decode step keeps is distinct, in range, ascending,
              and scores (exactly) within 1e-3 * (|s_k| + 1) of the oracle's k-th
  sparse O    max abs error <= 1e-2 against the oracle on the GPU's own set
  dense O     max abs error <= 5e-3
  lse         within 1e-3 * (1 + |lse|)
"""
import numpy as np
import pytest
import torch

import dsgen
import oracle.cxx as cxx
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import post_token_sparse_b200 as ds


@pytest.mark.parametrize("name", ["tiny-B1-H4-T1K", "llama2-7b-B8-H32-T4K"])
def test_workload_against_cxx_oracle(name):
    w = dsgen.workload(name)
    inp = gu.Inputs(w)
    BH = w.B * w.Hq
    ds.device_status(clear=True)
    label = torch.empty((w.B, w.Hq, w.T, w.r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, w.T)
    ref = cxx.sparse_step(inp.Q, inp.K, inp.V, inp.C, w.k, w.scale)
    assert np.array_equal(gu.host_bits(label), ref["label"])
    # ds_topk on the oracle's fp32 scores: the oracle's index set, bit for bit
    d_s = gu.dev_f32(ref["s32"].reshape(BH, w.T))
    idx_t = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    ds.topk(d_s, idx_t)
    assert np.array_equal(idx_t.cpu().numpy().reshape(w.B, w.Hq, w.k), ref["idx"])
    # the decode step and dense decode on the GPU
    idx = torch.empty((BH, w.k), dtype=torch.int32, device="cuda")
    O = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    ds.decode_step(inp.dQ, inp.dK, inp.dV, inp.dC, label, idx, O, w.T, w.scale, append=False,
                   lse=lse)
    Od = torch.empty_like(O)
    Ld = torch.empty_like(lse)
    ds.decode(inp.dQ, inp.dK, inp.dV, Od, w.T, w.scale, lse=Ld)
    torch.cuda.synchronize()
    I = idx.cpu().numpy().reshape(w.B, w.Hq, w.k)
    s64 = ref["s64"]
    for b in range(w.B):
        for h in range(w.Hq):
            sel = I[b, h]
            assert sel[0] >= 0 and sel[-1] < w.T and np.all(np.diff(sel) > 0), (b, h)
            s_k = np.sort(s64[b, h])[::-1][w.k - 1]
            assert np.all(s64[b, h][sel] >= s_k - 1e-3 * (abs(s_k) + 1)), (b, h)
    O_ref, L_ref = cxx.attend(inp.Q, inp.K, inp.V, I, w.scale)
    assert np.abs(O.cpu().numpy() - O_ref).max() <= 1e-2
    assert np.all(np.abs(lse.cpu().numpy() - L_ref) <= 1e-3 * (1 + np.abs(L_ref)))
    D_ref, DL_ref = cxx.dense(inp.Q, inp.K, inp.V, w.scale)
    assert np.abs(Od.cpu().numpy() - D_ref).max() <= 5e-3
    assert np.all(np.abs(Ld.cpu().numpy() - DL_ref) <= 1e-3 * (1 + np.abs(DL_ref)))
    assert ds.device_status() == 0
    inp.free()
