"""KV offload: K and V in page-locked host memory, read by the kernels over the
host link (only the kept rows in the sparse calls).

The kernels are the same, so every result must be bit-identical to the run
with K and V in device memory; the sparse output is also checked against the
oracle on the GPU's own index set.
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


def _pinned(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory()


@pytest.mark.parametrize("shape", [(2, 8, 2, 3000, 16, 100), (1, 4, 4, 20000, 8, 1250)],
                         ids=["gqa-T3000", "mha-T20000"])
def test_offloaded_kv_matches_device_kv(shape):
    B, Hq, Hkv, T, r, k = shape
    w = dsgen.Workload("offload", B=B, Hq=Hq, Hkv=Hkv, T=T, r=r, k=k, n_out=min(16, r),
                       seed=0x0FF + T)
    inp = gu.Inputs(w)
    hK, hV = _pinned(inp.K), _pinned(inp.V)
    BH = B * Hq

    def run(K, V):
        label = torch.zeros((B, Hq, T, r), dtype=torch.bfloat16, device="cuda")
        ds.label_append(K, inp.dC, label, 0, T - 1)
        ds.label_append(K, inp.dC, label, T - 1, 1)
        idx = torch.empty((BH, k), dtype=torch.int32, device="cuda")
        ds.score_topk(inp.dQ, inp.dC, label, idx, T)
        O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
        ds.sparse_decode(inp.dQ, K, V, idx, O, T, w.scale)
        Od = torch.empty_like(O)
        ds.decode(inp.dQ, K, V, Od, T, w.scale)
        label2 = label.clone()
        idx2 = torch.empty_like(idx)
        O2 = torch.empty_like(O)
        ds.decode_step(inp.dQ, K, V, inp.dC, label2, idx2, O2, T, w.scale, append=True)
        torch.cuda.synchronize()
        return label, idx, O, Od, idx2, O2

    dev = run(inp.dK, inp.dV)
    host = run(hK, hV)
    for a, b in zip(dev, host):
        assert torch.equal(a, b)
    I = host[1].cpu().numpy().reshape(B, Hq, k)
    ref_O, _ = oracle.attend(inp.Q, inp.K, inp.V, I, w.scale)
    assert np.abs(host[2].cpu().numpy() - ref_O).max() <= 1e-2
    assert ds.device_status() == 0
    inp.free()


def test_kv_append_from_device_and_pinned_host():
    B, Hkv, T_cap, d = 2, 3, 50, 128
    K = torch.randn(B, Hkv, T_cap, d, device="cuda").to(torch.bfloat16)
    V = torch.randn(B, Hkv, T_cap, d, device="cuda").to(torch.bfloat16)
    K0, V0 = K.clone(), V.clone()
    kn = torch.randn(B, Hkv, d).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, d).to(torch.bfloat16)
    ds.kv_append(kn.cuda(), vn.cuda(), K, V, 7)             # device source
    ds.kv_append(kn.pin_memory(), vn.pin_memory(), K, V, 49)  # pinned host source
    torch.cuda.synchronize()
    for t in (7, 49):
        assert torch.equal(K[:, :, t].cpu(), kn) and torch.equal(V[:, :, t].cpu(), vn)
    keep = [t for t in range(T_cap) if t not in (7, 49)]
    assert torch.equal(K[:, :, keep], K0[:, :, keep]) and torch.equal(V[:, :, keep], V0[:, :, keep])


@pytest.mark.parametrize("shape", [(8, 32, 32, 4096, 16, 256), (1, 4, 2, 40000, 8, 10000)],
                         ids=["one-launch", "separate-kernels"])
def test_decode_step_with_query_and_output_in_host_memory(shape):
    B, Hq, Hkv, T, r, k = shape
    w = dsgen.Workload("host-io", B=B, Hq=Hq, Hkv=Hkv, T=T, r=r, k=k, n_out=min(16, r),
                       seed=0x10 + T)
    inp = gu.Inputs(w)
    label = torch.empty((B, Hq, T, r), dtype=torch.bfloat16, device="cuda")
    ds.label_append(inp.dK, inp.dC, label, 0, T - 1)
    BH = B * Hq

    def run(Q, O, lse):
        lab = label.clone()
        idx = torch.empty((BH, k), dtype=torch.int32, device="cuda")
        ds.decode_step(Q, inp.dK, inp.dV, inp.dC, lab, idx, O, T, w.scale, append=True, lse=lse)
        torch.cuda.synchronize()
        return idx, O.cpu(), lse.cpu()

    dev = run(inp.dQ, torch.empty((B, Hq, w.d), device="cuda"), torch.empty((B, Hq), device="cuda"))
    host = run(inp.dQ.cpu().pin_memory(), torch.empty((B, Hq, w.d)).pin_memory(),
               torch.empty((B, Hq)).pin_memory())
    for a, b in zip(dev, host):
        assert torch.equal(a.cpu(), b.cpu())
    assert ds.device_status() == 0
    inp.free()


@pytest.mark.parametrize("shape", [(2, 16, 2, 9000, 16, 600), (1, 8, 2, 3000, 8, 100)],
                         ids=["g8-T9000", "g4-T3000"])
def test_group_decode_step_with_offloaded_kv(shape):
    """ds_group_decode_step with K and V in page-locked host memory (the label
    append reads the new token's channels and the attention the kept rows over
    the host link) gives the bits of the device-resident run."""
    B, Hq, Hkv, T, r, k = shape
    w = dsgen.Workload("offload-group", B=B, Hq=Hq, Hkv=Hkv, T=T, r=r, k=k, n_out=min(16, r),
                       seed=0x6F1 + T)
    inp = gu.Inputs(w)
    hK, hV = _pinned(inp.K), _pinned(inp.V)

    def run(K, V):
        label = torch.zeros((B, Hq, T, r), dtype=torch.bfloat16, device="cuda")
        ds.label_append(inp.dK, inp.dC, label, 0, T - 1)
        sg = torch.empty((B * Hkv, T), dtype=torch.float32, device="cuda")
        idx = torch.empty((B * Hkv, k), dtype=torch.int32, device="cuda")
        O = torch.empty((B, Hq, w.d), dtype=torch.float32, device="cuda")
        L = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        ds.group_decode_step(inp.dQ, K, V, inp.dC, label, sg, idx, O, T, w.scale, lse=L)
        torch.cuda.synchronize()
        return label, sg, idx, O, L

    dev = run(inp.dK, inp.dV)
    host = run(hK, hV)
    for a, b in zip(dev, host):
        assert torch.equal(a, b)
    I = host[2].cpu().numpy().reshape(B, Hkv, k)
    ref_O, _ = oracle.group_attend(inp.Q, inp.K, inp.V, I, w.scale)
    assert np.abs(host[3].cpu().numpy() - ref_O).max() <= 1e-2
    assert ds.device_status() == 0
    inp.free()
