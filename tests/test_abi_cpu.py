"""The C ABI on a machine without a GPU: symbols, host-side validation, sizes.

Nothing here launches a kernel: every call below is rejected by the host-side
argument checks before the library touches the CUDA runtime.
"""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import post_token_sparse_b200 as ds

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ds.h")
FAKE = 0x7000_0000_0000  # aligned, never dereferenced: the calls fail validation first


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ds_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for want in ("ds_label_append", "ds_score", "ds_topk", "ds_score_topk", "ds_sparse_decode",
                 "ds_decode", "ds_workspace_size", "ds_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ds.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", ds.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (ds_\w+)", out))
    assert set(declared_functions()) <= exported


def test_status_strings():
    lib = ds.lib()
    assert lib.ds_status_string(0) == b"DS_OK"
    assert lib.ds_status_string(1) == b"DS_ERR_INVALID_ARG"
    assert lib.ds_status_string(2) == b"DS_ERR_UNSUPPORTED"
    assert lib.ds_status_string(3) == b"DS_ERR_WORKSPACE"
    assert lib.ds_status_string(4) == b"DS_ERR_CUDA"


def _dims(**kw):
    base = dict(B=2, Hq=8, Hkv=2, d=128, T_cap=1000, r=16)
    base.update(kw)
    return ds.Dims(base["B"], base["Hq"], base["Hkv"], base["d"], base["T_cap"], base["r"])


P = ctypes.c_void_p(FAKE)
NUL = None


@pytest.mark.parametrize("dims,want", [
    (dict(B=0), ds.DS_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), ds.DS_ERR_INVALID_ARG),
    (dict(r=0), ds.DS_ERR_INVALID_ARG),
    (dict(r=129), ds.DS_ERR_INVALID_ARG),
    (dict(d=64, r=8), ds.DS_ERR_UNSUPPORTED),
    (dict(B=70000), ds.DS_ERR_UNSUPPORTED),
])
def test_bad_dims(dims, want):
    lib = ds.lib()
    d = _dims(**dims)
    assert lib.ds_label_append(P, P, P, d, 0, 1, NUL) == want
    assert lib.ds_score(P, P, P, P, d, 10, NUL) == want
    assert lib.ds_score_topk(P, P, P, NUL, P, d, 10, 5, NUL, 0, NUL) == want
    assert lib.ds_sparse_decode(P, P, P, P, P, NUL, d, 10, 5, 1.0, NUL, 0, NUL) == want
    assert lib.ds_decode(P, P, P, P, NUL, d, 10, 1.0, NUL, 0, NUL) == want


def test_bad_sizes_and_pointers():
    lib = ds.lib()
    d = _dims()
    bad = ds.DS_ERR_INVALID_ARG
    mis = ctypes.c_void_p(FAKE + 4)
    # label append range
    assert lib.ds_label_append(P, P, P, d, -1, 1, NUL) == bad
    assert lib.ds_label_append(P, P, P, d, 0, 0, NUL) == bad
    assert lib.ds_label_append(P, P, P, d, 990, 11, NUL) == bad
    assert lib.ds_label_append(NUL, P, P, d, 0, 1, NUL) == bad
    assert lib.ds_label_append(mis, P, P, d, 0, 1, NUL) == bad
    # score: T out of range, null/misaligned
    assert lib.ds_score(P, P, P, P, d, 0, NUL) == bad
    assert lib.ds_score(P, P, P, P, d, 1001, NUL) == bad
    assert lib.ds_score(P, P, P, mis, d, 10, NUL) == bad
    # top-k: k out of range
    assert lib.ds_topk(P, P, 4, 10, 0, NUL, 0, NUL) == bad
    assert lib.ds_topk(P, P, 4, 10, 11, NUL, 0, NUL) == bad
    assert lib.ds_topk(P, P, 0, 10, 1, NUL, 0, NUL) == bad
    assert lib.ds_topk(NUL, P, 4, 10, 1, NUL, 0, NUL) == bad
    assert lib.ds_topk(P, mis, 4, 10, 1, NUL, 0, NUL) == bad
    assert lib.ds_topk(P, P, 4, 16 * 65536 + 1, 1, NUL, 0, NUL) == ds.DS_ERR_UNSUPPORTED
    assert lib.ds_topk(P, P, 70000, 10, 1, NUL, 0, NUL) == ds.DS_ERR_UNSUPPORTED
    # fused score+topk: r not a multiple of 8 needs a score buffer
    assert lib.ds_score_topk(P, P, P, NUL, P, _dims(r=5), 10, 20, NUL, 0, NUL) == bad
    assert lib.ds_score_topk(P, P, P, NUL, P, _dims(r=5), 10, 5, NUL, 0, NUL) == \
        ds.DS_ERR_UNSUPPORTED
    # sparse decode: k > T, T > T_cap, misaligned lse
    assert lib.ds_sparse_decode(P, P, P, P, P, NUL, d, 10, 11, 1.0, NUL, 0, NUL) == bad
    assert lib.ds_sparse_decode(P, P, P, P, P, NUL, d, 1001, 5, 1.0, NUL, 0, NUL) == bad
    assert lib.ds_sparse_decode(P, P, P, P, P, mis, d, 10, 5, 1.0, NUL, 0, NUL) == bad
    assert lib.ds_decode(P, P, P, P, NUL, d, 0, 1.0, NUL, 0, NUL) == bad


def test_workspace_checked_before_launch():
    lib = ds.lib()
    d = _dims(B=1, Hq=4, Hkv=4, T_cap=100000)
    need = lib.ds_workspace_size(ds.OP_DECODE, d, 100000, 100000)
    assert need > 0  # few heads, long rows: the rows are split
    assert lib.ds_decode(P, P, P, P, NUL, d, 100000, 1.0, NUL, 0, NUL) == ds.DS_ERR_WORKSPACE
    assert lib.ds_decode(P, P, P, P, NUL, d, 100000, 1.0, P, need - 1, NUL) == \
        ds.DS_ERR_WORKSPACE
    need_s = lib.ds_workspace_size(ds.OP_SPARSE_DECODE, d, 100000, 20000)
    assert need_s > 0
    assert lib.ds_sparse_decode(P, P, P, P, P, NUL, d, 100000, 20000, 1.0, NUL, 0, NUL) == \
        ds.DS_ERR_WORKSPACE


def test_workspace_sizes():
    lib = ds.lib()
    # short rows: every warp takes whole heads, nothing to merge, no workspace
    d = _dims(B=32, Hq=32, Hkv=32, T_cap=32768, r=8)
    assert lib.ds_workspace_size(ds.OP_SPARSE_DECODE, d, 32768, 16) == 0
    # the one-launch selections keep 2-byte key prefixes of every token (T_pad a
    # power of two times 256) after 256 KiB of counters
    assert lib.ds_workspace_size(ds.OP_TOPK, d, 16384, 512) == 256 * 1024 + 32 * 32 * 16384 * 2
    assert lib.ds_workspace_size(ds.OP_TOPK, d, 4096, 512) == 0
    assert lib.ds_workspace_size(ds.OP_TOPK, d, 16385, 512) == 0
    assert lib.ds_workspace_size(ds.OP_SCORE_TOPK, d, 32768, 512) == \
        256 * 1024 + 32 * 32 * 32768 * 2
    assert lib.ds_workspace_size(ds.OP_SCORE_TOPK, d, 4096, 512) == 0  # one CTA per head
    assert lib.ds_workspace_size(ds.OP_SCORE_TOPK, d, 5000, 512) == \
        256 * 1024 + 32 * 32 * 8192 * 2
    # heads shared by warps: 256 KiB of counters, then 132 floats per slot
    n = lib.ds_workspace_size(ds.OP_SPARSE_DECODE, d, 32768, 2048)
    assert n > 256 * 1024 and n % 256 == 0
    assert (n - 256 * 1024) // (132 * 4) >= 1024
    # long single sequence
    d = _dims(B=1, Hq=32, Hkv=32, T_cap=262144, r=8)
    n = lib.ds_workspace_size(ds.OP_SPARSE_DECODE, d, 262144, 16384)
    assert n > 256 * 1024 and n % 256 == 0
    # invalid sizes give 0
    assert lib.ds_workspace_size(ds.OP_SPARSE_DECODE, d, 0, 1) == 0
    assert lib.ds_workspace_size(ds.OP_SPARSE_DECODE, d, 100, 101) == 0
    assert lib.ds_workspace_size(ds.OP_DECODE, _dims(d=64), 100, 100) == 0
    # depends only on the arguments
    assert lib.ds_workspace_size(ds.OP_DECODE, d, 262144, 1) == \
        lib.ds_workspace_size(ds.OP_DECODE, d, 262144, 1)


def test_decode_step_fuses_only_one_wave_of_heads():
    lib = ds.lib()
    # one launch (no workspace) while B*Hq <= 2 x 148; the separate kernels beyond
    assert lib.ds_workspace_size(ds.OP_DECODE_STEP, _dims(B=8, Hq=32, Hkv=32, T_cap=4096), 4096,
                                 256) == 0
    assert lib.ds_workspace_size(ds.OP_DECODE_STEP, _dims(B=9, Hq=32, Hkv=32, T_cap=4096), 4096,
                                 256) == 0
    assert lib.ds_workspace_size(ds.OP_DECODE_STEP, _dims(B=10, Hq=32, Hkv=32, T_cap=4096),
                                 4096, 256) > 0
    assert lib.ds_workspace_size(ds.OP_DECODE_STEP, _dims(B=32, Hq=32, Hkv=32, T_cap=32768, r=8),
                                 32768, 2048) > 0


def test_group_calls_validation():
    lib = ds.lib()
    bad = ds.DS_ERR_INVALID_ARG
    d = _dims(B=2, Hq=8, Hkv=2, T_cap=1000, r=16)
    mis = ctypes.c_void_p(FAKE + 4)
    assert lib.ds_group_score_topk(P, P, P, NUL, P, d, 100, 10, NUL) == bad  # scores required
    assert lib.ds_group_score_topk(P, P, P, P, P, d, 100, 101, NUL) == bad
    assert lib.ds_group_score_topk(P, P, P, P, P, d, 1001, 10, NUL) == bad
    assert lib.ds_group_score_topk(P, P, P, mis, P, d, 100, 10, NUL) == bad
    assert lib.ds_group_score_topk(P, P, P, P, P, _dims(Hq=6, Hkv=4), 100, 10, NUL) == bad
    assert lib.ds_group_score_topk(P, P, P, P, P, _dims(r=12), 100, 10, NUL) == \
        ds.DS_ERR_UNSUPPORTED
    assert lib.ds_group_sparse_decode(P, P, P, P, P, NUL, d, 100, 101, 1.0, NUL, 0, NUL) == bad
    assert lib.ds_group_sparse_decode(P, P, P, NUL, P, NUL, d, 100, 10, 1.0, NUL, 0, NUL) == bad
    # G = 4: the group-by-group plan over the 8 groups' shared rows
    dl = _dims(B=1, Hq=32, Hkv=8, T_cap=262144, r=8)
    slots = _group_plan(8, 16384)
    assert slots > 0
    need = lib.ds_workspace_size(ds.OP_GROUP_SPARSE_DECODE, dl, 262144, 16384)
    assert need == (256 * 1024 + slots * 8 * 132 * 4 + 255) // 256 * 256
    assert lib.ds_group_sparse_decode(P, P, P, P, P, NUL, dl, 262144, 16384, 1.0, P, need - 1,
                                      NUL) == ds.DS_ERR_WORKSPACE


def test_group_decode_step_workspace():
    """The attention's workspace, then (4096 < T <= 16384) the one-launch top-k's
    over the group scores, 256-byte aligned."""
    lib = ds.lib()
    d = _dims(B=16, Hq=64, Hkv=8, T_cap=16384, r=16)
    att = lib.ds_workspace_size(ds.OP_GROUP_SPARSE_DECODE, d, 16384, 1024)
    want = (att + 255) // 256 * 256 + 256 * 1024 + 128 * 16384 * 2
    assert lib.ds_workspace_size(ds.OP_GROUP_DECODE_STEP, d, 16384, 1024) == want
    assert lib.ds_workspace_size(ds.OP_GROUP_DECODE_STEP, d, 4096, 256) == \
        lib.ds_workspace_size(ds.OP_GROUP_SPARSE_DECODE, d, 4096, 256)


def test_group_decode_step_validation():
    lib = ds.lib()
    bad = ds.DS_ERR_INVALID_ARG
    d = _dims(B=2, Hq=8, Hkv=2, T_cap=1000, r=16)
    args = lambda **kw: [kw.get(n, P) for n in ("Q", "K", "V", "C", "label", "sg", "idx", "O")]
    assert lib.ds_group_decode_step(*args(sg=NUL), NUL, d, 100, 10, 1.0, 1, NUL, 0, NUL) == bad
    assert lib.ds_group_decode_step(*args(K=NUL), NUL, d, 100, 10, 1.0, 1, NUL, 0, NUL) == bad
    assert lib.ds_group_decode_step(*args(), NUL, d, 100, 101, 1.0, 1, NUL, 0, NUL) == bad
    assert lib.ds_group_decode_step(*args(), NUL, d, 1001, 10, 1.0, 1, NUL, 0, NUL) == bad
    assert lib.ds_group_decode_step(*args(), NUL, _dims(r=12), 100, 10, 1.0, 1, NUL, 0,
                                    NUL) == ds.DS_ERR_UNSUPPORTED
    dl = _dims(B=1, Hq=32, Hkv=8, T_cap=262144, r=8)
    need = lib.ds_workspace_size(ds.OP_GROUP_DECODE_STEP, dl, 262144, 16384)
    assert need > 0
    assert lib.ds_group_decode_step(*args(), NUL, dl, 262144, 16384, 1.0, 1, P, need - 1,
                                    NUL) == ds.DS_ERR_WORKSPACE


def test_block_calls_validation():
    lib = ds.lib()
    bad = ds.DS_ERR_INVALID_ARG
    d = _dims(B=2, Hq=8, Hkv=2, T_cap=1000, r=16)
    for bs in (0, 3, 128, -64):
        assert lib.ds_block_score_topk(P, P, P, P, P, d, 1000, bs, 1, NUL) == bad
        assert lib.ds_block_sparse_decode(P, P, P, P, P, NUL, d, 1000, bs, 1, 1.0, NUL, 0,
                                          NUL) == bad
    assert lib.ds_block_score_topk(P, P, P, P, P, d, 1000, 64, 17, NUL) == bad  # 16 blocks
    assert lib.ds_block_score_topk(P, P, P, P, P, d, 1000, 64, 0, NUL) == bad
    assert lib.ds_block_score_topk(P, P, P, NUL, P, d, 1000, 64, 4, NUL) == bad
    assert lib.ds_block_score_topk(P, P, P, P, P, d, 1001, 64, 4, NUL) == bad
    assert lib.ds_block_score_topk(P, P, P, P, P, _dims(r=12), 1000, 64, 4, NUL) == \
        ds.DS_ERR_UNSUPPORTED
    assert lib.ds_block_sparse_decode(P, P, P, P, P, NUL, d, 1000, 64, 17, 1.0, NUL, 0, NUL) == bad
    dl = _dims(B=1, Hq=4, Hkv=4, T_cap=262144, r=8)
    need = lib.ds_workspace_size(ds.OP_BLOCK_SPARSE_DECODE, dl, 262144, 256 * 64)
    assert need == lib.ds_workspace_size(ds.OP_SPARSE_DECODE, dl, 262144, 256 * 64) > 0
    assert lib.ds_block_sparse_decode(P, P, P, P, P, NUL, dl, 262144, 64, 256, 1.0, P, need - 1,
                                      NUL) == ds.DS_ERR_WORKSPACE


def test_kv_append_validation():
    lib = ds.lib()
    bad = ds.DS_ERR_INVALID_ARG
    d = _dims(B=2, Hq=8, Hkv=2, T_cap=1000, r=16)
    mis = ctypes.c_void_p(FAKE + 4)
    assert lib.ds_kv_append(P, P, P, P, d, -1, NUL) == bad
    assert lib.ds_kv_append(P, P, P, P, d, 1000, NUL) == bad
    assert lib.ds_kv_append(NUL, P, P, P, d, 0, NUL) == bad
    assert lib.ds_kv_append(P, P, mis, P, d, 0, NUL) == bad
    assert lib.ds_kv_append(P, P, P, P, _dims(d=64, r=8), 0, NUL) == ds.DS_ERR_UNSUPPORTED


def test_decode_step_kv_validation():
    lib = ds.lib()
    bad = ds.DS_ERR_INVALID_ARG
    d = _dims(B=2, Hq=8, Hkv=2, T_cap=1000, r=16)
    mis = ctypes.c_void_p(FAKE + 4)
    #                            Q  Kn   Vn   K  V  C  lab idx O  lse  dims T  k
    assert lib.ds_decode_step_kv(P, NUL, P, P, P, P, P, P, P, NUL, d, 10, 5, 1.0, NUL, 0,
                                 NUL) == bad
    assert lib.ds_decode_step_kv(P, P, NUL, P, P, P, P, P, P, NUL, d, 10, 5, 1.0, NUL, 0,
                                 NUL) == bad
    assert lib.ds_decode_step_kv(P, mis, P, P, P, P, P, P, P, NUL, d, 10, 5, 1.0, NUL, 0,
                                 NUL) == bad
    assert lib.ds_decode_step_kv(P, P, mis, P, P, P, P, P, P, NUL, d, 10, 5, 1.0, NUL, 0,
                                 NUL) == bad
    assert lib.ds_decode_step_kv(P, P, P, P, P, P, P, P, P, NUL, d, 0, 1, 1.0, NUL, 0,
                                 NUL) == bad
    assert lib.ds_decode_step_kv(P, P, P, P, P, P, P, P, P, NUL, d, 1001, 5, 1.0, NUL, 0,
                                 NUL) == bad
    assert lib.ds_decode_step_kv(P, P, P, P, P, P, P, P, P, NUL, d, 10, 11, 1.0, NUL, 0,
                                 NUL) == bad
    assert lib.ds_decode_step_kv(P, P, P, NUL, P, P, P, P, P, NUL, d, 10, 5, 1.0, NUL, 0,
                                 NUL) == bad


def test_hier_validation():
    lib = ds.lib()
    bad = ds.DS_ERR_INVALID_ARG
    d = _dims(B=2, Hq=8, Hkv=2, T_cap=5000, r=16)
    assert lib.ds_hier_score_topk(P, P, P, P, d, 5000, 2049, NUL) == ds.DS_ERR_UNSUPPORTED
    assert lib.ds_hier_score_topk(P, P, P, P, d, 100, 101, NUL) == bad
    assert lib.ds_hier_score_topk(P, P, P, P, d, 5001, 10, NUL) == bad
    assert lib.ds_hier_score_topk(P, P, P, P, d, 100, 0, NUL) == bad
    assert lib.ds_hier_score_topk(P, P, NUL, P, d, 100, 10, NUL) == bad
    assert lib.ds_hier_score_topk(P, P, P, P, _dims(r=12), 100, 10, NUL) == ds.DS_ERR_UNSUPPORTED


def test_calibrate_validation_and_workspace():
    lib = ds.lib()
    d = _dims(B=2, Hq=8, Hkv=2, T_cap=5000, r=16)
    bad = ds.DS_ERR_INVALID_ARG
    mis = ctypes.c_void_p(FAKE + 4)
    need = lib.ds_workspace_size(ds.OP_CALIBRATE, d, 5000, 16)
    # key chunk sums [B*Hkv][ceil(T/512)][128] + query sums [B*Hq][1][128], fp32, 256-rounded
    assert need == ((2 * 2 * 10 + 2 * 8 * 1) * 128 * 4 + 255) // 256 * 256
    assert lib.ds_workspace_size(ds.OP_CALIBRATE, d, 5000, 0) == 0
    assert lib.ds_calibrate(P, 16, P, d, 5000, P, NUL, P, need - 1, NUL) == ds.DS_ERR_WORKSPACE
    assert lib.ds_calibrate(P, 16, P, d, 5000, P, NUL, NUL, 0, NUL) == ds.DS_ERR_WORKSPACE
    assert lib.ds_calibrate(P, 0, P, d, 5000, P, NUL, P, need, NUL) == bad
    assert lib.ds_calibrate(P, 16, P, d, 0, P, NUL, P, need, NUL) == bad
    assert lib.ds_calibrate(P, 16, P, d, 5001, P, NUL, P, need, NUL) == bad
    assert lib.ds_calibrate(NUL, 16, P, d, 5000, P, NUL, P, need, NUL) == bad
    assert lib.ds_calibrate(P, 16, P, d, 5000, mis, NUL, P, need, NUL) == bad
    assert lib.ds_calibrate(P, 16, P, d, 5000, P, mis, P, need, NUL) == bad
    assert lib.ds_calibrate(P, 16, P, _dims(r=129), 500, P, NUL, P, need, NUL) == bad
    assert lib.ds_calibrate(P, 16, P, _dims(d=64, r=8), 500, P, NUL, P, need, NUL) == \
        ds.DS_ERR_UNSUPPORTED


def test_launch_counter_starts_untouched():
    assert ds.kernel_launches() >= 0


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A copy of the package with no libds.so must refuse to import."""
    pkg = tmp_path / "post_token_sparse_b200"
    pkg.mkdir()
    src = open(os.path.join(os.path.dirname(ds.__file__), "__init__.py")).read()
    (pkg / "__init__.py").write_text(src)
    res = subprocess.run([sys.executable, "-c", "import post_token_sparse_b200"],
                         cwd=tmp_path, capture_output=True, text=True)
    assert res.returncode != 0
    assert "libds.so is missing" in res.stderr


def _plan(heads, rows):
    """The documented work plan: a grid of 148 CTAs of 16 warps; the R = heads *
    rows rows are cut into ranges of `per` rows, per = ceil(R / (148 * 16)) but
    at least 16, rounded up to a multiple of 4.  When per >= rows every range is
    a whole number of heads and no workspace is needed; otherwise CTA c and head
    h share partial slot c + h."""
    R = heads * rows
    per = max(-(-R // (148 * 16)), 16)
    per = (per + 3) & ~3
    if per >= rows:
        return 0
    units = -(-R // per)
    return -(-units // 16) + heads


def _group_plan(groups, rows):
    """The documented plan of the group-by-group attention: 148 CTAs of 8 warps;
    per = ceil(R / (148 * 8)) but at least 16, rounded up to a multiple of 16.
    When per >= rows every range is a whole number of groups (no workspace);
    otherwise CTA c and group h share slot c + h, 8 heads of 132 floats."""
    R = groups * rows
    per = max(-(-R // (148 * 8)), 16)
    per = (per + 15) // 16 * 16
    if per >= rows:
        return 0
    units = -(-R // per)
    return -(-units // 8) + groups


@pytest.mark.parametrize("B,Hq,Hkv,T,k", [(1, 32, 8, 131072, 8192), (16, 64, 8, 16384, 1024),
                                          (2, 8, 2, 1000, 37), (1, 16, 2, 300000, 300000),
                                          (64, 64, 8, 4096, 256), (3, 12, 4, 16, 16),
                                          (1, 8, 1, 5000, 5000)])
def test_group_work_plan_follows_the_documented_rule(B, Hq, Hkv, T, k):
    """Dense decode and group-shared sparse decode with 2..8 query heads per KV
    head take the group plan; 1 or more than 8 take the per-head plan."""
    lib = ds.lib()
    d = _dims(B=B, Hq=Hq, Hkv=Hkv, T_cap=T, r=8)
    for op, rows in ((ds.OP_GROUP_SPARSE_DECODE, k), (ds.OP_DECODE, T)):
        slots = _group_plan(B * Hkv, rows)
        want = 0 if slots == 0 else (256 * 1024 + slots * 8 * 132 * 4 + 255) // 256 * 256
        assert lib.ds_workspace_size(op, d, T, k if op == ds.OP_GROUP_SPARSE_DECODE else T) == \
            want, (op, slots)
    d16 = _dims(B=B, Hq=16 * Hkv, Hkv=Hkv, T_cap=T, r=8)
    slots = _plan(B * 16 * Hkv, T)
    want = 0 if slots == 0 else (256 * 1024 + slots * 132 * 4 + 255) // 256 * 256
    assert lib.ds_workspace_size(ds.OP_DECODE, d16, T, T) == want


@pytest.mark.parametrize("B,H,T,k", [(1, 32, 262144, 16384), (32, 32, 32768, 512),
                                     (32, 32, 32768, 2048), (8, 32, 4096, 256),
                                     (16, 64, 16384, 1024), (1, 4, 1000, 1000),
                                     (3, 7, 5000, 300), (1, 1, 300000, 4000),
                                     (32, 32, 32768, 12)])
def test_work_plan_follows_the_documented_rule(B, H, T, k):
    lib = ds.lib()
    d = _dims(B=B, Hq=H, Hkv=H, T_cap=T, r=8)
    for op, rows in ((ds.OP_SPARSE_DECODE, k), (ds.OP_DECODE, T)):
        slots = _plan(B * H, rows)
        want = 0 if slots == 0 else (256 * 1024 + slots * 132 * 4 + 255) // 256 * 256
        assert lib.ds_workspace_size(op, d, T, k if op == ds.OP_SPARSE_DECODE else T) == want, \
            (op, slots)


def test_binding_noalloc_limit_matches_the_header():
    """The binding's copy of DS_NOALLOC_SCRATCH_BYTES is the header's value."""
    import re
    hdr = open(os.path.join(ROOT, "include", "ds.h")).read()
    m = re.search(r"#define DS_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m, "DS_NOALLOC_SCRATCH_BYTES not found in include/ds.h"
    assert ds.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
