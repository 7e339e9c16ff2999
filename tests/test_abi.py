"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and its host-side validation and sizing logic agree with the
oracle's definitions. No compute call reaches a kernel here (every call below
is rejected on the host before anything is enqueued)."""
import ctypes
import os
import re

import pytest

from block_sparse_causal_bsa_b200 import binding as bb
from oracle import bsa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "bsa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_]+)\s*\(", txt)))


def test_header_declares_expected_calls():
    assert set(_declared()) == set(bb.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = bb.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings():
    L = bb.lib()
    for st in range(4):
        assert L.bsa_status_string(st)


def _shape(**kw):
    base = dict(B=1, Hq=32, Hkv=8, N=131072, d=128, block_k=64, tile_q=128, dtype=bb.BSA_BF16)
    base.update(kw)
    return bb.Shape(*[base[f] for f, _ in bb.Shape._fields_])


@pytest.mark.parametrize("N,tq,bk,kf,kl,rho", [
    (131072, 128, 64, 64, 64, 2), (1024, 64, 64, 4, 4, 1), (65536, 128, 64, 128, 32, 1),
    (2048, 128, 64, 1, 1, 1), (4096, 64, 128, 8, 2, 3), (512, 128, 128, 100, 100, 1),
    (32768, 128, 64, 64, 64, 1)])
def test_kv_width_matches_oracle(N, tq, bk, kf, kl, rho):
    s = _shape(N=N, tile_q=tq, block_k=bk)
    p = bb.SelectParams(kf, kl, rho, 0.25, float("nan"))
    assert bb.bsa_kv_idx_width(s, p) == O.kv_idx_width(N, tq, bk, kf, kl, rho)


def test_workspace_sizes():
    s = _shape()
    n = bb.bsa_score_workspace_bytes(s, bb.BSA_SCORE_MEAN)
    nkb = 8 * 2048
    assert n >= nkb * 128 * (4 + 2) + nkb * 4          # fp32 pooled keys, fp16 copy, block scales
    n2 = bb.bsa_score_workspace_bytes(s, bb.BSA_SCORE_MEAN_VNORM)
    assert n2 >= n + nkb * 4
    p = bb.SelectParams(64, 64, 2, 0.25, float("nan"))
    sel = bb.bsa_select_workspace_bytes(s, p)
    assert sel >= 32 * 1024 * 128 * 4


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(block_k=32), dict(tile_q=256), dict(N=1000), dict(Hq=6, Hkv=4),
    dict(B=0), dict(dtype=7)])
def test_bad_shapes_rejected(bad):
    s = _shape(**bad)
    L = bb.lib()
    st = L.bsa_score(ctypes.byref(s), 0, 16, 16, None, 16, None, 256, 1 << 30, None)
    assert st in (bb.BSA_ERR_INVALID_ARG, bb.BSA_ERR_UNSUPPORTED)
    assert L.bsa_last_error()
    p = bb.SelectParams(8, 8, 1, 0.25, 0.0)
    assert bb.bsa_kv_idx_width(s, p) == -1
    assert bb.bsa_score_workspace_bytes(s, 0) == 0


def test_null_pointers_rejected():
    L = bb.lib()
    s = _shape()
    assert L.bsa_score(ctypes.byref(s), 0, None, 16, None, 16, None, 256, 1 << 30, None) == bb.BSA_ERR_INVALID_ARG
    # output-aware score without V
    assert L.bsa_score(ctypes.byref(s), 1, 16, 16, None, 16, None, 256, 1 << 30, None) == bb.BSA_ERR_INVALID_ARG
    # undersized workspace
    assert L.bsa_score(ctypes.byref(s), 0, 16, 16, None, 16, None, 256, 10, None) == bb.BSA_ERR_INVALID_ARG
    assert b"workspace" in L.bsa_last_error()
    # misaligned pointer
    assert L.bsa_score(ctypes.byref(s), 0, 18, 16, None, 16, None, 256, 1 << 30, None) == bb.BSA_ERR_INVALID_ARG
    assert L.bsa_attend(ctypes.byref(s), 16, 16, 16, 16, 16, 128, 0.1, 16, None, None, None) == bb.BSA_ERR_INVALID_ARG
    assert L.bsa_attend(ctypes.byref(s), 16, 16, 16, 16, 16, 0, 0.1, 16, None, 16, None) == bb.BSA_ERR_INVALID_ARG
    assert L.bsa_attend(ctypes.byref(s), 16, 16, 16, 16, 16, 128, -1.0, 16, None, 16, None) == bb.BSA_ERR_INVALID_ARG


@pytest.mark.parametrize("kf,kl,rho,q", [(4, 8, 1, 0.2), (0, 0, 1, 0.2), (8, 8, 0, 0.2), (8, 8, 2, 1.5)])
def test_bad_select_params_rejected(kf, kl, rho, q):
    L = bb.lib()
    s = _shape()
    p = bb.SelectParams(kf, kl, rho, q, 0.0)
    assert L.bsa_select(ctypes.byref(s), ctypes.byref(p), 16, 16, 16, None, None, None, None, None,
                        256, 1 << 34, None) == bb.BSA_ERR_INVALID_ARG


def test_select_size_limits():
    L = bb.lib()
    s = _shape(N=64 * 16384)      # more key blocks than the selection supports (8192)
    p = bb.SelectParams(8, 8, 1, 0.25, 0.0)
    assert L.bsa_select(ctypes.byref(s), ctypes.byref(p), 16, 16, 16, None, None, None, None, None,
                        256, 1 << 40, None) == bb.BSA_ERR_UNSUPPORTED


def test_decode_validation():
    L = bb.lib()
    dims = (ctypes.c_int * 2)(0, 1)
    ok_shape = bb.DecodeShape(2, 32, 8, 8192, 128, 128, bb.BSA_BF16)
    p = bb.DecodeParams(1e-3, 1e-4, 1, 1, 2, dims)
    # missing dev_status
    assert L.bsa_decode(ctypes.byref(ok_shape), ctypes.byref(p), 16, 16, 16, 0.1, 16, 16, None,
                        None, None) == bb.BSA_ERR_INVALID_ARG
    for bad in [dict(L=8000), dict(Hq=24), dict(block_kv=32), dict(dtype=bb.BSA_F32)]:
        f = dict(B=2, Hq=32, Hkv=8, L=8192, d=128, block_kv=128, dtype=bb.BSA_BF16)
        f.update(bad)
        sh = bb.DecodeShape(*[f[n] for n, _ in bb.DecodeShape._fields_])
        assert L.bsa_decode(ctypes.byref(sh), ctypes.byref(p), 16, 16, 16, 0.1, 16, 16, None, 16,
                            None) in (bb.BSA_ERR_INVALID_ARG, bb.BSA_ERR_UNSUPPORTED)
    bad_dims = (ctypes.c_int * 2)(0, 128)
    p2 = bb.DecodeParams(1e-3, 1e-4, 1, 1, 2, bad_dims)
    assert L.bsa_decode(ctypes.byref(ok_shape), ctypes.byref(p2), 16, 16, 16, 0.1, 16, 16, None, 16,
                        None) == bb.BSA_ERR_INVALID_ARG
    p3 = bb.DecodeParams(1e-3, 1e-4, 0, 1, 2, dims)
    assert L.bsa_decode(ctypes.byref(ok_shape), ctypes.byref(p3), 16, 16, 16, 0.1, 16, 16, None, 16,
                        None) == bb.BSA_ERR_INVALID_ARG


def test_score_kinds_validation():
    """The added score kinds: workspace sizes, and argument errors caught before any launch."""
    L = bb.lib()
    s = _shape()
    nkb = 8 * 2048
    n_mean = bb.bsa_score_workspace_bytes(s, bb.BSA_SCORE_MEAN)
    assert bb.bsa_score_workspace_bytes(s, bb.BSA_SCORE_MEAN_VLOG) >= n_mean + nkb * 4
    assert bb.bsa_score_workspace_bytes(s, bb.BSA_SCORE_KMINMAX) >= n_mean + nkb * 128 * (4 + 2)   # + kmax, rad
    assert bb.bsa_score_workspace_bytes(s, 7) == 0
    big = 1 << 34
    # the additive form needs beta: not through bsa_score, not with NULL params
    assert L.bsa_score(ctypes.byref(s), bb.BSA_SCORE_MEAN_VLOG, 16, 16, 16, 16, None, 256, big,
                       None) == bb.BSA_ERR_INVALID_ARG
    assert b"bsa_score_ex" in L.bsa_last_error()
    assert L.bsa_score_ex(ctypes.byref(s), bb.BSA_SCORE_MEAN_VLOG, None, 16, 16, 16, 16, None, 256,
                          big, None) == bb.BSA_ERR_INVALID_ARG
    for beta in (-1.0, float("nan"), float("inf")):
        p = bb.ScoreParams(beta)
        assert L.bsa_score_ex(ctypes.byref(s), bb.BSA_SCORE_MEAN_VLOG, ctypes.byref(p), 16, 16, 16,
                              16, None, 256, big, None) == bb.BSA_ERR_INVALID_ARG
    p = bb.ScoreParams(0.5)
    # V is required for the additive form, unknown kinds are rejected
    assert L.bsa_score_ex(ctypes.byref(s), bb.BSA_SCORE_MEAN_VLOG, ctypes.byref(p), 16, 16, None, 16,
                          None, 256, big, None) == bb.BSA_ERR_INVALID_ARG
    assert L.bsa_score_ex(ctypes.byref(s), 9, ctypes.byref(p), 16, 16, 16, 16, None, 256, big,
                          None) == bb.BSA_ERR_INVALID_ARG
    # undersized workspace for the bounds backbone
    assert L.bsa_score_ex(ctypes.byref(s), bb.BSA_SCORE_KMINMAX, None, 16, 16, None, 16, None, 256,
                          n_mean, None) == bb.BSA_ERR_INVALID_ARG
    assert b"workspace" in L.bsa_last_error()


def test_score_select_workspace_and_validation():
    """bsa_score_select: workspace = score + selection workspaces + the ranking kernel's row
    ring (fused shapes) or a scores array (the others); argument errors before any launch."""
    L = bb.lib()
    s = _shape()                                       # bf16, d 128, tiles of 128: fused
    p = bb.SelectParams(64, 64, 2, 0.25, float("nan"))
    n_sc = bb.bsa_score_workspace_bytes(s, bb.BSA_SCORE_MEAN)
    n_sel = bb.bsa_select_workspace_bytes(s, p)
    n = bb.bsa_score_select_workspace_bytes(s, bb.BSA_SCORE_MEAN, p)
    assert n >= n_sc + n_sel + 2 * 2 * 2048 * 4
    assert n < n_sc + n_sel + 32 * 1024 * 2048 * 4     # no scores array
    # K-min/K-max and fp32 inputs run unfused: the scores pass through the workspace
    nb = bb.bsa_score_select_workspace_bytes(s, bb.BSA_SCORE_KMINMAX, p)
    assert nb >= bb.bsa_score_workspace_bytes(s, bb.BSA_SCORE_KMINMAX) + n_sel + 32 * 1024 * 2048 * 4
    f = bb.Shape(1, 2, 2, 1024, 64, 64, 64, bb.BSA_F32)
    pf = bb.SelectParams(4, 4, 1, 0.25, float("nan"))
    nf = bb.bsa_score_select_workspace_bytes(f, bb.BSA_SCORE_MEAN, pf)
    assert nf >= bb.bsa_select_workspace_bytes(f, pf) + 2 * 16 * 16 * 4
    assert bb.bsa_score_select_workspace_bytes(s, 9, p) == 0
    assert bb.bsa_score_select_workspace_bytes(s, bb.BSA_SCORE_MEAN, bb.SelectParams(0, 0, 1, 0.25, 0.0)) == 0
    big = 1 << 36

    def call(kind=bb.BSA_SCORE_MEAN, sp=None, prm=p, q=256, k=256, v=None, kv=256, cnt=256, ws=256,
             wsb=big):
        return L.bsa_score_select(ctypes.byref(s), kind, sp, ctypes.byref(prm), q, k, v, None, kv, cnt,
                                  None, None, None, None, None, ws, wsb, None)
    assert call(kv=None) == bb.BSA_ERR_INVALID_ARG
    assert call(cnt=None) == bb.BSA_ERR_INVALID_ARG
    assert call(ws=None) == bb.BSA_ERR_INVALID_ARG
    assert call(q=None) == bb.BSA_ERR_INVALID_ARG
    assert call(ws=272) == bb.BSA_ERR_INVALID_ARG and b"256-byte" in L.bsa_last_error()
    assert call(q=264) == bb.BSA_ERR_INVALID_ARG and b"16-byte" in L.bsa_last_error()
    assert call(wsb=n - 1) == bb.BSA_ERR_INVALID_ARG and b"workspace" in L.bsa_last_error()
    assert call(kind=bb.BSA_SCORE_MEAN_VNORM) == bb.BSA_ERR_INVALID_ARG      # needs v
    assert call(kind=bb.BSA_SCORE_MEAN_VLOG, v=256) == bb.BSA_ERR_INVALID_ARG  # needs beta
    assert call(prm=bb.SelectParams(8, 9, 1, 0.25, 0.0)) == bb.BSA_ERR_INVALID_ARG


def test_decode_list_validation():
    L = bb.lib()
    ds = bb.DecodeShape(2, 32, 8, 8192, 128, 128, bb.BSA_BF16)
    dims = (ctypes.c_int * 4)(0, 1, 8, 9)
    dp = bb.DecodeParams(1e-3, 1e-4, 1, 1, 4, dims)
    args = (16, 16, 16)
    # list pointers required; width within 1..4096
    assert L.bsa_decode_list(ctypes.byref(ds), ctypes.byref(dp), *args, None, 16, 8, 0.1, 16, 16, None,
                             16, None) == bb.BSA_ERR_INVALID_ARG
    assert L.bsa_decode_list(ctypes.byref(ds), ctypes.byref(dp), *args, 16, 16, 0, 0.1, 16, 16, None,
                             16, None) == bb.BSA_ERR_UNSUPPORTED
    assert L.bsa_decode_list(ctypes.byref(ds), ctypes.byref(dp), *args, 16, 16, 5000, 0.1, 16, 16,
                             None, 16, None) == bb.BSA_ERR_UNSUPPORTED
    # the decode checks still apply
    bad = bb.DecodeParams(1e-3, 1e-4, 0, 1, 4, dims)
    assert L.bsa_decode_list(ctypes.byref(ds), ctypes.byref(bad), *args, 16, 16, 8, 0.1, 16, 16, None,
                             16, None) == bb.BSA_ERR_INVALID_ARG


def test_selftest_mode_validation():
    L = bb.lib()
    assert L.bsa_selftest_wait(3, 16, 16, None) == bb.BSA_ERR_INVALID_ARG
    assert L.bsa_selftest_wait(0, None, 16, None) == bb.BSA_ERR_INVALID_ARG


def test_attend_vs_validation():
    L = bb.lib()
    s = _shape(N=131072)
    assert bb.bsa_attend_vs_workspace_bytes(s, 64, 64) > 0
    assert bb.bsa_attend_vs_workspace_bytes(s, 64, 400) == 0          # 64 + 3*400 > 1024 lists
    assert bb.bsa_attend_vs_workspace_bytes(_shape(N=32768), 512, 512) > 0   # capped at n_kb = 512
    assert bb.bsa_attend_vs_workspace_bytes(_shape(d=64), 64, 64) == 0
    assert bb.bsa_attend_vs_workspace_bytes(_shape(tile_q=64), 64, 64) == 0
    assert bb.bsa_attend_vs_workspace_bytes(s, 0, 64) == 0
    big = 1 << 34
    assert L.bsa_attend_vs(ctypes.byref(s), 16, 16, 16, None, 16, 64, 16, 16, 64, 0.1, 16, None, 16, 256,
                           big, None) == bb.BSA_ERR_INVALID_ARG
    assert L.bsa_attend_vs(ctypes.byref(s), 16, 16, 16, 16, 16, 64, 16, 16, 400, 0.1, 16, None, 16, 256,
                           big, None) == bb.BSA_ERR_UNSUPPORTED
    assert L.bsa_attend_vs(ctypes.byref(s), 16, 16, 16, 16, 16, 64, 16, 16, 64, 0.1, 16, None, 16, 256,
                           100, None) == bb.BSA_ERR_INVALID_ARG
    assert b"workspace" in L.bsa_last_error()


def test_decode_cache_too_large_rejected():
    L = bb.lib()
    ds = bb.DecodeShape(64, 32, 8, 1 << 22, 128, 128, bb.BSA_BF16)     # 2^31 cache rows
    dims = (ctypes.c_int * 2)(0, 1)
    dp = bb.DecodeParams(1e-3, 1e-4, 1, 1, 2, dims)
    assert L.bsa_decode(ctypes.byref(ds), ctypes.byref(dp), 16, 16, 16, 0.1, 16, 16, None, 16,
                        None) == bb.BSA_ERR_UNSUPPORTED
    assert b"2^31" in L.bsa_last_error()


def test_kernel_path_queries():
    """Every shape the header lists as a CUDA-core fallback reports it, the workloads' shapes
    report tensor cores, and invalid arguments report -1 (nothing is launched)."""
    TC, CC = bb.BSA_PATH_TENSOR_CORES, bb.BSA_PATH_CUDA_CORES
    base = dict(B=1, Hq=32, Hkv=8, N=131072, d=128, block_k=64, tile_q=128, dtype=bb.BSA_BF16)

    def sh(**kw):
        a = dict(base, **kw)
        return bb.Shape(a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["block_k"], a["tile_q"], a["dtype"])
    # attend
    assert bb.bsa_attend_path(sh(), 128) == TC
    assert bb.bsa_attend_path(sh(), 1024) == TC
    assert bb.bsa_attend_path(sh(), 1025) == CC
    for kw in (dict(dtype=bb.BSA_F32), dict(d=64), dict(block_k=128), dict(tile_q=64)):
        assert bb.bsa_attend_path(sh(**kw), 64) == CC, kw
    assert bb.bsa_attend_path(sh(B=256, Hq=64, Hkv=8), 64) == CC         # B*Hq*N = 2^31
    assert bb.bsa_attend_path(sh(), 0) == -1 and bb.bsa_attend_path(sh(d=96), 64) == -1
    # score (and the fused score+select)
    for kind in range(4):
        assert bb.bsa_score_path(sh(), kind) == TC
        assert bb.bsa_score_path(sh(block_k=128), kind) == TC
        for kw in (dict(dtype=bb.BSA_F32), dict(d=64), dict(tile_q=64)):
            assert bb.bsa_score_path(sh(**kw), kind) == CC, (kind, kw)
    assert bb.bsa_score_path(sh(), 9) == -1
    # decode
    assert bb.bsa_decode_path(bb.DecodeShape(16, 32, 8, 65536, 128, 128, bb.BSA_BF16)) == TC
    assert bb.bsa_decode_path(bb.DecodeShape(2, 8, 8, 4096, 128, 128, bb.BSA_BF16)) == TC
    assert bb.bsa_decode_path(bb.DecodeShape(2, 8, 2, 4096, 64, 128, bb.BSA_BF16)) == CC
    assert bb.bsa_decode_path(bb.DecodeShape(2, 8, 2, 4096, 128, 64, bb.BSA_BF16)) == CC
    for hq, hkv in ((2, 2), (4, 2), (8, 1)):           # group sizes 1, 2, 8
        assert bb.bsa_decode_path(bb.DecodeShape(2, hq, hkv, 4096, 128, 128, bb.BSA_BF16)) == TC
    # shapes bsa_decode itself rejects: fp32 caches, a group of 3, L not a block multiple
    assert bb.bsa_decode_path(bb.DecodeShape(2, 8, 2, 4096, 128, 128, bb.BSA_F32)) == -1
    assert bb.bsa_decode_path(bb.DecodeShape(2, 6, 2, 4096, 128, 128, bb.BSA_BF16)) == -1
    assert bb.bsa_decode_path(bb.DecodeShape(2, 8, 2, 4000, 128, 128, bb.BSA_BF16)) == -1
    assert bb.bsa_decode_path(bb.DecodeShape(2, 6, 4, 4096, 128, 128, bb.BSA_BF16)) == -1
