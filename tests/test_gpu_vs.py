"""Vertical-slash sparse attention (bsa_attend_vs) against the oracle.

Each query row attends to its vertical columns j <= i and the keys i - o of its
slash offsets, each key once ([VSP] Metodologia A, B.3). Outputs within the
attention bar (2e-2 max, 1e-3 mean), lse within 1e-3, rows with no key give 0
and -inf; out-of-range indices set BSA_DEV_BAD_INDEX and are skipped.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from block_sparse_causal_bsa_b200 import synthetic as S
from oracle import bsa_oracle as O

from gpu_util import check_attend, inputs, out_rows

pytestmark = pytest.mark.gpu


def _dev(*xs):
    return [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in xs]


def _run(spec, seed, v_idx, v_cnt, s_off, s_cnt, rows=None, expect_status=0):
    (q, k, v), (qd, kd, vd) = inputs(spec, seed)
    out, lse, st = bb.attend_vs(qd, kd, vd, *_dev(v_idx, v_cnt, s_off, s_cnt), want_lse=True)
    torch.cuda.synchronize()
    assert int(st.item()) == expect_status
    ro, rl = O.attend_vs(q, k, v, v_idx, v_cnt, s_off, s_cnt, 1 / math.sqrt(spec.d), rows=rows)
    go, gl = out_rows(out), lse.cpu().numpy()
    if rows is None:
        check_attend(go, ro)
        sel = np.ones(rl.shape, bool)
    else:
        idx = tuple(np.array(rows).T)
        check_attend(go[idx], ro[idx])
        sel = np.zeros(rl.shape, bool)
        sel[idx] = True
    assert np.array_equal(np.isneginf(gl[sel]), np.isneginf(rl[sel]))
    fin = sel & np.isfinite(rl)
    np.testing.assert_allclose(gl[fin], rl[fin], atol=1e-3)
    return go, gl


def test_vs_full_rows():
    spec = S.WORKLOADS["prefill_32k_vs"].scaled(N=2048, Hq=4, Hkv=2)
    idx = S.vs_indices(spec, 1601, n_vertical=24, n_slash=20, n_local=8)
    _run(spec, 1602, *idx)


def test_vs_sampled_rows_long():
    """N = 16384: the merged block lists (width 32 + 3*24 = 104) are shorter than the
    256 key blocks, so the list construction matters; rows sampled over all tiles."""
    spec = S.WORKLOADS["prefill_32k_vs"].scaled(N=16384, Hq=4, Hkv=1)
    idx = S.vs_indices(spec, 1603, n_vertical=32, n_slash=24, n_local=16)
    rng = np.random.default_rng(3)
    rows = [(0, h, int(i)) for h in range(4) for i in rng.choice(16384, 300, replace=False)]
    rows += [(0, h, i) for h in range(4) for i in (0, 1, 127, 128, 16383)]
    _run(spec, 1604, *idx, rows=rows)


def test_vs_empty_rows_and_bad_entries():
    spec = S.WORKLOADS["prefill_32k_vs"].scaled(N=1024, Hq=2, Hkv=1)
    v_idx = np.array([[[700, 300, 5000, -2]] * 2], np.int32)       # two out of range
    v_cnt = np.array([[4, 2]], np.int32)
    s_off = np.array([[[200, 3, 64]] * 2], np.int32)
    s_cnt = np.array([[3, 7]], np.int32)                           # 7 > width: clamped, reported
    go, gl = _run(spec, 1605, v_idx, v_cnt, s_off, s_cnt, expect_status=bb.BSA_DEV_BAD_INDEX)
    # rows 0..2 see no key: no vertical column <= i and every offset > i
    assert not go[0, :, :3].any() and np.isneginf(gl[0, :, :3]).all()
    assert np.isfinite(gl[0, :, 3:]).all()


def test_vs_unsupported_shape_rejected():
    spec = S.PrefillSpec("vs64", B=1, Hq=2, Hkv=1, N=1024, d=64, block_k=64, tile_q=128, k_first=4,
                         k_last=4, rho=1, gate_quantile=0.25, score_kind="mean", dtype="bf16",
                         structure="iid")
    (_, (qd, kd, vd)) = inputs(spec, 1606)
    idx = _dev(*S.vs_indices(spec, 1607, 8, 8, 4))
    with pytest.raises(bb.BsaError):
        bb.attend_vs(qd, kd, vd, *idx)
