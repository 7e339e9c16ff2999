"""bsa_select_noalloc against bsa_select, through the C ABI.

bsa_select_noalloc serves callers that cannot allocate device memory (a plugin
whose host process owns all device memory through its own pool, a serving
loop where a cudaMalloc could synchronise the device): it takes no workspace
and uses a static scratch array inside libbsa.so instead. Its results must be
the ones bsa_select gives with a caller-provided workspace -- bit for bit,
the tolerance every selection test here uses -- on two calls in a row (the
second on different inputs, so stale scratch contents would show). This file
sorts last so that a run stopping at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from block_sparse_causal_bsa_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def _to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def _outputs(B, Hq, n_qt, W):
    dev = torch.device("cuda")
    return dict(kv_idx=torch.full((B, Hq, n_qt, W), -7, dtype=torch.int32, device=dev),
                kv_cnt=torch.full((B, Hq, n_qt), -7, dtype=torch.int32, device=dev),
                sigma=torch.full((B, Hq, n_qt), -7.0, dtype=torch.float32, device=dev),
                sigma_bar=torch.full((B, n_qt), -7.0, dtype=torch.float32, device=dev),
                trigger=torch.full((B, n_qt), 7, dtype=torch.uint8, device=dev),
                theta=torch.full((1,), -7.0, dtype=torch.float32, device=dev),
                dev_status=torch.full((1,), -7, dtype=torch.int32, device=dev))


def _same(a, b):
    for key in ("kv_idx", "kv_cnt", "trigger", "dev_status"):
        assert torch.equal(a[key], b[key]), key
    for key in ("sigma", "sigma_bar", "theta"):
        assert torch.equal(a[key].view(torch.int32), b[key].view(torch.int32)), key


def _case(seed, k):
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=8192, Hq=8, Hkv=2)
    q, kk, v = S.prefill_inputs(spec, seed)
    qd, kd = _to_dev(q), _to_dev(kk)
    scores = bb.score(qd, kd, block_k=64, tile_q=128)
    shape = bb.make_shape(qd, kd, 64, 128)
    params = bb.SelectParams(k, k, 2, 0.25, float("nan"))
    return shape, params, scores


def _run_both(shape, params, scores):
    L = bb.lib()
    W = bb.bsa_kv_idx_width(shape, params)
    B, Hq, n_qt, _ = scores.shape
    ref = _outputs(B, Hq, n_qt, W)
    got = _outputs(B, Hq, n_qt, W)
    nb = bb.bsa_select_workspace_bytes(shape, params)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = L.bsa_select(ctypes.byref(shape), ctypes.byref(params), scores.data_ptr(),
                      ref["kv_idx"].data_ptr(), ref["kv_cnt"].data_ptr(), ref["sigma"].data_ptr(),
                      ref["sigma_bar"].data_ptr(), ref["trigger"].data_ptr(),
                      ref["theta"].data_ptr(), ref["dev_status"].data_ptr(), ws.data_ptr(), nb,
                      stream)
    assert st == bb.BSA_OK, L.bsa_last_error()
    st = L.bsa_select_noalloc(ctypes.byref(shape), ctypes.byref(params), scores.data_ptr(),
                              got["kv_idx"].data_ptr(), got["kv_cnt"].data_ptr(),
                              got["sigma"].data_ptr(), got["sigma_bar"].data_ptr(),
                              got["trigger"].data_ptr(), got["theta"].data_ptr(),
                              got["dev_status"].data_ptr(), stream)
    assert st == bb.BSA_OK, L.bsa_last_error()
    torch.cuda.synchronize()
    assert int(ref["dev_status"].item()) == 0
    _same(ref, got)
    return got


def test_noalloc_matches_workspace_path_twice():
    first = _run_both(*_case(3001, 8))
    second = _run_both(*_case(3002, 12))    # other inputs and budget on the same scratch
    assert int(first["trigger"].sum()) > 0 and int(second["trigger"].sum()) > 0
    assert not torch.equal(first["kv_cnt"], second["kv_cnt"])


def test_noalloc_without_optional_outputs():
    """sigma, sigma_bar and trigger NULL: the call then keeps them in the static scratch's
    own regions, and kv_idx, kv_cnt and theta must still match bsa_select bit for bit."""
    shape, params, scores = _case(3003, 10)
    L = bb.lib()
    W = bb.bsa_kv_idx_width(shape, params)
    B, Hq, n_qt, _ = scores.shape
    ref = _outputs(B, Hq, n_qt, W)
    got = _outputs(B, Hq, n_qt, W)
    nb = bb.bsa_select_workspace_bytes(shape, params)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                               # twice: the second call finds stale scratch
        st = L.bsa_select(ctypes.byref(shape), ctypes.byref(params), scores.data_ptr(),
                          ref["kv_idx"].data_ptr(), ref["kv_cnt"].data_ptr(), None, None, None,
                          ref["theta"].data_ptr(), ref["dev_status"].data_ptr(), ws.data_ptr(), nb,
                          stream)
        assert st == bb.BSA_OK, L.bsa_last_error()
        st = L.bsa_select_noalloc(ctypes.byref(shape), ctypes.byref(params), scores.data_ptr(),
                                  got["kv_idx"].data_ptr(), got["kv_cnt"].data_ptr(), None, None, None,
                                  got["theta"].data_ptr(), got["dev_status"].data_ptr(), stream)
        assert st == bb.BSA_OK, L.bsa_last_error()
        torch.cuda.synchronize()
        for key in ("kv_idx", "kv_cnt", "dev_status"):
            assert torch.equal(ref[key], got[key]), key
        assert torch.equal(ref["theta"].view(torch.int32), got["theta"].view(torch.int32))
    assert int(got["dev_status"].item()) == 0


def test_noalloc_shape_just_under_the_limit():
    """A layer whose selection workspace fills 99 % of the static scratch (63 query heads
    at 128k, W = 128): the call accepts it and matches bsa_select. Scores are random
    (the selection reads any finite scores)."""
    L = bb.lib()
    limit = L.bsa_select_noalloc_max_bytes()
    shape = bb.Shape(1, 63, 7, 131072, 128, 64, 128, bb.BSA_BF16)
    params = bb.SelectParams(64, 64, 2, 0.25, float("nan"))
    need = bb.bsa_select_workspace_bytes(shape, params)
    assert 0.98 * limit < need <= limit
    g = torch.Generator(device="cuda").manual_seed(3004)
    scores = torch.randn(1, 63, 1024, 2048, device="cuda", generator=g)
    _run_both(shape, params, scores)
    del scores


def test_noalloc_rejects_oversized_shapes():
    L = bb.lib()
    limit = L.bsa_select_noalloc_max_bytes()
    assert limit == 32 << 20
    shape = bb.Shape(4, 32, 8, 131072, 128, 64, 128, bb.BSA_BF16)   # ranked lists alone: 64 MiB
    params = bb.SelectParams(64, 64, 2, 0.25, float("nan"))
    assert bb.bsa_select_workspace_bytes(shape, params) > limit
    st = L.bsa_select_noalloc(ctypes.byref(shape), ctypes.byref(params), 256, 256, 256, None, None,
                              None, None, None, None)
    assert st == bb.BSA_ERR_UNSUPPORTED
    assert b"static maximum" in L.bsa_last_error()
