"""The bounded device wait, driven to its limit on the GPU without a fault.

bsa_selftest_wait runs the library's mbarrier wait (the one the tensor-core
kernels use for every pipeline stage) on barriers that nothing completes: the
wait must give up after its limit, report BSA_DEV_TIMEOUT in the device status
word, release the second waiter through the abort flag, and leave the context
usable -- a small prefill afterwards still matches the oracle.
"""
import time

import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from block_sparse_causal_bsa_b200 import synthetic as S
from oracle import bsa_oracle as O

from gpu_util import check_attend, inputs, out_rows

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    done = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    bb.bsa_selftest_wait(0, st, done)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == bb.BSA_DEV_TIMEOUT
    assert done.tolist() == [0, 0]
    assert 0.9 <= dt < 10.0, dt


def test_wait_completes_in_control_case():
    st = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    done = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    bb.bsa_selftest_wait(1, st, done)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert done.tolist() == [1, 1]


def test_context_usable_after_timeout():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    done = torch.zeros(2, dtype=torch.int32, device="cuda")
    bb.bsa_selftest_wait(0, st, done)
    torch.cuda.synchronize()
    assert int(st.item()) == bb.BSA_DEV_TIMEOUT
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=2048, Hq=4, Hkv=1)
    (q, k, v), (qd, kd, vd) = inputs(spec, 1301)
    cfg = bb.SelectConfig(8, 8, spec.rho, spec.gate_quantile)
    out, sel, st2 = bb.prefill(qd, kd, vd, block_k=spec.block_k, tile_q=spec.tile_q, cfg=cfg)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    ref, _ = O.attend(q, k, v, sel["kv_idx"].cpu().numpy(), spec.tile_q, spec.block_k, 1 / 128 ** 0.5)
    check_attend(out_rows(out), ref)


def test_invalid_mode_rejected():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    done = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(bb.BsaError):
        bb.bsa_selftest_wait(2, st, done)
