"""Scores and selection in one call (bsa_score_select) against the oracle.

Where the tensor-core score kernel ranks the rows itself (bf16, d 128, query tiles
of 128, the mean-pooled kinds), the call must give:
  - scores (when asked for) within the 1e-3 relative bar of the oracle's;
  - a selection bit-identical to the oracle's selection on those scores
    ([UGS] steps 2-5: ranking, sigma, gate, kv_idx);
  - the same selection when the scores are not written out (the rows then pass
    through the kernel's L2 ring instead of the scores array);
  - the same selection as bsa_select run separately on the same scores.
Cases span several units per CTA (so the row ring and both Q buffers are reused),
one and two query heads per unit, key blocks of 64 and 128, and the output-aware
kinds. A non-finite input must raise BSA_DEV_BAD_SCORE without a fault.
"""
import numpy as np
import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from block_sparse_causal_bsa_b200 import synthetic as S
from oracle import bsa_oracle as O

from gpu_util import check_scores, check_selection, inputs

pytestmark = pytest.mark.gpu

SEL_KEYS = ("kv_idx", "kv_cnt", "sigma", "sigma_bar", "trigger", "theta")


def _same_selection(a, b):
    for key in SEL_KEYS:
        x, y = a[key], b[key]
        if x.dtype == torch.float32:
            x, y = x.view(torch.int32), y.view(torch.int32)
        assert torch.equal(x, y), key


def _case(spec, seed, kind="mean", beta=0.0, block_k=None):
    bk = block_k or spec.block_k
    (q, k, v), (qd, kd, vd) = inputs(spec, seed)
    cfg = bb.SelectConfig(spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    r = bb.score_select(qd, kd, vd, block_k=bk, tile_q=spec.tile_q, cfg=cfg, kind=kind, beta=beta,
                        want_scores=True)
    r2 = bb.score_select(qd, kd, vd, block_k=bk, tile_q=spec.tile_q, cfg=cfg, kind=kind, beta=beta,
                         want_scores=False)
    torch.cuda.synchronize()
    assert int(r["dev_status"].item()) == 0 and int(r2["dev_status"].item()) == 0
    g = r["scores"].cpu().numpy()
    okind = {"mean": "mean", "vnorm": "vnorm", "vlog": "vlog"}[kind]
    ref = O.block_scores(q, k, spec.tile_q, bk, V=v, kind=okind, beta=beta)
    check_scores(g, ref)
    ref_sel = O.select(g, spec.tile_q, bk, spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    check_selection(r, ref_sel)
    _same_selection(r, r2)
    # the standalone selection on the same scores
    shape = bb.make_shape(qd, kd, bk, spec.tile_q)
    r3 = bb.select(r["scores"], shape=shape, cfg=cfg)
    torch.cuda.synchronize()
    assert int(r3["dev_status"].item()) == 0
    _same_selection(r, r3)
    return r, ref_sel


def test_fused_gated_several_units_per_cta():
    # 2 KV heads x 128 tiles x 2 head pairs = 512 units on ~148 CTAs
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=16384, Hq=8, Hkv=2)
    r, ref = _case(spec, 2101)
    assert ref["trigger"].sum() > 0 and ref["cut"].sum() > 0


def test_fused_one_head_per_unit():
    # three query heads per KV head: odd group, one head per unit (N = 128 MMAs)
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=8192, Hq=6, Hkv=2)
    _case(spec, 2102)


def test_fused_key_blocks_of_128():
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=16384, Hq=4, Hkv=1, k_first=24, k_last=24,
                                                    block_k=128)
    _case(spec, 2103)


def test_fused_rows_not_16_byte_aligned():
    # n_kb = 74: score rows start on 8-byte boundaries, so the rank warps copy them one
    # element at a time
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=128 * 37, Hq=8, Hkv=2, k_first=12, k_last=12)
    _case(spec, 2108)


@pytest.mark.parametrize("kind,beta", [("vnorm", 0.0), ("vlog", 0.5)])
def test_fused_output_aware_with_budget_decay(kind, beta):
    spec = S.WORKLOADS["tpd_oam_prefill_64k"].scaled(N=8192, Hq=8, Hkv=2, B=2, k_first=32, k_last=8)
    _case(spec, 2104, kind=kind, beta=beta)


def test_fused_fixed_threshold_and_no_gate():
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=8192, Hq=4, Hkv=1)
    (q, k, v), (qd, kd, vd) = inputs(spec, 2105)
    for cfg in (bb.SelectConfig(16, 16, 2, -1.0, 0.3), bb.SelectConfig(16, 16, 1, 0.25)):
        r = bb.score_select(qd, kd, vd, block_k=64, tile_q=128, cfg=cfg, want_scores=True)
        torch.cuda.synchronize()
        ref = O.select(r["scores"].cpu().numpy(), 128, 64, cfg.k_first, cfg.k_first, cfg.rho,
                       cfg.gate_quantile, cfg.gate_threshold)
        check_selection(r, ref)


def test_fused_nonfinite_input_reports_bad_score():
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=4096, Hq=4, Hkv=1)
    (q, k, v), (qd, kd, vd) = inputs(spec, 2106)
    qd[0, 1, 3000, 5] = float("inf")
    cfg = bb.SelectConfig(8, 8, 2, 0.25)
    for want in (True, False):
        r = bb.score_select(qd, kd, vd, block_k=64, tile_q=128, cfg=cfg, want_scores=want)
        torch.cuda.synchronize()
        assert int(r["dev_status"].item()) == bb.BSA_DEV_BAD_SCORE
        # the tile holding the bad row reports NaN sigma; other heads' rows are untouched
        assert torch.isnan(r["sigma"][0, 1, 3000 // 128]).item()
        assert not torch.isnan(r["sigma"][0, 0]).any().item()


def test_standalone_score_matches_fused_scores():
    """bsa_score alone (the same kernel without the ranking warps) writes the same scores."""
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=8192, Hq=8, Hkv=2)
    (q, k, v), (qd, kd, vd) = inputs(spec, 2107)
    cfg = bb.SelectConfig(spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    r = bb.score_select(qd, kd, vd, block_k=64, tile_q=128, cfg=cfg, want_scores=True)
    s = bb.score(qd, kd, block_k=64, tile_q=128)
    torch.cuda.synchronize()
    assert torch.equal(r["scores"].view(torch.int32), s.view(torch.int32))
