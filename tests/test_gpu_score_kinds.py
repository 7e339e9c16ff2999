"""The added block-score backbones on the GPU against the oracle.

BSA_SCORE_MEAN_VLOG: the tile max of q . mean(K block) plus
beta * max(0, ln ||mean(V block)||^2) ([Stem] 2.B's additive Output-Aware
Metric at block level). BSA_SCORE_KMINMAX: the tile max of
sum_c max(q_c kmin_c, q_c kmax_c) (the K-min/K-max backbone of [UGS]
Metodologia step 1). Scores within 1e-3 (row-scale floor), the selection
bit-exact on the GPU's scores, attention within 2e-2 / 1e-3 -- on the
tensor-core shapes (bf16, d 128, tiles of 128) and on the CUDA-core ones.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from block_sparse_causal_bsa_b200 import synthetic as S
from oracle import bsa_oracle as O

from gpu_util import check_attend, check_scores, check_selection, inputs, out_rows, to_dev

pytestmark = pytest.mark.gpu


def _run(spec, seed, kind, beta=0.0):
    (q, k, v), (qd, kd, vd) = inputs(spec, seed)
    cfg = bb.SelectConfig(spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    out, sel, st = bb.prefill(qd, kd, vd, block_k=spec.block_k, tile_q=spec.tile_q, cfg=cfg,
                              kind=kind, beta=beta)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(sel["dev_status"].item()) == 0
    assert int(sel["score_status"].item()) == 0
    g = sel["scores"].cpu().numpy()
    okind = {"vlog": "vlog", "kminmax": "bounds"}[kind]
    ref = O.block_scores(q, k, spec.tile_q, spec.block_k, V=v, kind=okind, beta=beta)
    check_scores(g, ref)
    ref_sel = O.select(g, spec.tile_q, spec.block_k, cfg.k_first, cfg.k_last, cfg.rho,
                       cfg.gate_quantile)
    check_selection(sel, ref_sel)
    ro, _ = O.attend(q, k, v, ref_sel["kv_idx"], spec.tile_q, spec.block_k, 1 / math.sqrt(spec.d))
    check_attend(out_rows(out), ro, lognormal_v=spec.structure == "lognormal_v")
    return g, ref_sel


@pytest.mark.parametrize("beta", [0.5, 4.0])
def test_additive_value_term_tensor_core(beta):
    spec = S.WORKLOADS["tpd_oam_prefill_64k"].scaled(N=4096, Hq=8, Hkv=2, B=1, k_first=16,
                                                     k_last=4)
    g, _ = _run(spec, 1501, "vlog", beta)
    # the value term moves the scores away from the plain mean score
    _, (qd, kd, _) = inputs(spec, 1501)
    m = bb.score(qd, kd, block_k=64, tile_q=128).cpu().numpy()
    fin = np.isfinite(m)
    assert (g[fin] > m[fin]).any() and (g[fin] >= m[fin] - 1e-3 * np.abs(m[fin]) - 1e-6).all()


def test_kminmax_tensor_core():
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=4096, Hq=8, Hkv=2, k_first=12, k_last=12)
    g, ref_sel = _run(spec, 1502, "kminmax")
    assert ref_sel["trigger"].sum() > 0


@pytest.mark.parametrize("N,Hq,Hkv,bk", [(16384, 4, 1, 64), (32768, 2, 2, 128)])
def test_kminmax_scores_several_chunks(N, Hq, Hkv, bk):
    """K-min/K-max scores of whole layers whose late tiles span two chunks of 128 blocks,
    with several units per persistent CTA, one and four query heads per KV head."""
    spec = S.PrefillSpec("kmm", B=1, Hq=Hq, Hkv=Hkv, N=N, d=128, block_k=bk, tile_q=128,
                         k_first=8, k_last=8, rho=2, gate_quantile=0.25, score_kind="mean",
                         dtype="bf16", structure="twins", p_twin=0.36)
    (q, k, _), (qd, kd, _) = inputs(spec, 1504)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = bb.score(qd, kd, block_k=bk, tile_q=128, kind="kminmax", status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_scores(g.cpu().numpy(), O.block_scores(q, k, 128, bk, kind="bounds"))


def test_kminmax_scores_full_size_sampled():
    """The 128k gated workload's K-min/K-max scores on sampled rows (the first and last
    tiles included) against the oracle's per-row bound."""
    spec = S.WORKLOADS["gated_prefill_128k"]
    q, k, _ = S.prefill_inputs(spec, 1505)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = bb.score(to_dev(q), to_dev(k), block_k=spec.block_k, tile_q=spec.tile_q, kind="kminmax",
                 status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    G = spec.Hq // spec.Hkv
    rng = np.random.default_rng(1505)
    rows = [(0, 0, 0), (spec.B - 1, spec.Hq - 1, spec.n_qt - 1)] + [
        (int(rng.integers(spec.B)), int(rng.integers(spec.Hq)), int(rng.integers(spec.n_qt))) for _ in range(6)]
    bounds = {}
    for b, h, t in rows:
        if (b, h // G) not in bounds:
            bounds[b, h // G] = O.key_block_bounds(k[b, h // G], spec.block_k)
        kmin, kmax = bounds[b, h // G]
        _, J = O.tile_blocks(t, spec.tile_q, spec.block_k)
        ref = O.score_tile_bounds(q[b, h, t * spec.tile_q:(t + 1) * spec.tile_q], kmin, kmax, J)
        check_scores(g[b, h, t].cpu().numpy()[None], ref[None])


@pytest.mark.parametrize("kind", ["vlog", "kminmax"])
@pytest.mark.parametrize("tile_q,bk,d,dtype", [(64, 64, 128, "bf16"), (128, 64, 64, "f32")])
def test_score_kinds_cuda_core(kind, tile_q, bk, d, dtype):
    spec = S.PrefillSpec("kinds", B=1, Hq=4, Hkv=2, N=2048, d=d, block_k=bk, tile_q=tile_q,
                         k_first=6, k_last=3, rho=2, gate_quantile=0.5, score_kind="mean",
                         dtype=dtype, structure="iid")
    _run(spec, 1503, kind, beta=1.5)
