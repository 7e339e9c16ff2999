"""GPU path vs the CPU oracle, element by element, through the C ABI.

Every case draws seeded inputs from block_sparse_causal_bsa_b200.synthetic,
runs pool/score -> select -> attend (or decode) in libbsa.so, and compares:
scores within 1e-3 relative (row-scale floor), the whole selection
bit-exactly on the GPU's own scores, attention outputs within 2e-2 max-abs
and 1e-3 mean-abs, and the decode termination block bit-exactly on the GPU's
probe trace.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from block_sparse_causal_bsa_b200 import synthetic as S
from oracle import bsa_oracle as O

from gpu_util import (check_attend, check_scores, check_selection, inputs, out_rows, to_dev)

pytestmark = pytest.mark.gpu


def _cfg(spec, k_first=None, k_last=None):
    return bb.SelectConfig(k_first or spec.k_first, k_last or spec.k_last, spec.rho,
                           spec.gate_quantile)


def _run_prefill(spec, seed, k_first=None, k_last=None, tiles=None):
    (q, k, v), (qd, kd, vd) = inputs(spec, seed)
    oam = spec.score_kind == "mean_vnorm"
    cfg = _cfg(spec, k_first, k_last)
    out, sel, st = bb.prefill(qd, kd, vd, block_k=spec.block_k, tile_q=spec.tile_q, cfg=cfg,
                              output_aware=oam)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(sel["dev_status"].item()) == 0
    assert int(sel["score_status"].item()) == 0
    g_scores = sel["scores"].cpu().numpy()
    ref_scores = O.block_scores(q, k, spec.tile_q, spec.block_k, V=v if oam else None)
    check_scores(g_scores, ref_scores)
    ref_sel = O.select(g_scores, spec.tile_q, spec.block_k, cfg.k_first, cfg.k_last, cfg.rho,
                       cfg.gate_quantile)
    check_selection(sel, ref_sel)
    scale = 1.0 / math.sqrt(spec.d)
    ro, _ = O.attend(q, k, v, ref_sel["kv_idx"], spec.tile_q, spec.block_k, scale, tiles=tiles)
    go = out_rows(out)
    lognormal = spec.structure == "lognormal_v"
    if tiles is None:
        check_attend(go, ro, lognormal_v=lognormal)
    else:
        for b, h, t in tiles:
            r0 = t * spec.tile_q
            check_attend(go[b, h, r0:r0 + spec.tile_q], ro[b, h, r0:r0 + spec.tile_q],
                         lognormal_v=lognormal)
    return sel, ref_sel


def test_tiny_fp32_1k_full():
    spec = S.WORKLOADS["tiny_fp32_1k"]
    sel, ref = _run_prefill(spec, 1001)
    assert (sel["kv_cnt"].cpu().numpy()[0, :, 4:] == 4).all()


def test_prefill_vs_reduced():
    spec = S.WORKLOADS["prefill_32k_vs"].scaled(N=4096, Hq=8, Hkv=2)
    _run_prefill(spec, 1002, k_first=16, k_last=16)


def test_gated_reduced():
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=8192, Hq=8, Hkv=2)
    sel, ref = _run_prefill(spec, 1003, k_first=8, k_last=8)
    assert ref["trigger"].sum() > 0          # the gate fired somewhere
    assert ref["sigma"].min() == 0.0         # planted twins tie at the cut


def test_tpd_oam_reduced():
    spec = S.WORKLOADS["tpd_oam_prefill_64k"].scaled(N=4096, Hq=8, Hkv=2)
    _run_prefill(spec, 1004, k_first=16, k_last=4)


@pytest.mark.parametrize("tile_q,bk,d,dtype", [(64, 128, 64, "bf16"), (128, 128, 128, "bf16"),
                                               (64, 64, 128, "f32"), (128, 64, 64, "f32")])
def test_geometries(tile_q, bk, d, dtype):
    spec = S.PrefillSpec("geom", B=2, Hq=4, Hkv=4, N=2048, d=d, block_k=bk, tile_q=tile_q,
                         k_first=5, k_last=2, rho=2, gate_quantile=0.5, score_kind="mean",
                         dtype=dtype, structure="iid")
    _run_prefill(spec, 1005)


def test_single_tile_and_dense_budget():
    # one query tile only
    spec = S.PrefillSpec("one", B=1, Hq=2, Hkv=1, N=128, d=128, block_k=64, tile_q=128,
                         k_first=4, k_last=4, rho=1, gate_quantile=0.25, score_kind="mean",
                         dtype="bf16", structure="iid")
    _run_prefill(spec, 1006)
    # budget >= all blocks: block-sparse attention is dense causal attention
    spec = S.PrefillSpec("dense", B=1, Hq=2, Hkv=2, N=1024, d=64, block_k=64, tile_q=64,
                         k_first=16, k_last=16, rho=1, gate_quantile=0.25, score_kind="mean",
                         dtype="f32", structure="iid")
    (q, k, v), (qd, kd, vd) = inputs(spec, 1007)
    out, sel, st = bb.prefill(qd, kd, vd, block_k=64, tile_q=64, cfg=_cfg(spec))
    torch.cuda.synchronize()
    for h in range(2):
        ref = O.dense_causal_attention(q[0, h], k[0, h], v[0, h], 1 / 8.0)
        check_attend(out_rows(out)[0, h], ref)


# ---------------------------------------------------------------------------
# device-side error reporting (no fault, no trap: the bad work is skipped)

def test_bad_kv_idx_sets_status():
    spec = S.WORKLOADS["tiny_fp32_1k"]
    (q, k, v), (qd, kd, vd) = inputs(spec, 1008)
    s = bb.score(qd, kd, block_k=64, tile_q=64)
    shape = bb.make_shape(qd, kd, 64, 64)
    sel = bb.select(s, shape=shape, cfg=_cfg(spec))
    kv = sel["kv_idx"].clone()
    kv[0, 0, 5, 0] = 999          # beyond n_kb
    kv[0, 1, 3, 0] = 10           # beyond the tile's last visible block
    out, _, st = bb.attend(qd, kd, vd, kv, sel["kv_cnt"], block_k=64, tile_q=64)
    torch.cuda.synchronize()
    assert int(st.item()) & bb.BSA_DEV_BAD_INDEX
    # rows of untouched tiles are still right
    ref, _ = O.attend(q, k, v, sel["kv_idx"].cpu().numpy(), 64, 64, 1 / 8.0, tiles=[(0, 0, 6)])
    check_attend(out_rows(out)[0, 0, 384:448], ref[0, 0, 384:448])


def test_nonfinite_score_sets_status():
    spec = S.WORKLOADS["tiny_fp32_1k"]
    (q, k, v), (qd, kd, vd) = inputs(spec, 1009)
    s = bb.score(qd, kd, block_k=64, tile_q=64)
    s[0, 0, 10, 3] = float("nan")
    shape = bb.make_shape(qd, kd, 64, 64)
    sel = bb.select(s, shape=shape, cfg=_cfg(spec))
    torch.cuda.synchronize()
    assert int(sel["dev_status"].item()) & bb.BSA_DEV_BAD_SCORE
    assert math.isnan(float(sel["sigma"][0, 0, 10]))


# ---------------------------------------------------------------------------
# decode with run-time termination

def _decode_inputs(spec, seed):
    q, k, v = S.decode_inputs(spec, seed)
    return (q, k, v), (to_dev(q), to_dev(k), to_dev(v))


def _check_decode(spec, seed, tau, phi, patience, enable=True, groups=None):
    (q, k, v), (qd, kd, vd) = _decode_inputs(spec, seed)
    dims = S.default_probe_dims(32 if spec.d == 128 else 16)
    scale = 1.0 / math.sqrt(spec.d)
    out, used, trace, st = bb.decode(qd, kd, vd, block_kv=spec.block_kv, tau=tau, phi=phi,
                                     patience=patience, enable=enable, probe_dims=dims,
                                     want_trace=True)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    used = used.cpu().numpy()
    trace = trace.cpu().numpy()
    go = out_rows(out)
    G = spec.Hq // spec.Hkv
    nb = spec.L // spec.block_kv
    agree = 0
    pairs = [(b, g) for b in range(spec.B) for g in range(spec.Hkv)]
    for b, g in pairs:
        u = int(used[b, g])
        # bit-exact termination given the GPU's own probes
        exp = O.termination_block(trace[b, g], tau, phi, patience, n_blocks=nb) if enable else nb
        assert u == exp, (b, g, u, exp)
        assert np.isfinite(trace[b, g, :u]).all()
    for b, g in (pairs if groups is None else groups):
        u = int(used[b, g])
        # output = attention over exactly the processed blocks
        o_ref, _, _ = O.decode_group(q[b, g * G:(g + 1) * G], k[b, g, :u * spec.block_kv],
                                     v[b, g, :u * spec.block_kv], spec.block_kv, scale, tau, phi,
                                     patience, dims, enable=False)
        check_attend(go[b, g * G:(g + 1) * G], o_ref)
        # the oracle's own end-to-end decision
        _, u_ref, tr_ref = O.decode_group(q[b, g * G:(g + 1) * G], k[b, g], v[b, g], spec.block_kv,
                                          scale, tau, phi, patience, dims, enable=enable)
        agree += int(u_ref == u)
        np.testing.assert_allclose(trace[b, g, :min(u, u_ref)], tr_ref[:min(u, u_ref)], atol=2e-3)
    return used, agree


def test_decode_reduced():
    spec = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=2, L=8192)
    used, agree = _check_decode(spec, 1010, spec.tau, spec.phi, spec.patience)
    assert agree >= 0.8 * 16


def test_decode_limits():
    spec = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=1, L=4096)
    used, _ = _check_decode(spec, 1011, 0.0, 0.0, 1)
    assert (used == 32).all()                       # never stable: full scan
    used, _ = _check_decode(spec, 1011, float("inf"), float("inf"), 3)
    assert (used == 4).all()                        # stable every time: p + 1 blocks
    used, _ = _check_decode(spec, 1011, float("inf"), float("inf"), 1, enable=False)
    assert (used == 32).all()


def test_decode_decider_at_its_thresholds():
    """tau, then phi, set to the value the stability test computes on some block (its
    minimum or median over the blocks of one group), so that a fast approximate screen of the
    test cannot decide there and the defining fp64 evaluation has to: the stop must still
    be the one the oracle's decision function gives on the GPU's probe trace."""
    spec = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=1, L=4096)
    (_, _, _), (qd, kd, vd) = _decode_inputs(spec, 1012)
    dims = S.default_probe_dims(32)
    _, _, trace, st = bb.decode(qd, kd, vd, block_kv=spec.block_kv, tau=0.0, phi=0.0, patience=1,
                                enable=False, probe_dims=dims, want_trace=True)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    tr = trace.cpu().numpy()[0, 0]                      # group (0, 0), every block
    steps = [O.probe_step(tr[t - 1], tr[t]) for t in range(1, tr.shape[0])]
    ds = np.array([x[0] for x in steps])
    dd = np.array([x[1] for x in steps])
    f32 = lambda x: float(np.float32(x))
    for tau, phi in ((f32(ds.min()), 2.0), (f32(np.sort(ds)[len(ds) // 2]), 2.0),
                     (float("inf"), f32(dd.min())), (float("inf"), f32(np.sort(dd)[len(dd) // 2]))):
        _check_decode(spec, 1012, tau, phi, 1)


@pytest.mark.parametrize("nb", [1, 2, 3, 4, 5, 7, 9])
def test_decode_stop_on_each_late_block(nb):
    """A stop on every block of short caches, the last two included: the kernel reads the
    verdict on a block two blocks later, so a stop on the next-to-last block is settled
    after its loop, one on the last block leaves the full result, and a stop seen as a
    halt before the next score block arrives is traced back to its block."""
    spec = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=2, L=128 * nb)
    for p in range(1, nb + 1):
        used, _ = _check_decode(spec, 1014, float("inf"), float("inf"), p)
        assert (used == min(p + 1, nb)).all(), (nb, p, used)


@pytest.mark.parametrize("Hq,Hkv,d,bkv", [(8, 1, 128, 128), (2, 2, 128, 128), (4, 2, 128, 128),
                                          (4, 4, 64, 64), (8, 4, 128, 64)])
def test_decode_shapes(Hq, Hkv, d, bkv):
    """Group sizes 8, 1 and 2 on the tensor cores (4 is the workload's), and CUDA-core shapes."""
    spec = S.DecodeSpec("dec", B=2, Hq=Hq, Hkv=Hkv, L=2048, d=d, block_kv=bkv, tau=1e-2,
                        phi=1e-3, patience=2)
    _check_decode(spec, 1012, spec.tau, spec.phi, spec.patience)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_attend_arbitrary_lists(dtype):
    """Caller-made kv_idx rows: unsorted, odd and even counts, duplicates of
    nothing, rows without their diagonal block (their early rows see no key:
    output 0, lse -inf), and entries beyond kv_cnt that must be ignored."""
    spec = S.PrefillSpec("lists", B=1, Hq=4, Hkv=2, N=2048, d=128, block_k=64, tile_q=128,
                         k_first=8, k_last=8, rho=1, gate_quantile=0.25, score_kind="mean",
                         dtype=dtype, structure="iid")
    (q, k, v), (qd, kd, vd) = inputs(spec, 1013)
    rng = np.random.default_rng(5)
    n_qt, W = spec.n_qt, 9
    kv = np.full((1, 4, n_qt, W), -1, np.int32)
    cnt = np.zeros((1, 4, n_qt), np.int32)
    for h in range(4):
        for t in range(n_qt):
            J = 2 * t + 1
            c = int(rng.integers(0, min(W, J + 1) + 1))
            sel = rng.permutation(J + 1)[:c]
            kv[0, h, t, :c] = sel
            kv[0, h, t, c:] = rng.integers(0, J + 1, size=W - c)   # ignored garbage
            cnt[0, h, t] = c
    kvd, cntd = torch.from_numpy(kv).cuda(), torch.from_numpy(cnt).cuda()
    out, lse, st = bb.attend(qd, kd, vd, kvd, cntd, block_k=64, tile_q=128, want_lse=True)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    kv_used = kv.copy()
    for h in range(4):
        for t in range(n_qt):
            kv_used[0, h, t, cnt[0, h, t]:] = -1
    ro, rl = O.attend(q, k, v, kv_used, 128, 64, 1 / math.sqrt(128))
    check_attend(out_rows(out), ro)
    gl = lse.cpu().numpy()
    assert np.array_equal(np.isneginf(gl), np.isneginf(rl))
    fin = np.isfinite(rl)
    np.testing.assert_allclose(gl[fin], rl[fin], atol=1e-3)
