"""Pins for the CPU oracle: it is checked against things other than itself
(hand-worked fixtures, closed forms, library routines, brute force).

Sources: "Resumo Técnico: Seleção com Portão de Incerteza para Atenção de
Esparsidade em Blocos" (Metodologia steps 1-5), "Stem: Rethinking Causal
Information Flow in Sparse Attention" (2. Metodologia A and B),
"Resumo Técnico: ART (Attention Run-time Termination)" (2.1-2.4).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import bsa_oracle as O
from block_sparse_causal_bsa_b200 import synthetic as S


def _parse_float(s):
    return float("-inf") if s == "-inf" else float(s)


# ---------------------------------------------------------------------------
# sigma (hand-worked fixture)

def test_cut_margin_golden(golden_dir):
    n = 0
    for line in open(os.path.join(golden_dir, "cut_margin.txt")):
        if line.startswith("#") or not line.strip():
            continue
        m, scores, sigma, _ = [p.strip() for p in line.split(";")]
        s = np.array([float(x) for x in scores.split()], np.float32)
        order = O.rank_candidates(s, len(s))
        got = O.cut_margin(s, order, int(m))
        assert got == np.float32(float(sigma)), (line, got)
        n += 1
    assert n == 8


def test_sigma_in_unit_interval_and_ties():
    rng = np.random.default_rng(0)
    for _ in range(2000):
        n = int(rng.integers(2, 40))
        m = int(rng.integers(1, n))
        s = rng.standard_normal(n).astype(np.float32) * np.float32(10 ** rng.uniform(-3, 3))
        order = O.rank_candidates(s, n)
        sig = O.cut_margin(s, order, m)
        assert 0.0 <= sig <= 1.0
        # plant an exact tie across the cut: the block ranked m gets the score of rank m-1
        s2 = s.copy()
        s2[order[m]] = s2[order[m - 1]]
        o2 = O.rank_candidates(s2, n)
        assert O.cut_margin(s2, o2, m) == 0.0
    # a dominant kept set with a flat tail: sigma = 1 exactly
    s = np.array([9, 9, 9, 0, 0, 0], np.float32)
    assert O.cut_margin(s, O.rank_candidates(s, 6), 3) == 1.0


def test_rank_rejects_nonfinite():
    with pytest.raises(ValueError):
        O.rank_candidates(np.array([1, np.nan, 0], np.float32), 3)
    with pytest.raises(ValueError):
        O.rank_candidates(np.array([1, -np.inf, 0], np.float32), 3)


# ---------------------------------------------------------------------------
# top-k ranking against brute-force subset enumeration

def test_topk_brute_force():
    """For tiny rows, exactly one subset of size m has every kept block ranked
    above every dropped block under (score desc, index asc); it must equal the
    oracle's first m."""
    rng = np.random.default_rng(1)
    for _ in range(300):
        n = int(rng.integers(1, 8))
        m = int(rng.integers(0, n + 1))
        s = rng.integers(-3, 4, size=n).astype(np.float32)   # many ties
        def better(a, b):
            return s[a] > s[b] or (s[a] == s[b] and a < b)
        good = []
        for sub in itertools.combinations(range(n), m):
            kept = set(sub)
            if all(better(a, b) for a in kept for b in range(n) if b not in kept):
                good.append(kept)
        assert len(good) == 1
        assert set(O.rank_candidates(s, n)[:m].tolist()) == good[0]


# ---------------------------------------------------------------------------
# budget

def test_tpd_budget_golden(golden_dir):
    for line in open(os.path.join(golden_dir, "tpd_budget.txt")):
        if line.startswith("#") or not line.strip():
            continue
        t, k, _ = [p.strip() for p in line.split(";")]
        assert O.budget_k(int(t), 512, 128, 32) == int(k)


def test_budget_properties():
    for n_qt, kf, kl in [(512, 128, 32), (7, 10, 3), (1, 5, 2), (100, 64, 64)]:
        ks = [O.budget_k(t, n_qt, kf, kl) for t in range(n_qt)]
        assert ks[0] == kf and ks[-1] == (kl if n_qt > 1 else kf)
        assert all(a >= b for a, b in zip(ks, ks[1:]))
        assert all(kl <= k <= kf for k in ks)


def test_slots_and_width():
    # tile 128, blocks of 64: two forced blocks per tile, candidates 0..2t-1
    nF, nc, m, M = O.tile_slots(0, 1024, 128, 64, 64, 64, 2)
    assert (nF, nc, m, M) == (2, 0, 0, 0)
    nF, nc, m, M = O.tile_slots(10, 1024, 128, 64, 64, 64, 2)
    assert (nF, nc, m, M) == (2, 20, 20, 20)          # budget above the 22 visible blocks
    nF, nc, m, M = O.tile_slots(40, 1024, 128, 64, 64, 64, 2)
    assert (nF, nc, m, M) == (2, 80, 62, 80)
    nF, nc, m, M = O.tile_slots(500, 1024, 128, 64, 64, 64, 2)
    assert (nF, nc, m, M) == (2, 1000, 62, 126)
    assert O.kv_idx_width(131072, 128, 64, 64, 64, 2) == 128
    assert O.kv_idx_width(1024, 64, 64, 4, 4, 1) == 4
    assert O.kv_idx_width(65536, 128, 64, 128, 32, 1) == 128
    # forced blocks exceed a tiny budget
    nF, nc, m, M = O.tile_slots(5, 16, 128, 64, 1, 1, 1)
    assert (nF, m) == (2, 0)
    assert O.kv_idx_width(2048, 128, 64, 1, 1, 1) == 2
    # key blocks larger than the query tile: one forced block
    assert O.tile_blocks(5, 64, 128) == (2, 2)


# ---------------------------------------------------------------------------
# select / gate / finalize on the hand-worked layer

def _load_select_tiny(golden_dir):
    scores, kv, sig, trig, theta = {}, {}, {}, {}, None
    for line in open(os.path.join(golden_dir, "select_tiny.txt")):
        if line.startswith("#") or not line.strip():
            continue
        head, rest = line.split(":", 1)
        head = head.split()
        if head[0] == "scores":
            scores[int(head[1])] = [_parse_float(x) for x in rest.split()]
        elif head[0] == "kv":
            a, b, c = rest.split(";")
            kv[int(head[1])] = [int(x) for x in a.split()]
            sig[int(head[1])] = np.float32(float(b))
            trig[int(head[1])] = int(c)
        elif head[0] == "theta":
            theta = np.float32(float(rest))
    return scores, kv, sig, trig, theta


def test_select_golden(golden_dir):
    scores, kv, sig, trig, theta = _load_select_tiny(golden_dir)
    s = np.array([[[scores[t] for t in range(6)]]], np.float32)
    r = O.select(s, 64, 64, 3, 3, 2, 0.5)
    assert r["W"] == 6
    for t in range(6):
        assert r["kv_idx"][0, 0, t].tolist() == kv[t]
        assert r["kv_cnt"][0, 0, t] == sum(1 for x in kv[t] if x >= 0)
        assert r["sigma"][0, 0, t] == sig[t]
        assert r["trigger"][0, t] == trig[t]
    assert r["theta"] == theta


def test_gate_quantile_matches_numpy():
    rng = np.random.default_rng(2)
    for M in [1, 2, 3, 10, 257, 1024]:
        v = rng.random(M).astype(np.float32)
        for q in [0.0, 0.1, 0.25, 0.5, 0.9, 1.0]:
            th = O.empirical_quantile(v, q)
            ref = np.quantile(v.astype(np.float64), float(np.float32(q)), method="linear")
            assert abs(float(th) - ref) <= 4 * np.spacing(np.float32(max(abs(ref), 1e-30)))


def test_gate_trigger_counts():
    rng = np.random.default_rng(3)
    B, Hq, n_qt = 2, 4, 50
    sigma = rng.random((B, Hq, n_qt)).astype(np.float32)
    cut = np.ones(n_qt, bool)
    cut[:5] = False
    sigma[:, :, :5] = 1.0
    sbar, theta, trig = O.gate(sigma, cut, 2, 0.25)
    assert trig.sum() == int(((sbar < theta) & cut[None]).sum())
    assert trig[:, :5].sum() == 0
    # about a quarter of the cut tiles fall strictly below the 25% quantile
    assert abs(trig.sum() - 0.25 * B * 45) <= 2
    # q = 0: theta = min, strict comparison -> nothing triggers
    _, th0, t0 = O.gate(sigma, cut, 2, 0.0)
    assert t0.sum() == 0 and th0 == sbar[:, cut].min()
    # rho = 1: no expansion, no trigger
    _, thn, tn = O.gate(sigma, cut, 1, 0.25)
    assert tn.sum() == 0 and np.isnan(thn)
    # fixed external threshold
    _, thf, tf = O.gate(sigma, cut, 2, -1.0, 0.5)
    assert thf == np.float32(0.5) and tf.sum() == int(((sbar < 0.5) & cut[None]).sum())


def test_head_mean_order():
    # fp32 sum in head order then a correctly rounded divide
    sigma = np.array([[[1e-8]], [[1.0]], [[-1.0]]], np.float32).reshape(1, 3, 1)
    sb = O.head_mean(sigma)
    acc = np.float32(np.float32(np.float32(0) + np.float32(1e-8)) + np.float32(1.0))
    acc = np.float32(acc + np.float32(-1.0))
    assert sb[0, 0] == np.float32(acc / np.float32(3))


def test_select_structure_random():
    rng = np.random.default_rng(4)
    B, Hq, tile_q, bk, N = 2, 3, 128, 64, 64 * 40
    n_qt, n_kb = N // tile_q, N // bk
    scores = rng.standard_normal((B, Hq, n_qt, n_kb)).astype(np.float32)
    for t in range(n_qt):
        scores[:, :, t, O.tile_blocks(t, tile_q, bk)[1] + 1:] = -np.inf
    r = O.select(scores, tile_q, bk, 8, 4, 2, 0.3)
    W = r["W"]
    assert W == 16
    for b in range(B):
        for h in range(Hq):
            for t in range(n_qt):
                nF, nc, m, M = O.tile_slots(t, n_qt, tile_q, bk, 8, 4, 2)
                row = r["kv_idx"][b, h, t]
                cnt = r["kv_cnt"][b, h, t]
                assert cnt == nF + (M if r["trigger"][b, t] else m)
                assert np.all(row[cnt:] == -1) and np.all(row[:cnt] >= 0)
                assert np.all(np.diff(row[:cnt]) > 0)
                assert set(range(nc, nc + nF)) <= set(row[:cnt].tolist())
                # the kept candidates outrank every dropped candidate
                kept = [j for j in row[:cnt] if j < nc]
                drop = [j for j in range(nc) if j not in kept]
                if kept and drop:
                    s = scores[b, h, t]
                    assert min(s[kept]) >= max(s[drop])


# ---------------------------------------------------------------------------
# pooling and scores (closed forms)

def test_pool_closed_form():
    rng = np.random.default_rng(5)
    bk, d, nb = 64, 16, 5
    a = rng.standard_normal((nb, d))
    u = rng.standard_normal((nb, d))
    offs = np.arange(bk) - (bk - 1) / 2.0          # zero-sum offsets
    K = (a[:, None, :] + offs[None, :, None] * u[:, None, :] / 64).reshape(nb * bk, d)
    Kb = O.pool_keys(K.astype(np.float32).astype(np.float64), bk)
    np.testing.assert_allclose(Kb, a, atol=1e-6)
    # value-block weight: rows v_j + zero-sum offsets, v_j = c_j * (3, 4, 0, ...)
    c = rng.random(nb) + 0.5
    v = np.zeros((nb, d))
    v[:, 0], v[:, 1] = 3 * c, 4 * c
    V = (v[:, None, :] + offs[None, :, None] * u[:, None, :] / 64).reshape(nb * bk, d)
    np.testing.assert_allclose(O.value_block_norm(V, bk), 5 * c, rtol=1e-12)


def test_score_closed_forms():
    rng = np.random.default_rng(6)
    tile_q, bk, d, N = 4, 2, 8, 16
    n_kb = N // bk
    Kb = rng.standard_normal((n_kb, d))
    # one-hot query rows pick coordinates: score = max of the picked coordinates of K_bar_j
    cols = np.array([1, 5, 5, 2])
    Qt = np.zeros((tile_q, d))
    Qt[np.arange(tile_q), cols] = 1.0
    J = 5
    s = O.score_tile(Qt, Kb, J)
    exp = Kb[:, [1, 5, 2]].max(axis=1).astype(np.float32)
    assert np.array_equal(s[: J + 1], exp[: J + 1])
    assert np.all(np.isneginf(s[J + 1:]))
    # output-aware form multiplies the max by w_j (negative max gets more negative)
    w = rng.random(n_kb) + 0.1
    s2 = O.score_tile(Qt, Kb, J, w)
    assert np.array_equal(s2[: J + 1], (Kb[:, [1, 5, 2]].max(axis=1) * w).astype(np.float32)[: J + 1])


def test_score_equals_mean_of_key_dots():
    """q . K_bar_j = (1/bk) sum_r q . k_r (linearity), checked per key."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, N, d, tile_q, bk = 1, 4, 2, 256, 16, 32, 16
    Q = rng.standard_normal((B, Hq, N, d)).astype(np.float32)
    K = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    s = O.block_scores(Q, K, tile_q, bk)
    n_qt, n_kb = N // tile_q, N // bk
    finite = 0
    for h in range(Hq):
        g = h // 2
        per_key = Q[0, h].astype(np.float64) @ K[0, g].astype(np.float64).T      # [N, N]
        for t in range(n_qt):
            rows = per_key[t * tile_q:(t + 1) * tile_q]
            for j in range(n_kb):
                ref = rows[:, j * bk:(j + 1) * bk].mean(axis=1).max()
                if j <= ((t + 1) * tile_q - 1) // bk:
                    assert abs(s[0, h, t, j] - ref) <= 1e-6 * max(1.0, abs(ref))
                    finite += 1
                else:
                    assert np.isneginf(s[0, h, t, j])
    assert finite == Hq * sum(((t + 1) * tile_q - 1) // bk + 1 for t in range(n_qt))


# ---------------------------------------------------------------------------
# attend: full budget reduces to dense causal attention (library routine)

def _sdpa(Q, K, V, scale):
    q = torch.from_numpy(O.widen(Q))[None, None]
    k = torch.from_numpy(O.widen(K))[None, None]
    v = torch.from_numpy(O.widen(V))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, is_causal=True, scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("tile_q,bk", [(64, 64), (128, 64), (64, 128)])
def test_attend_full_budget_is_dense(tile_q, bk):
    rng = np.random.default_rng(8)
    N, d, Hq, Hkv = 512, 32, 4, 2
    Q = S.f32_to_bf16_bits(rng.standard_normal((1, Hq, N, d)).astype(np.float32))
    K = S.f32_to_bf16_bits(rng.standard_normal((1, Hkv, N, d)).astype(np.float32))
    V = S.f32_to_bf16_bits(rng.standard_normal((1, Hkv, N, d)).astype(np.float32))
    n_kb, n_qt = N // bk, N // tile_q
    scores = O.block_scores(Q, K, tile_q, bk)
    r = O.select(scores, tile_q, bk, n_kb, n_kb, 1, 0.25)
    scale = 1.0 / math.sqrt(d)
    out, lse = O.attend(Q, K, V, r["kv_idx"], tile_q, bk, scale)
    for h in range(Hq):
        ref = _sdpa(Q[0, h], K[0, h // 2], V[0, h // 2], scale)
        np.testing.assert_allclose(out[0, h], ref, atol=1e-12, rtol=1e-10)
        np.testing.assert_allclose(out[0, h], O.dense_causal_attention(
            Q[0, h], K[0, h // 2], V[0, h // 2], scale), atol=1e-12)
        # lse: log of the causal softmax denominator, by direct summation
        qf, kf = O.widen(Q[0, h]), O.widen(K[0, h // 2])
        lg = scale * qf @ kf.T
        lg[np.triu(np.ones((N, N), bool), 1)] = -np.inf
        np.testing.assert_allclose(lse[0, h], np.log(np.exp(lg).sum(axis=1)), rtol=1e-12)


def test_attend_permutation_invariant():
    rng = np.random.default_rng(9)
    N, d, tile_q, bk = 512, 16, 64, 32
    Q = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    K = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    V = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    s = O.block_scores(Q, K, tile_q, bk)
    r = O.select(s, tile_q, bk, 6, 6, 1, 0.25)
    kv = r["kv_idx"].copy()
    out1, _ = O.attend(Q, K, V, kv, tile_q, bk, 0.25)
    perm = kv.copy()
    for t in range(kv.shape[2]):
        c = r["kv_cnt"][0, 0, t]
        perm[0, 0, t, :c] = rng.permutation(kv[0, 0, t, :c])
    out2, _ = O.attend(Q, K, V, perm, tile_q, bk, 0.25)
    np.testing.assert_allclose(out1, out2, atol=1e-12)


def test_attend_sparse_matches_masked_dense():
    """A sparse row equals dense attention with the unselected blocks masked out."""
    rng = np.random.default_rng(10)
    N, d, tile_q, bk = 256, 16, 32, 32
    Q = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    K = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    V = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    s = O.block_scores(Q, K, tile_q, bk)
    r = O.select(s, tile_q, bk, 3, 3, 1, 0.25)
    out, _ = O.attend(Q, K, V, r["kv_idx"], tile_q, bk, 0.5)
    q = torch.from_numpy(Q[0, 0].astype(np.float64))
    k = torch.from_numpy(K[0, 0].astype(np.float64))
    v = torch.from_numpy(V[0, 0].astype(np.float64))
    mask = torch.zeros(N, N, dtype=torch.bool)
    for t in range(N // tile_q):
        for j in r["kv_idx"][0, 0, t]:
            if j >= 0:
                mask[t * tile_q:(t + 1) * tile_q, j * bk:(j + 1) * bk] = True
    mask &= torch.ones(N, N, dtype=torch.bool).tril()
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None, None], k[None, None], v[None, None], attn_mask=mask[None, None], scale=0.5)[0, 0]
    np.testing.assert_allclose(out[0, 0], ref.numpy(), atol=1e-12)


# ---------------------------------------------------------------------------
# decode: termination rule (hand-worked traces) and limits

def _load_art(golden_dir):
    cases, cur = [], None
    for line in open(os.path.join(golden_dir, "art_decision.txt")):
        if line.startswith("#") or not line.strip():
            continue
        p = line.split()
        if p[0] == "case":
            cur = dict(name=p[1], tau=float(p[2]), phi=float(p[3]), p=int(p[4]),
                       exp=int(p[5]), x=[])
            cases.append(cur)
        else:
            cur["x"].append([float(v) for v in p[1:]])
    return cases


def test_termination_golden(golden_dir):
    cases = _load_art(golden_dir)
    assert len(cases) == 7
    for c in cases:
        tr = np.array(c["x"], np.float32)
        assert O.termination_block(tr, c["tau"], c["phi"], c["p"]) == c["exp"], c["name"]


def test_probe_step_values():
    ds, dd = O.probe_step([3.0, 4.0], [6.0, 8.0])
    assert ds == 5.0 and abs(dd) < 1e-15
    ds, dd = O.probe_step([1.0, 0.0], [0.0, 2.0])
    assert ds == 1.0 and dd == 1.0
    ds, dd = O.probe_step([1.0, 0.0], [-1.0, 0.0])
    assert ds == 0.0 and dd == 2.0


def test_pairwise_sum64_order_and_bound():
    """The probe sums follow the stated pairwise order. Worked by hand: with terms
    1 (index 0), 2^-53 (index 1) and 2^-53 (index 33), index 1 and index 33 meet
    first (2^-52, exact) and the last step gives 1 + 2^-52, while a left-to-right sum
    rounds each 2^-53 away (ties to even) and returns 1."""
    t = np.zeros(34)
    t[0], t[1], t[33] = 1.0, 2.0 ** -53, 2.0 ** -53
    assert O.pairwise_sum64(t) == 1.0 + 2.0 ** -52
    left = 0.0
    for v in t:
        left += v
    assert left == 1.0
    # index 0 with index 32 first: 1 + 2^-53 rounds to 1 there
    t = np.zeros(64)
    t[0], t[32], t[1] = 1.0, 2.0 ** -53, 2.0 ** -53
    assert O.pairwise_sum64(t) == 1.0
    # exact rational sums: a tree of depth 6 is within 6 u sum|t| of the exact value,
    # and exact when every partial sum is representable (small integers)
    from fractions import Fraction
    rng = np.random.default_rng(3)
    for n in (1, 2, 31, 32, 33, 64):
        x = rng.standard_normal(n).astype(np.float32).astype(np.float64)
        terms = x * x
        exact = sum(Fraction(float(v)) for v in terms)
        got = O.pairwise_sum64(terms)
        bound = 6 * 2.0 ** -53 * float(sum(abs(Fraction(float(v))) for v in terms)) * 1.0001
        assert abs(Fraction(got) - exact) <= Fraction(bound), n
        ints = rng.integers(-1000, 1000, size=n).astype(np.float64)
        assert O.pairwise_sum64(ints) == float(ints.sum())


def test_probe_step_matches_exact_arithmetic():
    """d_scale and d_direction from random fp32 probes against the same quantities
    in exact rational arithmetic (the roots and the quotient within a few units of
    fp64 rounding)."""
    from fractions import Fraction
    rng = np.random.default_rng(4)
    for n in (1, 7, 32, 64):
        a = rng.standard_normal(n).astype(np.float32)
        b = (a + 0.01 * rng.standard_normal(n)).astype(np.float32)
        ds, dd = O.probe_step(a, b)
        sa = sum(Fraction(float(v)) ** 2 for v in a)
        sb = sum(Fraction(float(v)) ** 2 for v in b)
        dot = sum(Fraction(float(u)) * Fraction(float(v)) for u, v in zip(a, b))
        na, nb = math.sqrt(float(sa)), math.sqrt(float(sb))
        assert abs(ds - abs(nb - na)) <= 1e-14 * max(na, nb)
        assert abs(dd - (1 - float(dot) / (na * nb))) <= 1e-14


def _decode_case(seed=11, L=2048, d=128, G=4, bkv=128):
    rng = np.random.default_rng(seed)
    q = S.f32_to_bf16_bits(rng.standard_normal((G, d)).astype(np.float32))
    Kc = S.f32_to_bf16_bits(rng.standard_normal((L, d)).astype(np.float32))
    Vc = S.f32_to_bf16_bits(rng.standard_normal((L, d)).astype(np.float32))
    return q, Kc, Vc


def test_decode_no_termination_is_dense():
    q, Kc, Vc = _decode_case()
    dims = S.default_probe_dims(32)
    scale = 1 / math.sqrt(128)
    o, used, tr = O.decode_group(q, Kc, Vc, 128, scale, 0.0, 0.0, 1, dims)
    assert used == 16 and tr.shape == (16, 32)
    qq = torch.from_numpy(O.widen(q))[None, :, None, :]
    kk = torch.from_numpy(O.widen(Kc))[None, None].expand(1, 4, -1, -1)
    vv = torch.from_numpy(O.widen(Vc))[None, None].expand(1, 4, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)[0, :, 0]
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)


@pytest.mark.parametrize("p", [1, 2, 5])
def test_decode_infinite_thresholds_stop_after_p_plus_one(p):
    q, Kc, Vc = _decode_case()
    o, used, tr = O.decode_group(q, Kc, Vc, 128, 0.125, np.inf, np.inf, p, S.default_probe_dims())
    assert used == p + 1
    # the output is attention over exactly the first used*128 keys
    n = used * 128
    qq = torch.from_numpy(O.widen(q))[None, :, None, :]
    kk = torch.from_numpy(O.widen(Kc[:n]))[None, None].expand(1, 4, -1, -1)
    vv = torch.from_numpy(O.widen(Vc[:n]))[None, None].expand(1, 4, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=0.125)[0, :, 0]
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)


def test_decode_planted_convergence():
    """Keys of block 0 align with the query (huge logits), later keys point
    away: the output is fixed after block 0, so the first test (t = 1) is
    stable and streaming stops with 2 blocks."""
    q, Kc, Vc = _decode_case()
    qf = O.widen(q)[0]
    Kf = np.tile(-qf, (2048, 1))
    Kf[:128] = 4 * qf
    Kb = S.f32_to_bf16_bits(Kf.astype(np.float32))
    qb = np.tile(q[0], (4, 1))
    o, used, tr = O.decode_group(qb, Kb, Vc, 128, 0.125, 1e-3, 1e-4, 1, S.default_probe_dims())
    assert used == 2


def _small_prefill(seed, N=512, d=16, Hq=2, Hkv=1):
    rng = np.random.default_rng(seed)
    Q = S.f32_to_bf16_bits(rng.standard_normal((1, Hq, N, d)).astype(np.float32))
    K = S.f32_to_bf16_bits(rng.standard_normal((1, Hkv, N, d)).astype(np.float32))
    V = S.f32_to_bf16_bits((rng.standard_normal((1, Hkv, N, d)) * 1.5).astype(np.float32))
    return Q, K, V


def test_bounds_score_is_max_over_box_corners():
    """sum_c max(q_c kmin_c, q_c kmax_c) is the maximum of q . x over the corners of
    the block's bounding box: brute force over all 2^d corners for d = 4."""
    rng = np.random.default_rng(7)
    K = S.f32_to_bf16_bits(rng.standard_normal((1, 1, 256, 4)).astype(np.float32))
    Q = S.f32_to_bf16_bits(rng.standard_normal((1, 1, 256, 4)).astype(np.float32))
    s = O.block_scores(Q, K, 64, 32, kind="bounds")
    kmin, kmax = O.key_block_bounds(K[0, 0], 32)
    corners = np.array(np.meshgrid(*[[0, 1]] * 4, indexing="ij")).reshape(4, -1).T   # [16, 4]
    Qf = O.widen(Q[0, 0])
    for t in range(4):
        J = (t + 1) * 2 - 1
        for j in range(J + 1):
            box = np.where(corners == 1, kmax[j], kmin[j])                 # [16, 4]
            ref = (Qf[t * 64:(t + 1) * 64] @ box.T).max()
            assert abs(float(s[0, 0, t, j]) - ref) <= 1e-6 * max(1.0, abs(ref))
        assert np.isneginf(s[0, 0, t, J + 1:]).all()


def test_bounds_score_bounds_every_key_and_is_exact_for_constant_blocks():
    Q, K, _ = _small_prefill(8)
    s = O.block_scores(Q, K, 64, 32, kind="bounds")
    m = O.block_scores(Q, K, 64, 32, kind="mean")
    Qf, Kf = O.widen(Q[0, 0]), O.widen(K[0, 0])
    for t in range(8):
        J = 2 * t + 1
        dots = Qf[t * 64:(t + 1) * 64] @ Kf[:(J + 1) * 32].T              # every key
        true_max = dots.reshape(64, J + 1, 32).max(axis=(0, 2))
        assert (s[0, 0, t, :J + 1] >= true_max.astype(np.float32) - 1e-5).all()
        assert (s[0, 0, t, :J + 1] >= m[0, 0, t, :J + 1] - 1e-5).all()
    # a block whose keys are all equal: the bound is the exact tile max of q . k
    Kc = K.copy()
    Kc[0, 0, 64:96] = Kc[0, 0, 64]
    s2 = O.block_scores(Q, Kc, 64, 32, kind="bounds")
    m2 = O.block_scores(Q, Kc, 64, 32, kind="mean")
    assert s2[0, 1, 3, 2] == m2[0, 1, 3, 2]


def test_additive_value_term_closed_forms():
    Q, K, V = _small_prefill(9)
    m = O.block_scores(Q, K, 64, 32, kind="mean")
    assert np.array_equal(O.block_scores(Q, K, 64, 32, V=V, kind="vlog", beta=0.0), m)
    # block 5: every V row equals a vector of squared norm e^2 -> ln = 2 -> term = 2 beta
    Vc = O.widen(V).copy()
    u = np.zeros(16)
    u[3] = math.e
    Vc[0, 0, 160:192] = u
    term = O.value_log_term(Vc[0, 0], 32, 0.75)
    assert abs(term[5] - 1.5) < 1e-12
    # a block whose mean value vector has squared norm below 1 contributes nothing
    Vc[0, 0, 192:224] = 0.5 * np.ones(16) / 4.0
    assert O.value_log_term(Vc[0, 0], 32, 0.75)[6] == 0.0
    Vc[0, 0, 224:256] = 0.0
    assert O.value_log_term(Vc[0, 0], 32, 0.75)[7] == 0.0
    s = O.block_scores(Q, K, 64, 32, V=Vc, kind="vlog", beta=0.75)
    np.testing.assert_allclose(s[0, :, 3, 5], (m[0, :, 3, 5].astype(np.float64) + 1.5), rtol=1e-6)
    assert np.array_equal(s[0, :, 3, 6], m[0, :, 3, 6]) and np.array_equal(s[0, :, 3, 7], m[0, :, 3, 7])


def _vs_case(seed=21, N=256, d=16):
    rng = np.random.default_rng(seed)
    Q = S.f32_to_bf16_bits(rng.standard_normal((1, 2, N, d)).astype(np.float32))
    K = S.f32_to_bf16_bits(rng.standard_normal((1, 1, N, d)).astype(np.float32))
    V = S.f32_to_bf16_bits(rng.standard_normal((1, 1, N, d)).astype(np.float32))
    return Q, K, V


def _vs_lists(v, s, Hq=2):
    vi = np.array([v] * Hq, np.int32)[None]
    so = np.array([s] * Hq, np.int32)[None]
    return vi, np.full((1, Hq), vi.shape[-1], np.int32), so, np.full((1, Hq), so.shape[-1], np.int32)


def test_vs_every_diagonal_or_every_column_is_dense_causal():
    Q, K, V = _vs_case()
    N = 256
    dense = O.dense_causal_attention(Q[0, 1], K[0, 0], V[0, 0], 0.25)
    for v, s in ([[], list(range(N))], [list(range(N)), []], [list(range(N)), list(range(N))]):
        vi, vc, so, sc = _vs_lists(v if v else [0], s if s else [0])
        if not v:
            vc[:] = 0
        if not s:
            sc[:] = 0
        o, lse = O.attend_vs(Q, K, V, vi, vc, so, sc, 0.25)
        np.testing.assert_allclose(o[0, 1], dense, atol=1e-12)   # union: no key counted twice


def test_vs_single_diagonal_returns_own_value():
    """S = {0}, no vertical columns: each row attends only to itself, O_i = v_i."""
    Q, K, V = _vs_case()
    vi, vc, so, sc = _vs_lists([0], [0])
    vc[:] = 0
    o, lse = O.attend_vs(Q, K, V, vi, vc, so, sc, 0.25)
    np.testing.assert_array_equal(o[0, 0], O.widen(V[0, 0]))
    np.testing.assert_allclose(lse[0, 0], 0.25 * np.einsum("nd,nd->n", O.widen(Q[0, 0]), O.widen(K[0, 0])),
                               atol=1e-12)


def test_vs_random_sets_match_masked_sdpa():
    """Random vertical columns and slash offsets (with duplicates, out-of-range entries and
    entries past the counts), two query heads per KV head: the oracle equals torch's fp64
    scaled_dot_product_attention under the boolean mask (j <= i and j a column) or (i - j an
    offset), built here pair by pair; its lse equals the masked logsumexp, and exactly the
    rows with an empty mask row come out 0 / -inf."""
    rng = np.random.default_rng(33)
    B, Hq, Hkv, N, d = 1, 4, 2, 96, 16
    Q = S.f32_to_bf16_bits(rng.standard_normal((B, Hq, N, d)).astype(np.float32))
    K = S.f32_to_bf16_bits(rng.standard_normal((B, Hkv, N, d)).astype(np.float32))
    V = S.f32_to_bf16_bits(rng.standard_normal((B, Hkv, N, d)).astype(np.float32))
    Wv, Ws = 12, 9
    v_idx = rng.integers(-5, N + 5, size=(B, Hq, Wv)).astype(np.int32)
    s_off = rng.integers(-3, N + 3, size=(B, Hq, Ws)).astype(np.int32)
    v_idx[0, 0, :3] = [40, 40, 7]                      # duplicates count once
    s_off[0, 0, :2] = [5, 5]
    v_cnt = np.array([[Wv, 7, 0, 12]], np.int32)
    s_cnt = np.array([[Ws, 0, 4, 9]], np.int32)
    scale = 0.3
    o, lse = O.attend_vs(Q, K, V, v_idx, v_cnt, s_off, s_cnt, scale)
    for h in range(Hq):
        cols = {int(j) for j in v_idx[0, h, :v_cnt[0, h]] if 0 <= j < N}
        offs = {int(x) for x in s_off[0, h, :s_cnt[0, h]] if 0 <= x < N}
        mask = np.zeros((N, N), bool)
        for i in range(N):
            for j in range(i + 1):
                mask[i, j] = j in cols or (i - j) in offs
        q = torch.from_numpy(O.widen(Q[0, h]))
        k = torch.from_numpy(O.widen(K[0, h // 2]))
        v = torch.from_numpy(O.widen(V[0, h // 2]))
        m = torch.from_numpy(mask)
        live = mask.any(axis=1)
        ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=m[None],
                                                               scale=scale)[0].numpy()
        np.testing.assert_allclose(o[0, h, live], ref[live], rtol=0, atol=1e-12)
        lg = (scale * (q @ k.T)).masked_fill(~m, float("-inf"))
        np.testing.assert_allclose(lse[0, h, live], torch.logsumexp(lg, dim=1).numpy()[live], rtol=0, atol=1e-12)
        assert not o[0, h, ~live].any() and np.isneginf(lse[0, h, ~live]).all()
        assert live.sum() > N // 4


def test_vs_key_sets_and_empty_rows():
    assert list(O.vs_keys(10, [0, 3, 11, 40], [0, 2, 10, 20])) == [0, 3, 8, 10]
    assert list(O.vs_keys(1, [5], [4])) == []
    Q, K, V = _vs_case()
    vi, vc, so, sc = _vs_lists([100], [64])
    o, lse = O.attend_vs(Q, K, V, vi, vc, so, sc, 0.25)
    assert not o[0, 0, :64].any() and np.isneginf(lse[0, 0, :64]).all()     # nothing visible yet
    np.testing.assert_array_equal(o[0, 0, 64], O.widen(V[0, 0, 0]))      # only key 0 = 64 - 64
    # rows 100..163: key 100 and key i - 64 (distinct) -> a two-key softmax
    i = 120
    ks = [56, 100]
    lg = 0.25 * (O.widen(K[0, 0, ks]) @ O.widen(Q[0, 0, i]))
    p = np.exp(lg - lg.max())
    np.testing.assert_allclose(o[0, 0, i], (p @ O.widen(V[0, 0, ks])) / p.sum(), atol=1e-12)


def test_decode_list_in_order_matches_decode():
    """Visiting blocks 0, 1, ... through the list form gives the in-order decode."""
    q, Kc, Vc = _decode_case()
    dims = S.default_probe_dims(32)
    for tau, phi in [(1e-3, 1e-4), (0.0, 0.0), (np.inf, np.inf)]:
        a = O.decode_group(q, Kc, Vc, 128, 0.125, tau, phi, 1, dims)
        b = O.decode_group_list(q, Kc, Vc, 128, 0.125, range(16), tau, phi, 1, dims)
        assert a[1] == b[1]
        np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-13)
        np.testing.assert_array_equal(a[2], b[2])


def _sdpa_over_blocks(q, Kc, Vc, blocks, scale):
    rows = np.concatenate([np.arange(j * 128, (j + 1) * 128) for j in blocks])
    qq = torch.from_numpy(O.widen(q))[None, :, None, :]
    kk = torch.from_numpy(O.widen(Kc)[rows])[None, None].expand(1, q.shape[0], -1, -1)
    vv = torch.from_numpy(O.widen(Vc)[rows])[None, None].expand(1, q.shape[0], -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)[0, :, 0].numpy()


def test_decode_list_full_pass_is_attention_over_listed_blocks():
    """With tau = phi = 0 nothing is stable: the output is textbook attention over
    the keys of the listed blocks, whatever their order ([ART] 2.4)."""
    q, Kc, Vc = _decode_case()
    dims = S.default_probe_dims(32)
    blocks = [0, 13, 7, 2, 9]
    o, used, tr = O.decode_group_list(q, Kc, Vc, 128, 0.125, blocks, 0.0, 0.0, 1, dims)
    assert used == 5 and tr.shape == (5, 32)
    np.testing.assert_allclose(o, _sdpa_over_blocks(q, Kc, Vc, blocks, 0.125), atol=1e-12)
    o2, _, _ = O.decode_group_list(q, Kc, Vc, 128, 0.125, [9, 2, 0, 13, 7], 0.0, 0.0, 1, dims)
    np.testing.assert_allclose(o, o2, atol=1e-13)


@pytest.mark.parametrize("p", [1, 3])
def test_decode_list_infinite_thresholds(p):
    """tau = phi = inf: every test passes, so the visit stops after p + 1 listed blocks
    and the output is attention over exactly those."""
    q, Kc, Vc = _decode_case()
    blocks = [0, 15, 14, 3, 8, 1]
    o, used, tr = O.decode_group_list(q, Kc, Vc, 128, 0.125, blocks, np.inf, np.inf, p,
                                      S.default_probe_dims())
    assert used == p + 1
    np.testing.assert_allclose(o, _sdpa_over_blocks(q, Kc, Vc, blocks[:p + 1], 0.125), atol=1e-12)


def test_decode_list_planted_first_block():
    """The first listed block dominates (its keys align with the query): the
    output is fixed after it, so the first test is stable and 2 steps are used."""
    q, Kc, Vc = _decode_case()
    qf = O.widen(q)[0]
    Kf = np.tile(-qf, (2048, 1))
    Kf[5 * 128:6 * 128] = 4 * qf
    Kb = S.f32_to_bf16_bits(Kf.astype(np.float32))
    qb = np.tile(q[0], (4, 1))
    _, used, _ = O.decode_group_list(qb, Kb, Vc, 128, 0.125, [5, 0, 1, 2], 1e-3, 1e-4, 1,
                                     S.default_probe_dims())
    assert used == 2
    _, used, _ = O.decode_group_list(qb, Kb, Vc, 128, 0.125, [0, 1, 5, 2], 1e-3, 1e-4, 1,
                                     S.default_probe_dims())
    assert used > 2


def test_decode_list_empty():
    q, Kc, Vc = _decode_case()
    o, used, tr = O.decode_group_list(q, Kc, Vc, 128, 0.125, [], 1e-3, 1e-4, 1, S.default_probe_dims())
    assert used == 0 and tr.shape == (0, 32) and not o.any()


def test_decode_block_list_generator():
    d = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=2, L=4096)
    lists, cnt = S.decode_block_lists(d, 3, "recency")
    assert lists.shape == (2, 8, 32) and (cnt == 32).all()
    assert list(lists[1, 3]) == [0] + list(range(31, 0, -1))
    lists, cnt = S.decode_block_lists(d, 3, "subset", keep=9)
    assert lists.shape == (2, 8, 9) and (lists[:, :, 0] == 0).all()
    for row in lists.reshape(-1, 9):
        assert len(set(row)) == 9 and (np.diff(row[1:]) < 0).all() and row[1:].min() >= 1


def test_vs_index_generator():
    """Synthetic vertical-slash indices: distinct, in range, the KV head's planted anchors and the
    first four positions among the vertical columns, the local band among the slash offsets."""
    spec = S.WORKLOADS["prefill_32k_vs"].scaled(N=4096, Hq=4, Hkv=2)
    v, vc, so, sc = S.vs_indices(spec, 11, n_vertical=24, n_slash=20, n_local=8)
    assert v.shape == (1, 4, 24) and so.shape == (1, 4, 20)
    assert (vc == 24).all() and (sc == 20).all()
    for h in range(4):
        assert len(set(v[0, h])) == 24 and len(set(so[0, h])) == 20
        assert v[0, h].min() >= 0 and v[0, h].max() < 4096 and so[0, h].min() >= 0 and so[0, h].max() < 4096
        anchors = set(int(x) for x in S._vertical_positions(spec, 11, 0, h // 2))
        assert anchors | {0, 1, 2, 3} <= set(int(x) for x in v[0, h])
        assert set(range(8)) <= set(int(x) for x in so[0, h])


def test_generator_structure():
    """The seeded generators plant the stated structure (not method arithmetic)."""
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=4096, Hq=4, Hkv=1)
    k = S.prefill_head(spec, 1002, "k", 0, 0).reshape(-1, 64, 128)
    twins = sum(np.array_equal(k[2 * m], k[2 * m + 1]) for m in range(32))
    near = sum((k[2 * m] != k[2 * m + 1]).sum() == 1 for m in range(32))
    assert twins + near >= 3
    d = S.DECODE_WORKLOADS["decode_art_64k"].scaled(L=8192)
    kk = S.bf16_bits_to_f32(S.decode_head(d, 1004, "k", 0, 0))
    assert 1.6 < kk[:4096].std() / kk[4096:].std() < 2.4
    a = S.prefill_head(spec, 5, "q", 0, 3)
    b = S.prefill_head(spec, 5, "q", 0, 3)
    assert np.array_equal(a, b)


def test_attend_empty_rows():
    """Rows that see no listed key (a caller-made list without the tile's own
    block) get output 0 and lse -inf; rows that do see keys are unaffected."""
    rng = np.random.default_rng(12)
    N, d, tile_q, bk = 256, 8, 64, 64
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = rng.standard_normal((N, d)).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    # tile 1 (rows 64..127) lists only block 1: every row sees keys 64..row
    o, l = O.attend_tile(Q[64:128], K, V, np.array([1, -1]), 64, bk, 0.3)
    assert np.isfinite(l).all()
    # tile 0 listing nothing at all
    o, l = O.attend_tile(Q[0:64], K, V, np.array([-1, -1]), 0, bk, 0.3)
    assert (o == 0).all() and np.isneginf(l).all()
    # tile 1 listing only block 2, which is after every row of the tile
    o, l = O.attend_tile(Q[64:128], K, V, np.array([2]), 64, bk, 0.3)
    assert (o == 0).all() and np.isneginf(l).all()


def test_gated_workload_near_tie_fraction():
    """The 128k gated workload is drawn so that about a fifth of the (head, cut
    tile) pairs have a gap below 1e-3 between the last kept and the first dropped
    candidate score (oracle scores; every 4th tile of all 32 heads)."""
    spec = S.WORKLOADS["gated_prefill_128k"]
    G = spec.Hq // spec.Hkv
    near = tot = 0
    for g in range(spec.Hkv):
        kb = O.pool_keys(S.prefill_head(spec, 1003, "k", 0, g), spec.block_k)
        for h in range(g * G, (g + 1) * G):
            q = S.prefill_head(spec, 1003, "q", 0, h)
            for t in range(1 + (h % 4), spec.n_qt, 4):
                nF, nc, m, M = O.tile_slots(t, spec.n_qt, spec.tile_q, spec.block_k, 64, 64, 2)
                if not nc > m >= 1:
                    continue
                s = O.score_tile(q[t * 128:(t + 1) * 128], kb, O.tile_blocks(t, 128, 64)[1])
                o = O.rank_candidates(s, nc)
                near += float(s[o[m - 1]]) - float(s[o[m]]) < 1e-3
                tot += 1
    assert 0.15 <= near / tot <= 0.25, near / tot


# ---------------------------------------------------------------------------
# bf16 storage: the oracle's widening and the generator's rounding, each against
# an implementation that shares nothing with it

def _bf16_value(bits: int) -> float:
    """A bf16 bit pattern's value from its fields (sign, 8-bit exponent, 7-bit
    fraction), written out for a handful of fixed cases."""
    sign = -1.0 if bits & 0x8000 else 1.0
    e, f = (bits >> 7) & 0xFF, bits & 0x7F
    if e == 0xFF:
        return sign * math.inf
    if e == 0:
        return sign * f * 2.0 ** -133               # subnormal: f * 2^(1 - 127 - 7)
    return sign * (1.0 + f / 128.0) * 2.0 ** (e - 127)


def test_widen_bf16_every_pattern_matches_torch():
    """Every non-NaN bf16 pattern widens to the value torch's bfloat16 holds."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    nan = ((bits & 0x7F80) == 0x7F80) & ((bits & 0x7F) != 0)
    bits = bits[~nan]
    ours = O.widen(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert ours.dtype == np.float64
    np.testing.assert_array_equal(ours, ref)
    # the sign of zero survives too
    assert np.array_equal(np.signbit(ours), np.signbit(ref))


@pytest.mark.parametrize("bits", [0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x0080, 0x3F80, 0xBF80,
                                  0x4000, 0xC000, 0x3F81, 0x4049, 0x7F7F, 0xFF7F, 0x7F80, 0xFF80])
def test_widen_bf16_special_values(bits):
    """+-0, the smallest and largest subnormals, the smallest normal, +-1, +-2, 1 + 2^-7,
    3.140625, the largest finite values and the infinities, from their fields."""
    got = float(O.widen(np.array([bits], np.uint16))[0])
    exp = _bf16_value(bits)
    assert got == exp and math.copysign(1.0, got) == math.copysign(1.0, exp)


def test_generator_rounding_matches_torch():
    """The generator's float32 -> bf16 rounding (nearest, ties to even) against
    torch's conversion: random values over the whole exponent range, subnormals,
    values that round up to infinity, and exact ties with even and odd upper halves."""
    rng = np.random.default_rng(11)
    u = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    x = u.view(np.float32)
    x = x[np.isfinite(x)]
    hi = rng.integers(0, 1 << 16, size=4096, dtype=np.uint32)
    hi = hi[((hi & 0x7F80) != 0x7F80)]
    ties = ((hi << 16) | 0x8000).astype(np.uint32).view(np.float32)           # exactly halfway
    near = np.concatenate([((hi << 16) | 0x7FFF), ((hi << 16) | 0x8001)]).astype(np.uint32).view(np.float32)
    extra = np.array([0.0, -0.0, 1e-45, -1e-45, 1.17549435e-38, 3.4028235e38, -3.4028235e38,
                      np.float32(np.inf), -np.float32(np.inf), 1.0, -1.0, 1.00390625, 1.01171875],
                     np.float32)
    for arr in (x, ties, near, extra):
        ours = S.f32_to_bf16_bits(arr)
        ref = torch.from_numpy(np.ascontiguousarray(arr)).to(torch.bfloat16).view(torch.int16).numpy()
        np.testing.assert_array_equal(ours.view(np.int16), ref)
    # ties go to the even neighbour: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert S.f32_to_bf16_bits(np.array([1.00390625], np.float32))[0] == 0x3F80
    assert S.f32_to_bf16_bits(np.array([1.01171875], np.float32))[0] == 0x3F82


def test_decode_list_skips_entries_outside_the_cache():
    """Entries outside [0, L/block_kv) are not visit steps: a list holding -7, one
    past the last block and valid blocks gives what the valid blocks alone give,
    and a full pass is textbook attention over exactly those blocks."""
    q, Kc, Vc = _decode_case()
    dims = S.default_probe_dims(32)
    nb = Kc.shape[0] // 128
    raw = [3, -7, 11, nb, 0, nb + 40, 6]
    valid = [3, 11, 0, 6]
    assert O.decode_visit_steps(raw, nb) == valid
    for tau, phi in [(0.0, 0.0), (1e-3, 1e-4), (np.inf, np.inf)]:
        a = O.decode_group_list(q, Kc, Vc, 128, 0.125, raw, tau, phi, 1, dims)
        b = O.decode_group_list(q, Kc, Vc, 128, 0.125, valid, tau, phi, 1, dims)
        assert a[1] == b[1]
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[2], b[2])
    o, used, _ = O.decode_group_list(q, Kc, Vc, 128, 0.125, raw, 0.0, 0.0, 1, dims)
    assert used == 4
    np.testing.assert_allclose(o, _sdpa_over_blocks(q, Kc, Vc, valid, 0.125), atol=1e-12)
    # only bad entries: nothing to visit
    o, used, tr = O.decode_group_list(q, Kc, Vc, 128, 0.125, [-1, nb], 0.0, 0.0, 1, dims)
    assert used == 0 and tr.shape == (0, 32) and not o.any()


def test_decode_list_counts_are_clamped():
    """list_cnt outside [0, W] is clamped: a negative count visits nothing, a count
    above the width visits the whole row."""
    q, Kc, Vc = _decode_case()
    dims = S.default_probe_dims(32)
    qq = np.stack([np.tile(q, (1, 1))])                   # [1, G, d]
    lists = np.array([[[0, 5, 9]]], np.int32)
    _, used, _ = O.decode_list(qq, Kc[None, None], Vc[None, None], 128, 0.125, lists,
                               np.array([[-3]]), 0.0, 0.0, 1, dims)
    assert used[0, 0] == 0
    _, used, _ = O.decode_list(qq, Kc[None, None], Vc[None, None], 128, 0.125, lists,
                               np.array([[17]]), 0.0, 0.0, 1, dims)
    assert used[0, 0] == 3
