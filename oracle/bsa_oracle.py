"""CPU oracle for block-sparse causal attention: plain, slow, fp64.

TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import or run this module. The product path
(the CUDA library and its binding) never calls it, and it imports nothing
from the product.

Sources (summary pages, cited by title and section):

* [UGS] "Resumo Técnico: Seleção com Portão de Incerteza para Atenção de
  Esparsidade em Blocos" -- Metodologia steps 1-5 (block scoring backbone,
  per-tile top-k with the tile's max over rows, the normalised cut margin
  sigma, head mean + per-layer quantile trigger, rho*k expansion with
  sentinel-padded kv_idx).
* [Stem] "Stem: Rethinking Causal Information Flow in Sparse Attention" --
  Resumo técnico, 2. Metodologia, A (Token Position-Decay budget), B
  (Output-Aware Metric) and "Implementação" (block downsampling, dynamic
  budget, sparse aggregation).
* [ART] "Resumo Técnico: ART (Attention Run-time Termination)" -- 2.1
  (tile-wise streaming exposes the partial output O^(t)), 2.2 (probe vector,
  d_scale and d_direction against tau and phi), 2.3 (patience p), 2.4
  (block 0 always evaluated).
* [VSP] "VSPrefill: Vertical-Slash Sparse Attention with Lightweight
  Indexing for Long-Context Prefilling" -- 2. Metodologia A (vertical
  columns and slash diagonals), B.3 (a fused kernel attends over the merged
  vertical and diagonal indices).

Conventions: inputs are bf16 values widened exactly to fp64 (or fp32 values
widened); arithmetic is fp64 unless a step says fp32. Layouts: Q [B,Hq,N,d],
K and V [B,Hkv,N,d]; query head h reads KV head h // (Hq // Hkv).

Readings taken where the pages are silent (each is also listed in the design
notes): no 1/sqrt(d) factor in block scores; the tile max runs over all rows
of the tile, unmasked; the blocks that intersect the tile's own rows are
always kept and count toward k; ties in the ranking go to the lower block
index; sigma of a non-cut tile is 1; the quantile is the linear-interpolation
empirical quantile over the cut tiles of the call; the trigger compares
strictly (sigma_bar < theta) and is shared by all heads of a (batch, tile);
the sentinel is -1. For decode: the probe is a fixed set of coordinates of the
first query head of the KV group; d_scale is the absolute difference of the
probe norms; d_direction is 1 - cosine, taken as 1 when a norm is zero;
termination is decided per (batch, KV head).

Readings for the added paths: the additive Output-Aware Metric is taken at
block level (the block's mean value vector for V_j, natural log, weight beta,
no 1/sqrt(d) on the score); the K-min/K-max score is the tile max of
sum_c max(q_c kmin_c, q_c kmax_c); a vertical-slash row attends to the union,
each key once, of its vertical columns j <= i and the keys i - o of its slash
offsets; a decode over a block list visits the list in order, skips entries
outside the cache (they are not visit steps) and never tests its first visit.

bf16 inputs: ``widen`` reads a uint16 array as bf16 bit patterns (the upper
half of a float32), exact in fp64; it is pinned over all 65,536 patterns
against torch's own bfloat16 type and against hand-computed values.

Parity status: every function below is pinned by CPU tests against closed
forms, library routines (torch scaled_dot_product_attention, numpy.quantile)
or brute force (the K-min/K-max score against the maximum over all 2^d box
corners) -- except the exact termination block on random decode data, which
the pages do not fix ("parity unpinned" for that value; the decision rule
itself is pinned by hand-worked traces).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

NEG_INF32 = np.float32(-np.inf)


def widen(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) or float32 values -> float64, exactly."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# tile geometry and budget

def tile_blocks(t: int, tile_q: int, block_k: int):
    """Key blocks touched by query tile t.

    Returns (f_lo, J): the forced blocks are f_lo..J (the blocks that
    intersect the tile's own rows, J = the block of the tile's last row) and
    the scored candidates are 0..f_lo-1. [UGS step 2] selects per query tile;
    keeping the diagonal block is the causal self-visibility rule.
    """
    f_lo = (t * tile_q) // block_k
    J = ((t + 1) * tile_q - 1) // block_k
    return f_lo, J


def budget_k(t: int, n_qt: int, k_first: int, k_last: int) -> int:
    """Per-tile budget k_t. [Stem, 2.A, TPD]: linear decay from the first to the
    last tile, k_t = k_first - floor((k_first - k_last) * t / (n_qt - 1));
    with k_first == k_last this is the fixed top-k of [UGS step 2]."""
    if n_qt <= 1 or k_first == k_last:
        return k_first
    return k_first - ((k_first - k_last) * t) // (n_qt - 1)


def tile_slots(t: int, n_qt: int, tile_q: int, block_k: int,
               k_first: int, k_last: int, rho: int):
    """(n_forced, n_cand, m_t, M_t): forced block count, candidate count,
    scored slots at the base budget and at the rho-expanded budget
    [UGS step 5: top-rho*k instead of top-k], both capped at the J_t+1 blocks
    the tile can see and never below the forced blocks."""
    f_lo, J = tile_blocks(t, tile_q, block_k)
    nF = J - f_lo + 1
    k = budget_k(t, n_qt, k_first, k_last)
    K = max(nF, min(k, J + 1))
    KM = max(nF, min(rho * k, J + 1))
    return nF, f_lo, K - nF, KM - nF


def kv_idx_width(N: int, tile_q: int, block_k: int, k_first: int, k_last: int, rho: int) -> int:
    """Uniform kv_idx row width W (data independent), [UGS step 5 uniform dispatch shape]."""
    n_kb = N // block_k
    f_max = max(1, tile_q // block_k)      # most forced blocks any tile has
    return min(n_kb, max(rho * max(k_first, k_last), f_max))


# ---------------------------------------------------------------------------
# a1/a2: pooling and block scores

def pool_keys(K: np.ndarray, block_k: int) -> np.ndarray:
    """K_bar[..., j, :] = mean of the block_k keys of block j ([UGS step 1],
    mean-pooled keys; [Stem, Implementação] block downsampling). fp64."""
    K = widen(K)
    *lead, N, d = K.shape
    return K.reshape(*lead, N // block_k, block_k, d).mean(axis=-2)


def value_block_norm(V: np.ndarray, block_k: int) -> np.ndarray:
    """w[..., j] = || mean of the block's V rows ||_2 (output-aware block weight,
    motivated by [Stem, 2.B]: value magnitude enters the metric). fp64."""
    Vb = pool_keys(V, block_k)
    return np.sqrt((Vb * Vb).sum(axis=-1))


def score_tile(Q_tile: np.ndarray, Kbar: np.ndarray, J: int,
               w: Optional[np.ndarray] = None) -> np.ndarray:
    """One row of block scores for a query tile ([UGS step 2]: the tile's block
    score is the max over the tile's rows of q_i . K_bar_j).

    Q_tile [tile_q, d], Kbar [n_kb, d] (fp64). Blocks j > J are not visible
    to any row of the tile and score -inf. With w given (output-aware form),
    the max is multiplied by w_j in fp64 before rounding. Returns fp32.
    """
    Q_tile = widen(Q_tile)
    n_kb = Kbar.shape[0]
    out = np.full(n_kb, NEG_INF32, dtype=np.float32)
    dots = Q_tile @ Kbar[: J + 1].T            # [tile_q, J+1]
    s = dots.max(axis=0)
    if w is not None:
        s = s * w[: J + 1]
    out[: J + 1] = s.astype(np.float32)
    return out


def value_log_term(V: np.ndarray, block_k: int, beta: float) -> np.ndarray:
    """beta * max(0, ln ||mean of the block's V rows||^2): the value-magnitude term of
    [Stem, 2.B]'s additive Output-Aware Metric, taken at block level (the block's
    mean value vector stands for V_j). fp64; a zero mean vector gives 0."""
    Vb = pool_keys(V, block_k)
    e = (Vb * Vb).sum(axis=-1)
    with np.errstate(divide="ignore"):
        lg = np.log(e)
    return float(beta) * np.maximum(0.0, lg)


def key_block_bounds(K: np.ndarray, block_k: int):
    """(kmin, kmax)[..., j, :]: per-coordinate minimum and maximum over the keys of
    block j -- the K-min/K-max backbone named in [UGS, Metodologia] (per-coordinate
    upper bounds, Quest style). fp64."""
    K = widen(K)
    *lead, N, d = K.shape
    Kb = K.reshape(*lead, N // block_k, block_k, d)
    return Kb.min(axis=-2), Kb.max(axis=-2)


def score_tile_bounds(Q_tile: np.ndarray, kmin: np.ndarray, kmax: np.ndarray, J: int) -> np.ndarray:
    """One row of K-min/K-max block scores: s(t,j) = max over the tile's rows i of
    sum_c max(q_ic kmin_jc, q_ic kmax_jc). Each term is the largest value q_ic x
    takes for x in [kmin_jc, kmax_jc], so the sum bounds q_i . k from above for
    every key k of block j ([UGS, Metodologia] step 1, "limites superiores por
    coordenada"; step 2, max over the tile's rows). fp64, returned as fp32; -inf for
    j > J."""
    Q = widen(Q_tile)
    n_kb = kmin.shape[0]
    out = np.full(n_kb, NEG_INF32, dtype=np.float32)
    for j0 in range(0, J + 1, 32):
        j1 = min(J + 1, j0 + 32)
        a = Q[:, None, :] * kmin[None, j0:j1, :]
        b = Q[:, None, :] * kmax[None, j0:j1, :]
        out[j0:j1] = np.maximum(a, b).sum(axis=-1).max(axis=0).astype(np.float32)
    return out


def block_scores(Q: np.ndarray, K: np.ndarray, tile_q: int, block_k: int,
                 V: Optional[np.ndarray] = None, Hkv: Optional[int] = None,
                 kind: Optional[str] = None, beta: float = 0.0) -> np.ndarray:
    """scores [B, Hq, n_qt, n_kb] fp32.

    kind "mean": tile max of q . K_bar ([UGS] steps 1-2). "vnorm" (the default when
    V is given): that max times ||mean V_j||_2. "vlog": that max plus
    value_log_term (the additive form of [Stem, 2.B], weight beta). "bounds": the
    K-min/K-max score of score_tile_bounds."""
    if kind is None:
        kind = "vnorm" if V is not None else "mean"
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    n_qt, n_kb = N // tile_q, N // block_k
    out = np.empty((B, Hq, n_qt, n_kb), np.float32)
    for b in range(B):
        for g in range(Hkv):
            if kind == "bounds":
                kmin, kmax = key_block_bounds(K[b, g], block_k)
            else:
                Kbar = pool_keys(K[b, g], block_k)
            w = value_block_norm(V[b, g], block_k) if kind == "vnorm" else None
            add = value_log_term(V[b, g], block_k, beta) if kind == "vlog" else None
            for h in range(g * G, (g + 1) * G):
                Qh = widen(Q[b, h])
                for t in range(n_qt):
                    _, J = tile_blocks(t, tile_q, block_k)
                    Qt = Qh[t * tile_q:(t + 1) * tile_q]
                    if kind == "bounds":
                        out[b, h, t] = score_tile_bounds(Qt, kmin, kmax, J)
                    elif kind == "vlog":
                        Qt64 = widen(Qt)
                        row = np.full(n_kb, NEG_INF32, dtype=np.float32)
                        row[: J + 1] = ((Qt64 @ Kbar[: J + 1].T).max(axis=0) + add[: J + 1]).astype(np.float32)
                        out[b, h, t] = row
                    else:
                        out[b, h, t] = score_tile(Qt, Kbar, J, w)
    return out


# ---------------------------------------------------------------------------
# a4: ranking and the cut margin sigma

def rank_candidates(s_row: np.ndarray, n_cand: int) -> np.ndarray:
    """Candidate blocks 0..n_cand-1 ordered by (score descending, index
    ascending). Raises on a non-finite candidate score."""
    s = np.asarray(s_row[:n_cand], dtype=np.float32)
    if not np.all(np.isfinite(s)):
        raise ValueError("non-finite candidate score")
    idx = np.arange(n_cand)
    return np.lexsort((idx, -s)).astype(np.int64)


def cut_margin(s_row: np.ndarray, order: np.ndarray, m: int) -> np.float32:
    """sigma = (s_(m-1) - s_(m)) / (s_(0) - s_(m)) in fp32 ([UGS step 3]), with
    ranks 0-based over the ordered candidates; an all-tied head (0/0) gives 0."""
    s = np.asarray(s_row, dtype=np.float32)
    top, km1, km = s[order[0]], s[order[m - 1]], s[order[m]]
    num = np.float32(km1 - km)
    den = np.float32(top - km)
    if den == 0:
        return np.float32(0.0)
    return np.float32(num / den)


def select(scores: np.ndarray, tile_q: int, block_k: int, k_first: int, k_last: int,
           rho: int, gate_quantile: float, gate_threshold: float = float("nan")):
    """a3-a6: budget, ranking, sigma, gate and kv_idx for a whole layer call.

    scores [B, Hq, n_qt, n_kb] fp32. Returns a dict with kv_idx [B,Hq,n_qt,W]
    (ascending, -1 padded), kv_cnt, sigma [B,Hq,n_qt], sigma_bar [B,n_qt],
    trigger [B,n_qt] (uint8), theta (fp32 scalar, NaN when undefined), cut
    [n_qt] (bool) and W.
    """
    B, Hq, n_qt, n_kb = scores.shape
    N = n_kb * block_k
    W = kv_idx_width(N, tile_q, block_k, k_first, k_last, rho)
    sigma = np.ones((B, Hq, n_qt), np.float32)
    cut = np.zeros(n_qt, bool)
    ranked = {}
    slots = [tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho) for t in range(n_qt)]
    for t in range(n_qt):
        nF, n_cand, m, M = slots[t]
        cut[t] = n_cand > m >= 1
        for b in range(B):
            for h in range(Hq):
                order = rank_candidates(scores[b, h, t], n_cand)
                ranked[b, h, t] = order
                if cut[t]:
                    sigma[b, h, t] = cut_margin(scores[b, h, t], order, m)

    sigma_bar, theta, trigger = gate(sigma, cut, rho, gate_quantile, gate_threshold)

    kv_idx = np.full((B, Hq, n_qt, W), -1, np.int32)
    kv_cnt = np.zeros((B, Hq, n_qt), np.int32)
    for t in range(n_qt):
        nF, n_cand, m, M = slots[t]
        forced = np.arange(n_cand, n_cand + nF)
        for b in range(B):
            take = M if trigger[b, t] else m
            for h in range(Hq):
                sel = np.sort(np.concatenate([ranked[b, h, t][:take], forced]))
                kv_idx[b, h, t, : len(sel)] = sel
                kv_cnt[b, h, t] = len(sel)
    return dict(kv_idx=kv_idx, kv_cnt=kv_cnt, sigma=sigma, sigma_bar=sigma_bar,
                trigger=trigger, theta=theta, cut=cut, W=W)


# ---------------------------------------------------------------------------
# a5: gate

def head_mean(sigma: np.ndarray) -> np.ndarray:
    """sigma_bar[b, t] = (sum over heads in order h = 0..Hq-1, fp32) / Hq in fp32
    ([UGS step 4]: per-head sigma averaged into one signal per query tile)."""
    B, Hq, n_qt = sigma.shape
    acc = np.zeros((B, n_qt), np.float32)
    for h in range(Hq):
        acc = (acc + sigma[:, h, :]).astype(np.float32)
    return (acc / np.float32(Hq)).astype(np.float32)


def empirical_quantile(values: np.ndarray, q: float) -> np.float32:
    """Linear-interpolation empirical quantile with a fixed operation order:
    pos = q*(M-1) (fp64), lo = floor(pos), hi = min(lo+1, M-1),
    f = fp32(pos - lo), theta = v_lo + f*(v_hi - v_lo) with fp32 rounding
    after each operation. NaN for an empty population."""
    v = np.sort(np.asarray(values, dtype=np.float32))
    M = len(v)
    if M == 0:
        return np.float32(np.nan)
    pos = float(np.float32(q)) * (M - 1)
    lo = int(math.floor(pos))
    hi = min(lo + 1, M - 1)
    f = np.float32(pos - lo)
    diff = np.float32(v[hi] - v[lo])
    return np.float32(v[lo] + np.float32(f * diff))


def gate(sigma: np.ndarray, cut: np.ndarray, rho: int, q: float,
         fixed_threshold: float = float("nan")):
    """Head mean, per-layer quantile threshold theta over the cut tiles of the
    call, and trigger = cut and sigma_bar < theta ([UGS step 4]). With rho == 1
    nothing expands, so no trigger is raised and theta is NaN. A negative q
    selects a fixed, externally calibrated threshold instead."""
    sigma_bar = head_mean(sigma)
    B, n_qt = sigma_bar.shape
    trigger = np.zeros((B, n_qt), np.uint8)
    if rho <= 1:
        return sigma_bar, np.float32(np.nan), trigger
    if q < 0:
        theta = np.float32(fixed_threshold)
    else:
        theta = empirical_quantile(sigma_bar[:, cut].reshape(-1), q)
    trig = (sigma_bar < theta) & cut[None, :]
    return sigma_bar, theta, trig.astype(np.uint8)


# ---------------------------------------------------------------------------
# a7: block-sparse attend

def attend_tile(Q_tile: np.ndarray, K: np.ndarray, V: np.ndarray, kv_row: np.ndarray,
                row0: int, block_k: int, scale: float):
    """Softmax attention of the tile's rows over the listed key blocks
    ([UGS step 5], [Stem, Implementação]: sparse aggregation over the selected
    blocks), with the causal rule key <= query. K, V [N, d] of the head's KV
    group. Returns (O [rows, d], lse [rows]) in fp64; lse is the natural log of
    the softmax denominator."""
    Qt = widen(Q_tile)
    blocks = [int(j) for j in kv_row if j >= 0]
    if not blocks:
        return np.zeros((Qt.shape[0], K.shape[-1])), np.full(Qt.shape[0], -np.inf)
    keys = np.concatenate([np.arange(j * block_k, (j + 1) * block_k) for j in blocks])
    Kt, Vt = widen(K[keys]), widen(V[keys])
    logits = scale * (Qt @ Kt.T)
    rows = row0 + np.arange(Qt.shape[0])
    logits[keys[None, :] > rows[:, None]] = -np.inf
    seen = np.isfinite(logits).any(axis=1)
    # a row that sees no key of the listed blocks (possible only for a caller-made
    # list without the tile's own block) has an empty softmax: output 0, lse -inf
    mx = np.where(seen, logits.max(axis=1), 0.0)[:, None]
    p = np.exp(logits - mx)
    den = p.sum(axis=1, keepdims=True)
    out = np.where(seen[:, None], (p @ Vt) / np.where(den > 0, den, 1.0), 0.0)
    lse = np.where(seen, (mx + np.log(np.where(den > 0, den, 1.0)))[:, 0], -np.inf)
    return out, lse


def attend(Q, K, V, kv_idx, tile_q, block_k, scale, tiles=None):
    """O [B,Hq,N,d] fp64 and lse [B,Hq,N]; with ``tiles`` (a list of (b, h, t))
    only those tiles are computed and the rest is left NaN."""
    B, Hq, N, d = Q.shape
    G = Hq // K.shape[1]
    O = np.full((B, Hq, N, d), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    if tiles is None:
        tiles = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(N // tile_q)]
    for b, h, t in tiles:
        r0 = t * tile_q
        o, l = attend_tile(Q[b, h, r0:r0 + tile_q], K[b, h // G], V[b, h // G],
                           kv_idx[b, h, t], r0, block_k, scale)
        O[b, h, r0:r0 + tile_q] = o
        lse[b, h, r0:r0 + tile_q] = l
    return O, lse


def dense_causal_attention(Q, K, V, scale):
    """Textbook softmax(scale * Q K^T + causal mask) V for [N, d] operands, fp64."""
    Q, K, V = widen(Q), widen(K), widen(V)
    N = Q.shape[0]
    logits = scale * (Q @ K.T)
    logits[np.triu(np.ones((N, N), bool), 1)] = -np.inf
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)) @ V


def vs_keys(i: int, v_cols: Sequence[int], s_offs: Sequence[int]) -> np.ndarray:
    """Key positions of query row i under a vertical-slash pattern ([VSP,
    Metodologia A]: vertical columns are keys every later query attends to; a
    slash offset o is the diagonal of keys j = i - o): the union, each key once,
    of {j in v_cols : j <= i} and {i - o : o in s_offs, o <= i}, ascending."""
    keys = {int(j) for j in v_cols if 0 <= int(j) <= i}
    keys.update(i - int(o) for o in s_offs if 0 <= int(o) <= i)
    return np.array(sorted(keys), dtype=np.int64)


def attend_vs(Q, K, V, v_idx, v_cnt, s_off, s_cnt, scale, rows=None):
    """Softmax attention of every query row over its vertical-slash key set
    ([VSP, Metodologia B.3]: the sparse attention over the merged vertical and
    diagonal indices). Q [B,Hq,N,d], K/V [B,Hkv,N,d]; v_idx [B,Hq,Wv] and s_off
    [B,Hq,Ws] with counts v_cnt, s_cnt [B,Hq]: entries beyond the count, and
    entries outside [0, N), are ignored. Returns (O [B,Hq,N,d], lse [B,Hq,N]) in
    fp64; a row with an empty key set has output 0 and lse -inf. With ``rows``
    (a list of (b, h, i)) only those rows are computed, the rest left NaN."""
    B, Hq, N, d = Q.shape
    G = Hq // K.shape[1]
    O = np.full((B, Hq, N, d), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(N)]
    cache = {}
    for b, h, i in rows:
        if (b, h) not in cache:
            vc = [int(j) for j in v_idx[b, h, :int(v_cnt[b, h])] if 0 <= int(j) < N]
            so = [int(o) for o in s_off[b, h, :int(s_cnt[b, h])] if 0 <= int(o) < N]
            cache[b, h] = (vc, so, widen(K[b, h // G]), widen(V[b, h // G]), widen(Q[b, h]))
        vc, so, Kf, Vf, Qf = cache[b, h]
        keys = vs_keys(i, vc, so)
        if keys.size == 0:
            O[b, h, i] = 0.0
            lse[b, h, i] = -np.inf
            continue
        logits = scale * (Kf[keys] @ Qf[i])
        mx = logits.max()
        p = np.exp(logits - mx)
        den = p.sum()
        O[b, h, i] = (p @ Vf[keys]) / den
        lse[b, h, i] = mx + math.log(den)
    return O, lse


# ---------------------------------------------------------------------------
# a8: decode with run-time termination

def pairwise_sum64(terms) -> float:
    """Sum of at most 64 fp64 terms in one fixed pairwise order, each add rounded
    (IEEE, to nearest): term i is added to term i + 32 (zero where there is none),
    then values 16, 8, 4, 2 and 1 apart. The pages give no order for the probe
    sums of [ART, 2.2]; this one is the reading chosen (a warp of 32 lanes holding
    two coordinates each evaluates it in five steps)."""
    t = np.asarray(terms, dtype=np.float64)
    assert t.ndim == 1 and t.size <= 64
    a = np.zeros(64)
    a[:t.size] = t
    a = a[:32] + a[32:]
    while a.size > 1:
        h = a.size // 2
        a = a[:h] + a[h:]
    return float(a[0])


def probe_step(x_prev: Sequence[float], x_cur: Sequence[float]):
    """(d_scale, d_direction) between consecutive probes ([ART, 2.2]):
    the absolute difference of their L2 norms and one minus their cosine.
    fp64 on the fp32 probe values (at most 64): products rounded on their own
    (exact, being products of fp32 values), sums in the pairwise order of
    pairwise_sum64; d_direction = 1 when a norm is zero."""
    xc = np.asarray(x_cur, dtype=np.float32).astype(np.float64)
    xp = np.asarray(x_prev, dtype=np.float32).astype(np.float64)
    s_cur = pairwise_sum64(xc * xc)
    s_prev = pairwise_sum64(xp * xp)
    dot = pairwise_sum64(xc * xp)
    n_cur = math.sqrt(s_cur)
    n_prev = math.sqrt(s_prev)
    d_scale = abs(n_cur - n_prev)
    den = n_cur * n_prev
    d_dir = 1.0 if den == 0.0 else 1.0 - dot / den
    return d_scale, d_dir


def termination_block(trace: np.ndarray, tau: float, phi: float, patience: int,
                      n_blocks: Optional[int] = None) -> int:
    """blocks_used from a probe trace [n_blocks, n_probe] (fp32): block 0 is
    always processed ([ART, 2.4]); after each block t >= 1 the block is stable
    iff d_scale < tau and d_direction < phi ([ART, 2.2]); streaming stops after
    block t once ``patience`` consecutive stable blocks end at t ([ART, 2.3]).
    Returns t+1, or the total block count when it never stops. tau and phi are
    compared as fp32 parameters widened to fp64."""
    trace = np.asarray(trace, dtype=np.float32)
    n = trace.shape[0] if n_blocks is None else n_blocks
    tau64 = float(np.float32(tau))
    phi64 = float(np.float32(phi))
    run = 0
    for t in range(1, n):
        ds, dd = probe_step(trace[t - 1], trace[t])
        if ds < tau64 and dd < phi64:
            run += 1
        else:
            run = 0
        if run >= patience:
            return t + 1
    return n


def decode_group(q: np.ndarray, Kc: np.ndarray, Vc: np.ndarray, block_kv: int, scale: float,
                 tau: float, phi: float, patience: int, probe_dims: np.ndarray,
                 enable: bool = True):
    """One (batch, KV head): q [G, d] (the group's query heads), caches [L, d].

    Blocks 0, 1, ... of block_kv keys are visited in order ([ART, 2.1]); after
    block t the normalised partial output O^(t) of each head is the softmax
    over all keys of blocks 0..t applied to V (fp64; the common max shift
    cancels in the ratio). The probe x^(t) is O^(t) of the group's first head
    at ``probe_dims``, rounded to fp32. Returns (O [G, d] fp64 at the final
    block, blocks_used, trace [n_blocks, n_probe] fp32 up to blocks_used).
    """
    qf, Kf, Vf = widen(q), widen(Kc), widen(Vc)
    L = Kf.shape[0]
    nb = L // block_kv
    logits = scale * (qf @ Kf.T)                       # [G, L]
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    eb = e.reshape(e.shape[0], nb, block_kv)
    num = np.cumsum(np.einsum("gbk,bkd->gbd", eb, Vf.reshape(nb, block_kv, -1)), axis=1)
    den = np.cumsum(eb.sum(axis=2), axis=1)            # [G, nb]
    partial = num / den[:, :, None]                    # O^(t) for every t: [G, nb, d]
    trace = partial[0][:, probe_dims].astype(np.float32)
    used = termination_block(trace, tau, phi, patience) if enable else nb
    return partial[:, used - 1, :], used, trace[:used]


def decode(q, Kc, Vc, block_kv, scale, tau, phi, patience, probe_dims, enable=True):
    """q [B,Hq,d], caches [B,Hkv,L,d] -> (O [B,Hq,d] fp64, blocks_used [B,Hkv],
    traces dict {(b, g): trace})."""
    B, Hq, d = q.shape
    Hkv = Kc.shape[1]
    G = Hq // Hkv
    O = np.empty((B, Hq, d))
    used = np.empty((B, Hkv), np.int32)
    traces = {}
    for b in range(B):
        for g in range(Hkv):
            o, u, tr = decode_group(q[b, g * G:(g + 1) * G], Kc[b, g], Vc[b, g], block_kv,
                                    scale, tau, phi, patience, probe_dims, enable)
            O[b, g * G:(g + 1) * G] = o
            used[b, g] = u
            traces[b, g] = tr
    return O, used, traces


def decode_visit_steps(blocks: Sequence[int], n_blocks: int) -> list:
    """The visit sequence of a decode block list: its entries in list order, with
    every entry outside [0, n_blocks) skipped. A skipped entry is not a visit step
    (it is neither streamed nor tested); the library reports it as a bad index.
    [ART, 2.4] only fixes that the traversal order may change; what an index
    outside the cache means is the library's reading: nothing to visit."""
    return [int(j) for j in blocks if 0 <= int(j) < n_blocks]


def decode_group_list(q: np.ndarray, Kc: np.ndarray, Vc: np.ndarray, block_kv: int, scale: float,
                      blocks: Sequence[int], tau: float, phi: float, patience: int,
                      probe_dims: np.ndarray, enable: bool = True):
    """One (batch, KV head) visiting the listed KV blocks in list order ([ART, 2.4]:
    the result of a full pass does not depend on the order, so a selector's blocks
    may be visited first block first, then most important or most recent first).

    The visit steps are ``decode_visit_steps(blocks, L // block_kv)``: entries
    outside the cache are skipped. After visit step t the normalised partial output
    O^(t) of each head is the softmax over all keys of the first t+1 visited blocks
    applied to V (fp64); the probe, the stability test and the stop rule are those
    of ``decode_group`` with the visit step in place of the block number (the first
    visited block is never tested). No visit step gives O = 0 and blocks_used = 0.
    Returns (O [G, d] fp64, blocks_used, trace [steps used, n_probe] fp32).
    """
    qf, Kf, Vf = widen(q), widen(Kc), widen(Vc)
    G, d = qf.shape
    blocks = decode_visit_steps(blocks, Kf.shape[0] // block_kv)
    n = len(blocks)
    if n == 0:
        return np.zeros((G, d)), 0, np.zeros((0, len(probe_dims)), np.float32)
    rows = np.concatenate([np.arange(j * block_kv, (j + 1) * block_kv) for j in blocks])
    Kv, Vv = Kf[rows], Vf[rows]                        # keys in visit order
    logits = scale * (qf @ Kv.T)                       # [G, n * block_kv]
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    eb = e.reshape(G, n, block_kv)
    num = np.cumsum(np.einsum("gsk,skd->gsd", eb, Vv.reshape(n, block_kv, d)), axis=1)
    den = np.cumsum(eb.sum(axis=2), axis=1)
    partial = num / den[:, :, None]                    # O^(t) after each visit step
    trace = partial[0][:, probe_dims].astype(np.float32)
    used = termination_block(trace, tau, phi, patience) if enable else n
    return partial[:, used - 1, :], used, trace[:used]


def decode_list(q, Kc, Vc, block_kv, scale, block_list, list_cnt, tau, phi, patience, probe_dims,
                enable=True):
    """q [B,Hq,d], caches [B,Hkv,L,d], block_list [B,Hkv,W] int (visit order, the
    first list_cnt[b,g] entries used; a count outside [0, W] is clamped to it, and
    entries outside the cache are skipped by ``decode_group_list``) ->
    (O [B,Hq,d] fp64, blocks_used [B,Hkv], traces {(b, g): trace})."""
    B, Hq, d = q.shape
    Hkv = Kc.shape[1]
    G = Hq // Hkv
    O = np.empty((B, Hq, d))
    used = np.empty((B, Hkv), np.int32)
    traces = {}
    for b in range(B):
        for g in range(Hkv):
            W = block_list.shape[-1]
            lst = np.asarray(block_list[b, g][:min(max(int(list_cnt[b, g]), 0), W)])
            o, u, tr = decode_group_list(q[b, g * G:(g + 1) * G], Kc[b, g], Vc[b, g], block_kv,
                                         scale, lst, tau, phi, patience, probe_dims, enable)
            O[b, g * G:(g + 1) * G] = o
            used[b, g] = u
            traces[b, g] = tr
    return O, used, traces
