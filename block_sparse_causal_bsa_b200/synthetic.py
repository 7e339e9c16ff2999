"""Seeded synthetic inputs for block-sparse causal attention.

This module only draws random numbers and plants structure in them; it holds
none of the method's arithmetic (no pooling, scoring, selection or softmax).
The CUDA path, the CPU oracle and the benchmark all take their inputs from
here, so both sides of every parity check see the same bits.

Every tensor slice is drawn from its own generator, keyed by
``(seed, tensor, batch, head)``, so a single (b, h) slice of a 128k-token
workload can be regenerated without drawing the rest.

bf16 tensors are returned as ``uint16`` arrays of bf16 bit patterns
(round-to-nearest-even from float32); fp32 tensors as ``float32``.

Workloads (sizes and structure of the pages' settings):

* ``tiny_fp32_1k``: B=1, 2 heads (no GQA), N=1024, d=64, key block 64,
  query tile 64, fixed k=4, fp32 N(0,1).
* ``prefill_32k_vs``: B=1, 32 query / 8 KV heads, N=32768, d=128, key block
  64, query tile 128, k=64; N(0,1) plus vertical-slash structure (the
  "Vertical-Slash" observation of the VSPrefill page, Metodologia A): 4 key
  positions per KV head with K scaled by 4, and a local band built from a
  per-KV-head latent that is linearly interpolated every 128 tokens and
  added to both Q and K.
* ``gated_prefill_128k``: B=1, 32/8 heads, N=131072, d=128, block 64, tile
  128, base k=64, rho=2, quantile 0.25. K rows are a per-block mean plus
  unit noise; adjacent block pairs (2m, 2m+1) become twins with probability
  ``p_twin`` = 0.36 (exact copies, or copies with one element moved by one
  bf16 ulp), which plants near-tied block scores at the top-k cut: about a
  fifth of the (head, cut tile) pairs then have s_(k-1) - s_(k) < 1e-3.
* ``tpd_oam_prefill_64k``: B=2, 32/8 heads, N=65536, d=128, block 64, tile
  128, k decaying linearly from 128 to 32, output-aware score; V rows are
  exp(N(0,1)) * N(0, I) (log-normal row norms, sigma=1).
* ``decode_art_64k``: batch 16, 32/8 heads, one query per sequence, KV
  cache 65536, d=128, KV block 128; K, V ~ N(0,1) with K of the first 4096
  positions scaled by 2.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "vertical": 4, "latent": 5,
               "blockmean": 6, "twin": 7, "vscale": 8, "blocklist": 9, "vsidx": 10}


@dataclasses.dataclass(frozen=True)
class PrefillSpec:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    block_k: int
    tile_q: int
    k_first: int
    k_last: int
    rho: int
    gate_quantile: float
    score_kind: str          # "mean" or "mean_vnorm"
    dtype: str               # "bf16" or "f32"
    structure: str           # "iid", "vertical_slash", "twins", "lognormal_v"
    p_twin: float = 0.0
    block_mean_std: float = 0.0

    @property
    def n_qt(self) -> int:
        return self.N // self.tile_q

    @property
    def n_kb(self) -> int:
        return self.N // self.block_k

    def scaled(self, N: Optional[int] = None, B: Optional[int] = None,
               Hq: Optional[int] = None, Hkv: Optional[int] = None,
               **kw) -> "PrefillSpec":
        """Same structure at another size (for parity cases the oracle finishes quickly)."""
        ch = {}
        if N is not None:
            ch["N"] = N
        if B is not None:
            ch["B"] = B
        if Hq is not None:
            ch["Hq"] = Hq
        if Hkv is not None:
            ch["Hkv"] = Hkv
        ch.update(kw)
        return dataclasses.replace(self, **ch)


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    block_kv: int
    tau: float
    phi: float
    patience: int
    early_len: int = 4096
    early_k_scale: float = 2.0

    def scaled(self, **kw) -> "DecodeSpec":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_fp32_1k": PrefillSpec(
        "tiny_fp32_1k", B=1, Hq=2, Hkv=2, N=1024, d=64, block_k=64, tile_q=64,
        k_first=4, k_last=4, rho=1, gate_quantile=0.25, score_kind="mean",
        dtype="f32", structure="iid"),
    "prefill_32k_vs": PrefillSpec(
        "prefill_32k_vs", B=1, Hq=32, Hkv=8, N=32768, d=128, block_k=64,
        tile_q=128, k_first=64, k_last=64, rho=1, gate_quantile=0.25,
        score_kind="mean", dtype="bf16", structure="vertical_slash"),
    "gated_prefill_128k": PrefillSpec(
        "gated_prefill_128k", B=1, Hq=32, Hkv=8, N=131072, d=128, block_k=64,
        tile_q=128, k_first=64, k_last=64, rho=2, gate_quantile=0.25,
        score_kind="mean", dtype="bf16", structure="twins", p_twin=0.36,
        block_mean_std=1.0),
    "tpd_oam_prefill_64k": PrefillSpec(
        "tpd_oam_prefill_64k", B=2, Hq=32, Hkv=8, N=65536, d=128, block_k=64,
        tile_q=128, k_first=128, k_last=32, rho=1, gate_quantile=0.25,
        score_kind="mean_vnorm", dtype="bf16", structure="lognormal_v"),
}

DECODE_WORKLOADS = {
    "decode_art_64k": DecodeSpec(
        "decode_art_64k", B=16, Hq=32, Hkv=8, L=65536, d=128, block_kv=128,
        tau=1e-3, phi=1e-4, patience=1),
}


# ---------------------------------------------------------------------------
# bf16 bit helpers (storage format only)

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, tensor: str, *idx: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), _TENSOR_IDS[tensor]] + [int(i) for i in idx])


# ---------------------------------------------------------------------------
# prefill

def _band_latent(spec: PrefillSpec, seed: int, b: int, g: int) -> np.ndarray:
    """Latent w(i) for the local band: a N(0, I) vector every 128 tokens, linearly interpolated."""
    seg = 128
    n_seg = spec.N // seg + 2
    L = _rng(seed, "latent", b, g).standard_normal((n_seg, spec.d), dtype=np.float32)
    i = np.arange(spec.N)
    m = i // seg
    frac = ((i % seg) / seg).astype(np.float32)[:, None]
    return (1.0 - frac) * L[m] + frac * L[m + 1]


def _vertical_positions(spec: PrefillSpec, seed: int, b: int, g: int) -> np.ndarray:
    return _rng(seed, "vertical", b, g).choice(spec.N, size=4, replace=False)


def prefill_k_f32(spec: PrefillSpec, seed: int, b: int, g: int) -> np.ndarray:
    """K[b, g] as float32 values before the final bf16 rounding."""
    d, N = spec.d, spec.N
    k = _rng(seed, "k", b, g).standard_normal((N, d), dtype=np.float32)
    if spec.structure == "vertical_slash":
        k += _band_latent(spec, seed, b, g)
        k[_vertical_positions(spec, seed, b, g)] *= 4.0
    elif spec.structure == "twins":
        nb = N // spec.block_k
        mu = _rng(seed, "blockmean", b, g).standard_normal((nb, d), dtype=np.float32)
        k = (k.reshape(nb, spec.block_k, d) + spec.block_mean_std * mu[:, None, :]).reshape(N, d)
    return k


def _plant_twins(spec: PrefillSpec, seed: int, b: int, g: int, kbits: np.ndarray) -> None:
    """Make block 2m+1 a copy of block 2m (exact, or one element moved by one bf16 ulp)."""
    bk, d = spec.block_k, spec.d
    nb = spec.N // bk
    r = _rng(seed, "twin", b, g)
    u = r.random(nb // 2)
    kind = r.random(nb // 2)
    row = r.integers(0, bk, size=nb // 2)
    col = r.integers(0, d, size=nb // 2)
    blocks = kbits.reshape(nb, bk, d)
    for m in np.nonzero(u < spec.p_twin)[0]:
        blocks[2 * m + 1] = blocks[2 * m]
        if kind[m] < 0.5:
            e = blocks[2 * m + 1, row[m], col[m]]
            if (int(e) & 0x7FFF) not in (0, 0x7F7F):   # not +-0, not the largest finite
                blocks[2 * m + 1, row[m], col[m]] = np.uint16(int(e) + 1)


def prefill_head(spec: PrefillSpec, seed: int, tensor: str, b: int, h: int) -> np.ndarray:
    """One [N, d] slice of Q (h = query head) or K/V (h = KV head).

    Returns uint16 bf16 bits for bf16 workloads, float32 for fp32 ones.
    """
    d, N = spec.d, spec.N
    G = spec.Hq // spec.Hkv
    if tensor == "q":
        x = _rng(seed, "q", b, h).standard_normal((N, d), dtype=np.float32)
        if spec.structure == "vertical_slash":
            x += _band_latent(spec, seed, b, h // G)
    elif tensor == "k":
        x = prefill_k_f32(spec, seed, b, h)
    elif tensor == "v":
        x = _rng(seed, "v", b, h).standard_normal((N, d), dtype=np.float32)
        if spec.structure == "lognormal_v":
            s = np.exp(_rng(seed, "vscale", b, h).standard_normal(N, dtype=np.float32))
            x *= s[:, None]
    else:
        raise ValueError(tensor)
    if spec.dtype == "f32":
        return x
    bits = f32_to_bf16_bits(x)
    if tensor == "k" and spec.structure == "twins":
        _plant_twins(spec, seed, b, h, bits)
    return bits


def prefill_inputs(spec: PrefillSpec, seed: int):
    """Full Q [B,Hq,N,d], K and V [B,Hkv,N,d] (bf16 bits or float32)."""
    dt = np.float32 if spec.dtype == "f32" else np.uint16
    q = np.empty((spec.B, spec.Hq, spec.N, spec.d), dt)
    k = np.empty((spec.B, spec.Hkv, spec.N, spec.d), dt)
    v = np.empty((spec.B, spec.Hkv, spec.N, spec.d), dt)
    for b in range(spec.B):
        for h in range(spec.Hq):
            q[b, h] = prefill_head(spec, seed, "q", b, h)
        for g in range(spec.Hkv):
            k[b, g] = prefill_head(spec, seed, "k", b, g)
            v[b, g] = prefill_head(spec, seed, "v", b, g)
    return q, k, v


# ---------------------------------------------------------------------------
# decode

def decode_head(spec: DecodeSpec, seed: int, tensor: str, b: int, h: int) -> np.ndarray:
    """bf16 bits: q [d] for query head h, or K/V cache [L, d] for KV head h."""
    if tensor == "q":
        x = _rng(seed, "q", b, h).standard_normal(spec.d, dtype=np.float32)
    elif tensor == "k":
        x = _rng(seed, "k", b, h).standard_normal((spec.L, spec.d), dtype=np.float32)
        x[: spec.early_len] *= spec.early_k_scale
    elif tensor == "v":
        x = _rng(seed, "v", b, h).standard_normal((spec.L, spec.d), dtype=np.float32)
    else:
        raise ValueError(tensor)
    return f32_to_bf16_bits(x)


def decode_inputs(spec: DecodeSpec, seed: int):
    q = np.empty((spec.B, spec.Hq, spec.d), np.uint16)
    k = np.empty((spec.B, spec.Hkv, spec.L, spec.d), np.uint16)
    v = np.empty((spec.B, spec.Hkv, spec.L, spec.d), np.uint16)
    for b in range(spec.B):
        for h in range(spec.Hq):
            q[b, h] = decode_head(spec, seed, "q", b, h)
        for g in range(spec.Hkv):
            k[b, g] = decode_head(spec, seed, "k", b, g)
            v[b, g] = decode_head(spec, seed, "v", b, g)
    return q, k, v


def default_probe_dims(n_probe: int = 32) -> np.ndarray:
    """Default probe coordinates {8m, 8m+1 : m = 0..n_probe/2-1}."""
    m = np.arange(n_probe // 2)
    return np.stack([8 * m, 8 * m + 1], axis=1).reshape(-1).astype(np.int32)


def decode_block_lists(spec: DecodeSpec, seed: int, kind: str = "recency", keep: int = 0):
    """Visiting orders for decode over a block list (index arithmetic only).

    kind "recency": every block, block 0 first and then the most recent first
    (n-1, n-2, ..., 1). kind "subset": block 0 first, then ``keep - 1`` other
    blocks drawn without replacement per (batch, KV head), most recent first --
    the shape of a selector's kv_idx visited recency-first. Returns
    (lists [B, Hkv, W] int32 padded with -1, counts [B, Hkv] int32)."""
    n = spec.L // spec.block_kv
    if kind == "recency":
        W = n
    elif kind == "subset":
        if not 1 <= keep <= n:
            raise ValueError("keep must be in 1..n_blocks")
        W = keep
    else:
        raise ValueError(kind)
    lists = np.full((spec.B, spec.Hkv, W), -1, np.int32)
    cnt = np.full((spec.B, spec.Hkv), W, np.int32)
    for b in range(spec.B):
        for g in range(spec.Hkv):
            if kind == "recency":
                lists[b, g] = np.concatenate([[0], np.arange(n - 1, 0, -1)])
            else:
                rest = _rng(seed, "blocklist", b, g).choice(np.arange(1, n), size=keep - 1, replace=False)
                lists[b, g] = np.concatenate([[0], np.sort(rest)[::-1]])
    return lists, cnt


def vs_indices(spec: PrefillSpec, seed: int, n_vertical: int = 64, n_slash: int = 64,
               n_local: int = 32):
    """Vertical and slash indices per (batch, query head) shaped like a vertical-slash
    indexer's output (index arithmetic only): the vertical columns are the KV head's
    planted anchor positions (the "vertical_slash" structure), the first 4 positions,
    and seeded random positions, n_vertical in all; the slash offsets are the local
    band 0..n_local-1 and seeded random offsets, n_slash in all. Both lists are
    shuffled (their order carries no meaning). Returns (v_idx [B,Hq,n_vertical],
    v_cnt [B,Hq], s_off [B,Hq,n_slash], s_cnt [B,Hq]), int32."""
    G = spec.Hq // spec.Hkv
    v_idx = np.empty((spec.B, spec.Hq, n_vertical), np.int32)
    s_off = np.empty((spec.B, spec.Hq, n_slash), np.int32)
    for b in range(spec.B):
        for h in range(spec.Hq):
            rng = _rng(seed, "vsidx", b, h)
            fixed = list(dict.fromkeys([int(x) for x in _vertical_positions(spec, seed, b, h // G)] +
                                       [0, 1, 2, 3]))[:n_vertical]
            rest = np.setdiff1d(np.arange(spec.N), fixed)
            vc = np.concatenate([fixed, rng.choice(rest, size=n_vertical - len(fixed), replace=False)])
            local = np.arange(min(n_local, n_slash))
            so = np.concatenate([local, rng.choice(np.arange(len(local), spec.N), size=n_slash - len(local),
                                                   replace=False)])
            v_idx[b, h] = rng.permutation(vc)
            s_off[b, h] = rng.permutation(so)
    cnt_v = np.full((spec.B, spec.Hq), n_vertical, np.int32)
    cnt_s = np.full((spec.B, spec.Hq), n_slash, np.int32)
    return v_idx, cnt_v, s_off, cnt_s
