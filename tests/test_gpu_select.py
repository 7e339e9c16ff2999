"""Selection (budget, ranking, cut margin, gate, kv_idx) on adversarial score
matrices, bit-exact against the oracle.

The scores are drawn here, seeded, per row from one of six structures that
stress the exact ranking: plain Gaussian values, a handful of levels (long runs
of ties broken by block index), a constant row, values a few ulps apart (keys
that differ only in their lowest bits), mixed signs with signed zeros, and
magnitudes from 1e-30 to 1e30. Together they reach both ranking paths of the
selection kernel: the value-bucket path (short candidate lists ranked by
pairwise counts) and its exact radix fallback (constant rows, long tie runs,
buckets or lists too large for the short path). Row widths run from 512 to 4096
candidate blocks.
"""
import numpy as np
import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from oracle import bsa_oracle as O

from gpu_util import check_selection

pytestmark = pytest.mark.gpu


def adversarial_scores(B, Hq, n_qt, n_kb, seed):
    rng = np.random.default_rng(seed)
    s = np.empty((B, Hq, n_qt, n_kb), np.float32)
    for b in range(B):
        for h in range(Hq):
            for t in range(n_qt):
                kind = (7 * h + t + b) % 6
                if kind == 0:
                    row = rng.standard_normal(n_kb)
                elif kind == 1:
                    row = rng.integers(0, 4, n_kb).astype(np.float64)
                elif kind == 2:
                    row = np.full(n_kb, 0.25)
                elif kind == 3:
                    ulp = np.spacing(np.float32(1.0))
                    row = np.float32(1.0) + rng.integers(0, 6, n_kb).astype(np.float32) * ulp
                elif kind == 4:
                    row = rng.choice(np.array([-1.5, -0.0, 0.0, 0.5, 2.0]), n_kb)
                else:
                    row = rng.choice(np.array([1e-30, -1e-30, 0.0, -0.0, 1e30, -1e30, 3.0]), n_kb)
                s[b, h, t] = row.astype(np.float32)
    return s


@pytest.mark.parametrize("N,block_k,tile_q,kf,kl,rho", [
    (32768, 64, 128, 24, 8, 3),      # 512 candidates per row at most
    (65536, 64, 128, 40, 16, 2),     # 1024
    (131072, 64, 128, 64, 16, 2),    # 2048
    (262144, 64, 128, 48, 48, 2),    # 4096
    (8192, 64, 64, 12, 12, 1),       # no expansion: the top-M set is the top-m set
    (16384, 128, 64, 9, 3, 4),       # 128 blocks, 64-row tiles
])
def test_select_adversarial(N, block_k, tile_q, kf, kl, rho):
    B, Hq = 1, 2
    n_qt, n_kb = N // tile_q, N // block_k
    s = adversarial_scores(B, Hq, n_qt, n_kb, seed=N + kf)
    shape = bb.Shape(B, Hq, Hq, N, 128, block_k, tile_q, bb.BSA_BF16)
    cfg = bb.SelectConfig(kf, kl, rho, 0.9)
    sel = bb.select(torch.from_numpy(s).cuda(), shape=shape, cfg=cfg)
    torch.cuda.synchronize()
    assert int(sel["dev_status"].item()) == 0
    ref = O.select(s, tile_q, block_k, kf, kl, rho, 0.9)
    check_selection(sel, ref)
    assert (ref["sigma"] == 0.0).any() and (ref["sigma"] > 0.0).any()
    assert (ref["trigger"].sum() > 0) == (rho > 1)
