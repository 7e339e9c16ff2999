"""The benchmark's host logic on CPU: two gloo ranks run its rank-level logic
(independent problems per rank, max-over-ranks timing, summed work), and its
count of unmasked (row, key) pairs is checked against enumeration."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    step = 10.0 + rank           # rank 1 is the slower one
    att = 8.0 + 2 * rank
    e2e = 20.0 - rank
    flops = 1e12 * (rank + 1)
    out = bench.reduce_over_ranks(step, att, e2e, flops, world, torch.device("cpu"))
    q.put((rank, out, bench.rank_seed(rank)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_reduce_and_seed():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, (step, att, e2e, fl), seed in res:
        assert step == 11.0 and att == 10.0 and e2e == 20.0 and fl == 3e12
    assert res[0][2] != res[1][2]      # independent problems per rank


def test_unmasked_pair_count_matches_brute_force():
    """The bench's count of unmasked (row, key) pairs, against enumeration on small lists."""
    import itertools
    import bench as B
    rng = np.random.default_rng(9)
    for tq, bk in ((128, 64), (64, 64), (128, 128), (64, 128)):
        n_qt, W = 6, 5
        kv = np.full((1, 2, n_qt, W), -1, np.int32)
        cnt = np.zeros((1, 2, n_qt), np.int32)
        for h, t in itertools.product(range(2), range(n_qt)):
            J = ((t + 1) * tq - 1) // bk
            c = int(rng.integers(0, min(W, J + 1) + 1))
            kv[0, h, t, :c] = rng.permutation(J + 1)[:c]
            cnt[0, h, t] = c
        got = B.unmasked_pair_count(torch, torch.from_numpy(kv), torch.from_numpy(cnt), tq, bk)
        ref = 0
        for h, t in itertools.product(range(2), range(n_qt)):
            for w in range(cnt[0, h, t]):
                j0 = int(kv[0, h, t, w]) * bk
                rows = t * tq + np.arange(tq)[:, None]
                ref += int((j0 + np.arange(bk)[None, :] <= rows).sum())
        assert got == ref, (tq, bk, got, ref)


def test_path_rooflines_closed_forms():
    """The bench's score and selection work counts against closed forms: with 128-row tiles
    and 64-key blocks, tile t sees 2t + 2 causal blocks and ranks 2t candidates."""
    import bench as B
    from block_sparse_causal_bsa_b200 import synthetic as S
    spec = S.WORKLOADS[B.WORKLOAD]
    assert (spec.tile_q, spec.block_k) == (128, 64)
    n_qt, heads = spec.N // 128, spec.B * spec.Hq
    r = B.path_rooflines(spec, 2.0, {"score_ms": 3.0, "select_ms": 0.5},
                         {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0})
    flop = 2 * spec.d * 128 * heads * n_qt * (n_qt + 1)
    f = r["score_select"]
    assert f["algorithmic_tflop"] == pytest.approx(flop / 1e12)
    assert f["tflops"] == pytest.approx(flop / 2e-3 / 1e12)
    assert f["frac_tensor_burst"] == pytest.approx(flop / 2e-3 / 1e12 / 1000.0)
    q_k = (heads + spec.B * spec.Hkv) * spec.N * spec.d * 2
    W = min(spec.rho * spec.k_first, spec.N // 64)
    assert f["bytes"] == q_k + heads * n_qt * (W + 1) * 4            # kv_idx and kv_cnt written
    assert f["frac_hbm"] == pytest.approx(f["bytes"] / 2e-3 / 1e9 / 5000.0)
    u = r["unfused"]
    assert u["score_tflops"] == pytest.approx(flop / 3e-3 / 1e12)
    assert u["score_GBps"] == pytest.approx((q_k + heads * n_qt * (n_qt + 1) * 4) / 3e-3 / 1e9)
    sel = heads * n_qt * (n_qt - 1) * 4 + heads * n_qt * W * 4
    assert u["select_GBps"] == pytest.approx(sel / 0.5e-3 / 1e9)
    assert u["select_frac_hbm"] == pytest.approx(sel / 0.5e-3 / 1e9 / 5000.0)
