"""Benchmark: block-sparse causal prefill at 128k on B200, plus decode with
run-time termination.

One step = one pass of the prefill hot path over one batch: pool + block score
with the per-row top-k ranked inside the score kernel, uncertainty gate and
kv_idx (bsa_score_select) -> block-sparse attend (bsa_attend), on the gated 128k
workload (B=1, 32 query / 8 KV heads,
N=131072, d=128, key block 64, query tile 128, k=64, rho=2, quantile 0.25).
value = effective TFLOP/s = (4 * tile_q * block_k * d per selected block, from
kv_cnt) / device time of the whole step. The decode row (batch 16, 64k cache,
termination on) is timed in the same run and reported under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun): every rank runs its own independent problem (weak
scaling; no collective on the data path); value sums all ranks' work over the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "gated_prefill_128k"
DECODE_WORKLOAD = "decode_art_64k"
METRIC = "effective TFLOP/s, bf16 block-sparse causal prefill at 128k; % of tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# inputs

def _gen_prefill(spec, seed):
    from block_sparse_causal_bsa_b200 import synthetic as S
    q = np.empty((spec.B, spec.Hq, spec.N, spec.d), np.uint16)
    k = np.empty((spec.B, spec.Hkv, spec.N, spec.d), np.uint16)
    v = np.empty((spec.B, spec.Hkv, spec.N, spec.d), np.uint16)
    jobs = [(q, "q", b, h) for b in range(spec.B) for h in range(spec.Hq)]
    jobs += [(k, "k", b, g) for b in range(spec.B) for g in range(spec.Hkv)]
    jobs += [(v, "v", b, g) for b in range(spec.B) for g in range(spec.Hkv)]

    def one(j):
        arr, name, b, h = j
        arr[b, h] = S.prefill_head(spec, seed, name, b, h)

    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(one, jobs))
    return q, k, v


def _gen_decode(spec, seed):
    from block_sparse_causal_bsa_b200 import synthetic as S
    q = np.empty((spec.B, spec.Hq, spec.d), np.uint16)
    k = np.empty((spec.B, spec.Hkv, spec.L, spec.d), np.uint16)
    v = np.empty((spec.B, spec.Hkv, spec.L, spec.d), np.uint16)
    jobs = [(q, "q", b, h) for b in range(spec.B) for h in range(spec.Hq)]
    jobs += [(k, "k", b, g) for b in range(spec.B) for g in range(spec.Hkv)]
    jobs += [(v, "v", b, g) for b in range(spec.B) for g in range(spec.Hkv)]

    def one(j):
        arr, name, b, h = j
        arr[b, h] = S.decode_head(spec, seed, name, b, h)

    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(one, jobs))
    return q, k, v


def _bf16(torch, a, device, pin=False):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    if pin:
        return t.pin_memory()
    return t.to(device)


# ---------------------------------------------------------------------------
# clocks

class Clocks:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.5)           # let the sampler start before the timed region
        return self

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def __exit__(self, *a):
        if self.p:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        import datetime
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9 and p[1].replace(".", "").isdigit():
                try:
                    ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                rows.append((ts, p))
        os.unlink(self.f.name)
        t0, t1 = getattr(self, "t0", None), getattr(self, "t1", None)
        inside = [p for ts, p in rows if ts is not None and t0 is not None and t0 - 0.05 <= ts <= t1 + 0.05]
        rows = inside if inside else [p for _, p in rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)

def cpu_sample(spec, seed, n_tiles: int, rng_seed: int = 7, cache=None):
    """Run the oracle's prefill path on a seeded sample of (b, h, t) tiles:
    pooling of the sampled heads' KV groups, block scores for the sampled
    rows, ranking + sigma, the gate over the sampled population, and sparse
    attend of the sampled tiles. Returns (seconds, selected-block flops)."""
    from block_sparse_causal_bsa_b200 import synthetic as S
    from oracle import bsa_oracle as O
    rng = np.random.default_rng(rng_seed)
    G = spec.Hq // spec.Hkv
    n_qt = spec.n_qt
    tiles = [(int(rng.integers(spec.B)), int(rng.integers(spec.Hq)), int(rng.integers(n_qt)))
             for _ in range(n_tiles)]
    heads = sorted({(b, h) for b, h, _ in tiles})
    groups = sorted({(b, h // G) for b, h in heads})
    data = {} if cache is None else cache      # generated inputs (untimed), reusable across calls
    for b, g in groups:
        for name in ("k", "v"):
            if (name, b, g) not in data:
                data[name, b, g] = S.prefill_head(spec, seed, name, b, g)
    for b, h in heads:
        if ("q", b, h) not in data:
            data["q", b, h] = S.prefill_head(spec, seed, "q", b, h)
    t0 = time.perf_counter()
    kbar = {bg: O.pool_keys(data["k", bg[0], bg[1]], spec.block_k) for bg in groups}
    rows = []
    for b, h, t in tiles:
        _, J = O.tile_blocks(t, spec.tile_q, spec.block_k)
        qt = data["q", b, h][t * spec.tile_q:(t + 1) * spec.tile_q]
        s = O.score_tile(qt, kbar[b, h // G], J)
        rows.append(s)
    scores = np.stack(rows)[None, :, None, :]          # treat each sampled tile as its own row
    n_kb = spec.n_kb
    sig = np.ones(len(tiles), np.float32)
    cut = np.zeros(len(tiles), bool)
    ranked = []
    for i, (b, h, t) in enumerate(tiles):
        nF, nc, m, M = O.tile_slots(t, n_qt, spec.tile_q, spec.block_k, spec.k_first, spec.k_last, spec.rho)
        order = O.rank_candidates(rows[i], nc)
        ranked.append(order)
        cut[i] = nc > m >= 1
        if cut[i]:
            sig[i] = O.cut_margin(rows[i], order, m)
    theta = O.empirical_quantile(sig[cut], spec.gate_quantile) if spec.rho > 1 and cut.any() else np.nan
    flops = 0.0
    scale = 1.0 / math.sqrt(spec.d)
    for i, (b, h, t) in enumerate(tiles):
        nF, nc, m, M = O.tile_slots(t, n_qt, spec.tile_q, spec.block_k, spec.k_first, spec.k_last, spec.rho)
        take = M if (cut[i] and sig[i] < theta) else m
        sel = np.sort(np.concatenate([ranked[i][:take], np.arange(nc, nc + nF)]))
        r0 = t * spec.tile_q
        O.attend_tile(data["q", b, h][r0:r0 + spec.tile_q], data["k", b, h // G],
                      data["v", b, h // G], sel, r0, spec.block_k, scale)
        flops += 4.0 * spec.tile_q * spec.block_k * spec.d * len(sel)
    del scores
    return time.perf_counter() - t0, flops


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(spec, seed, target_s=15.0):
    # size the sample from a probe so the measured run lasts about target_s
    cache = {}
    n = 48
    dt, _ = cpu_sample(spec, seed, n, rng_seed=3, cache=cache)
    n = int(max(16, min(8192, n * target_s / max(dt, 1e-3))))
    dt, fl = cpu_sample(spec, seed, n, cache=cache)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(),
            "host_cpus": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} random (b,h,t) tiles of {spec.name}: pooling of their KV groups, "
                      f"scores, ranking+sigma, gate over the sample, sparse attend; "
                      f"{dt:.1f} s, selected-block flops / time"}


def _causal_score_flops(spec):
    """Algorithmic block-score flops of a whole layer: 2 * d * tile_q per (b, h, tile, causal block)."""
    n_qt = spec.N // spec.tile_q
    causal = sum(((t + 1) * spec.tile_q - 1) // spec.block_k + 1 for t in range(n_qt))
    return 2.0 * spec.d * spec.tile_q * causal * spec.B * spec.Hq


def cpu_config_baselines(n_rows_c4=192, n_groups_c5=6):
    """The oracle timed per workload on the host cores, in the unit of the matching GPU
    figure (bounded samples where a whole layer would take minutes). Input generation is
    outside the timed region. Returns {workload: entry}."""
    from block_sparse_causal_bsa_b200 import synthetic as S
    from oracle import bsa_oracle as O
    cores, host = _blas_threads(), os.cpu_count()
    out = {}

    def entry(value, unit, dt, sample):
        return {"value": value, "unit": unit, "cores": cores, "host_cpus": host, "kind": "oracle",
                "seconds": dt, "sample": sample}

    # tiny fp32: the whole path (scores, selection, attend)
    spec = S.WORKLOADS["tiny_fp32_1k"]
    q, k, v = S.prefill_inputs(spec, 1001)
    t0 = time.perf_counter()
    sc = O.block_scores(q, k, spec.tile_q, spec.block_k)
    sel = O.select(sc, spec.tile_q, spec.block_k, spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    O.attend(q, k, v, sel["kv_idx"], spec.tile_q, spec.block_k, 1.0 / math.sqrt(spec.d))
    dt = time.perf_counter() - t0
    fl = 4.0 * spec.tile_q * spec.block_k * spec.d * float(sel["kv_cnt"].sum())
    out[spec.name] = entry(fl / dt / 1e12, "TFLOP/s", dt, "the whole problem: scores, selection and "
                           "attend of every tile; selected-block flops / time")
    # 32k vertical-slash workload: scores and selection of the whole layer
    spec = S.WORKLOADS["prefill_32k_vs"]
    q, k, _ = S.prefill_inputs(spec, 1002)
    t0 = time.perf_counter()
    sc = O.block_scores(q, k, spec.tile_q, spec.block_k)
    O.select(sc, spec.tile_q, spec.block_k, spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    dt = time.perf_counter() - t0
    out[spec.name] = entry(_causal_score_flops(spec) / dt / 1e12, "TFLOP/s", dt,
                           "scores and selection of the whole layer; algorithmic score flops / time")
    del q, k, sc
    # 64k position-decay budget, output-aware score: a seeded sample of (b, h, tile) rows
    spec = S.WORKLOADS["tpd_oam_prefill_64k"]
    rng = np.random.default_rng(11)
    G = spec.Hq // spec.Hkv
    rows = [(int(rng.integers(spec.B)), int(rng.integers(spec.Hq)), int(rng.integers(spec.n_qt)))
            for _ in range(n_rows_c4)]
    data = {}
    for b, h, _ in rows:
        for name, hh in (("q", h), ("k", h // G), ("v", h // G)):
            if (name, b, hh) not in data:
                data[name, b, hh] = S.prefill_head(spec, 1004, name, b, hh)
    t0 = time.perf_counter()
    pooled = {}
    fl = 0.0
    sig = []
    for b, h, t in rows:
        g = h // G
        if (b, g) not in pooled:
            pooled[b, g] = (O.pool_keys(data["k", b, g], spec.block_k),
                            O.value_block_norm(data["v", b, g], spec.block_k))
        kbar, w = pooled[b, g]
        f_lo, J = O.tile_blocks(t, spec.tile_q, spec.block_k)
        row = O.score_tile(data["q", b, h][t * spec.tile_q:(t + 1) * spec.tile_q], kbar, J, w)
        nF, nc, m, M = O.tile_slots(t, spec.n_qt, spec.tile_q, spec.block_k, spec.k_first, spec.k_last,
                                    spec.rho)
        order = O.rank_candidates(row, nc)
        if nc > m >= 1:
            sig.append(O.cut_margin(row, order, m))
        fl += 2.0 * spec.d * spec.tile_q * (J + 1)
    dt = time.perf_counter() - t0
    out[spec.name] = entry(fl / dt / 1e12, "TFLOP/s", dt,
                           f"{n_rows_c4} random (b,h,t) rows: pooling of their KV heads (keys and "
                           "value norms), output-aware scores, ranking and sigma; score flops / time")
    del data, pooled
    # decode with run-time termination: a sample of (batch, KV head) groups
    dspec = S.DECODE_WORKLOADS["decode_art_64k"]
    G = dspec.Hq // dspec.Hkv
    dims = S.default_probe_dims(32)
    groups = [(int(b), int(g)) for b, g in zip(rng.integers(dspec.B, size=n_groups_c5),
                                               rng.integers(dspec.Hkv, size=n_groups_c5))]
    ins = {(b, g): (np.stack([S.decode_head(dspec, 2005, "q", b, g * G + i) for i in range(G)]),
                    S.decode_head(dspec, 2005, "k", b, g), S.decode_head(dspec, 2005, "v", b, g))
           for b, g in groups}
    t0 = time.perf_counter()
    used = 0
    for b, g in groups:
        qg, kc, vc = ins[b, g]
        _, u, _ = O.decode_group(qg, kc, vc, dspec.block_kv, 1.0 / math.sqrt(dspec.d), dspec.tau,
                                 dspec.phi, dspec.patience, dims)
        used += u
    dt = time.perf_counter() - t0
    byts = used * dspec.block_kv * dspec.d * 2 * 2
    out[dspec.name] = entry(byts / dt / 1e9, "GB/s", dt,
                            f"{n_groups_c5} random (batch, KV head) groups with termination on; KV bytes "
                            "of the blocks used / time (the oracle forms every block's partial output)")
    return out


# ---------------------------------------------------------------------------
# GPU arm

def rank_seed(rank: int) -> int:
    """Each rank draws its own independent problem (weak scaling)."""
    return 1003 + 1000 * rank


def reduce_over_ranks(step_ms, attend_ms, e2e_ms, flops, world, device):
    """Max of the per-rank times and sum of the per-rank work (the slowest rank sets
    the job's time; value = all ranks' work / that time). No data moves between
    ranks on the compute path; this is the only collective besides the barriers."""
    import torch
    t = torch.tensor([step_ms, attend_ms, e2e_ms, flops], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        mx = t.clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        tot = t.clone()
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
        return float(mx[0]), float(mx[1]), float(mx[2]), float(tot[3])
    return step_ms, attend_ms, e2e_ms, flops


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def main_gpu(args):
    import torch
    import torch.distributed as dist
    from block_sparse_causal_bsa_b200 import binding as bb
    from block_sparse_causal_bsa_b200 import synthetic as S

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    spec = S.WORKLOADS[WORKLOAD]
    seed = rank_seed(rank)
    qh, kh, vh = _gen_prefill(spec, seed)
    q, k, v = _bf16(torch, qh, dev), _bf16(torch, kh, dev), _bf16(torch, vh, dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    shape = bb.make_shape(q, k, spec.block_k, spec.tile_q)
    cfg = bb.SelectConfig(spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    prm = cfg.c()
    W = bb.bsa_kv_idx_width(shape, prm)
    paths = {"score_select": bb.bsa_score_path(shape, bb.BSA_SCORE_MEAN),
             "attend": bb.bsa_attend_path(shape, W)}
    if any(v != bb.BSA_PATH_TENSOR_CORES for v in paths.values()):
        raise RuntimeError(f"the benchmark shape would leave the tensor cores: {paths}")
    B, Hq, N, d = q.shape
    n_qt, n_kb = N // spec.tile_q, N // spec.block_k
    scores = torch.empty(B, Hq, n_qt, n_kb, dtype=torch.float32, device=dev)
    kv_idx = torch.empty(B, Hq, n_qt, W, dtype=torch.int32, device=dev)
    kv_cnt = torch.empty(B, Hq, n_qt, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    st_sel = torch.zeros(1, dtype=torch.int32, device=dev)
    st_score = torch.zeros(1, dtype=torch.int32, device=dev)
    st_att = torch.zeros(1, dtype=torch.int32, device=dev)
    st_acc = torch.zeros(1, dtype=torch.int32, device=dev)       # OR of every timed call's status
    theta = torch.empty(1, dtype=torch.float32, device=dev)
    ws_s_n = bb.bsa_score_workspace_bytes(shape, bb.BSA_SCORE_MEAN)
    ws_s = torch.empty(ws_s_n, dtype=torch.uint8, device=dev)
    ws_l_n = bb.bsa_select_workspace_bytes(shape, prm)
    ws_l = torch.empty(ws_l_n, dtype=torch.uint8, device=dev)
    ws_f_n = bb.bsa_score_select_workspace_bytes(shape, bb.BSA_SCORE_MEAN, prm)
    ws_f = torch.empty(ws_f_n, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(d)

    def time_call(fn, reps=5, status=None):
        """Mean device time (ms) of fn over reps calls, L2 flushed before each."""
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            fn()
            b_.record(stream)
            ts.append((a_, b_))
        torch.cuda.synchronize()
        if status is not None and int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())}")
        return statistics.mean(a_.elapsed_time(b_) for a_, b_ in ts)

    def step(q_, k_, v_, out_, ev=None):
        # scores and selection in one call (the ranking runs inside the score kernel; the
        # scores are not written out), then the sparse attend
        if ev:
            ev[0].record(stream)
        bb.bsa_score_select(shape, bb.BSA_SCORE_MEAN, None, prm, q_, k_, None, None, kv_idx, kv_cnt,
                            None, None, None, theta, st_sel, ws_f, ws_f_n, sh)
        if ev:
            ev[1].record(stream)
        bb.bsa_attend(shape, q_, k_, v_, kv_idx, kv_cnt, W, scale, out_, None, st_att, sh)
        if ev:
            ev[2].record(stream)

    def unfused(ev=None):
        # the same selection through the separate calls: bsa_score writes the scores, bsa_select
        # reads them back
        if ev:
            ev[0].record(stream)
        bb.bsa_score(shape, bb.BSA_SCORE_MEAN, q, k, None, scores, st_score, ws_s, ws_s_n, sh)
        if ev:
            ev[1].record(stream)
        bb.bsa_select(shape, prm, scores, kv_idx, kv_cnt, None, None, None, theta, st_sel,
                      ws_l, ws_l_n, sh)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step(q, k, v, out)
    torch.cuda.synchronize()
    assert int(st_sel.item()) == 0 and int(st_att.item()) == 0 and int(st_score.item()) == 0
    sel_blocks = int(kv_cnt.sum().item())
    flops = 4.0 * spec.tile_q * spec.block_k * d * sel_blocks
    # unmasked (i, j) pairs of the selected blocks (j <= i), for the alternative count: a block
    # wholly below the tile's first row contributes tile_q * block_k pairs, a diagonal block fewer
    unmasked_pairs = unmasked_pair_count(torch, kv_idx, kv_cnt, spec.tile_q, spec.block_k)
    launches_per_step = 5     # pool, score+rank, gate, finalize, attend

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        clk.mark(True)
        for i in range(args.steps):
            flush.zero_()
            step(q, k, v, out, evs[i])
            st_acc.bitwise_or_(st_sel).bitwise_or_(st_att)   # after the events
        torch.cuda.synchronize()
        clk.mark(False)
    if int(st_acc.item()) != 0:
        raise RuntimeError(f"prefill step: device status {int(st_acc.item())} in a timed step")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = clk.summary()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(2)] for i in range(args.steps)])
    step_ms = float(per.sum(axis=1).mean())
    score_select_ms, attend_ms = (float(x) for x in per.mean(axis=0))
    kv_fused = kv_idx.clone()

    # warm variant: the same steps without the L2 flush in between
    wevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(5)]
    for i in range(5):
        step(q, k, v, out, wevs[i])
    torch.cuda.synchronize()
    wper = np.array([[wevs[i][j].elapsed_time(wevs[i][j + 1]) for j in range(2)] for i in range(5)])
    warm = {"step_ms": float(wper.sum(axis=1).mean()), "score_select_ms": float(wper[:, 0].mean()),
            "attend_ms": float(wper[:, 1].mean())}

    # the separate calls, timed the same way (cold), for comparison with the fused call
    uevs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(5)]
    for i in range(5):
        flush.zero_()
        unfused(uevs[i])
    torch.cuda.synchronize()
    if int(st_sel.item()) != 0 or int(st_score.item()) != 0:
        raise RuntimeError("unfused score/select: device status")
    if not torch.equal(kv_idx, kv_fused):
        raise RuntimeError("the fused and the separate score/select calls selected different blocks")
    uper = np.array([[uevs[i][j].elapsed_time(uevs[i][j + 1]) for j in range(2)] for i in range(5)])
    unfused_ms = {"score_ms": float(uper[:, 0].mean()), "select_ms": float(uper[:, 1].mean())}

    # end to end through the C ABI with host buffers: every step copies its Q, K, V from
    # pinned host memory to the device and its O back, all inside the timed region. The
    # copies run on two copy streams with two device slots, so step i+1's host-to-device
    # copy and step i's device-to-host copy overlap step i's kernels (PCIe is full duplex).
    qp, kp, vp = _bf16(torch, qh, dev, pin=True), _bf16(torch, kh, dev, pin=True), _bf16(torch, vh, dev, pin=True)
    op = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    # as many steps as the device-timed loop: the first upload and the last step's kernel and
    # download (the pipeline's fill and drain) stay inside the timed region, spread over them
    e2e_steps = max(2, args.steps)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slots = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(out))
             for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]      # slot's inputs landed
    ev_done = [torch.cuda.Event() for _ in range(2)]    # slot's kernels finished
    ev_out = [torch.cuda.Event() for _ in range(2)]     # slot's output copied back
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def upload(slot):
        with torch.cuda.stream(up):
            qd_, kd_, vd_, _ = slots[slot]
            qd_.copy_(qp, non_blocking=True)
            kd_.copy_(kp, non_blocking=True)
            vd_.copy_(vp, non_blocking=True)
            ev_in[slot].record(up)

    torch.cuda.synchronize()
    e0.record(up)
    upload(0)
    for i in range(e2e_steps):
        sl = i % 2
        qd_, kd_, vd_, od_ = slots[sl]
        stream.wait_event(ev_in[sl])
        if i >= 2:
            stream.wait_event(ev_out[sl])               # step i-2's output has left the slot
        step(qd_, kd_, vd_, od_)
        ev_done[sl].record(stream)
        if i + 1 < e2e_steps:
            if i >= 1:
                up.wait_event(ev_done[1 - sl])          # step i-1 finished reading that slot
            upload(1 - sl)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[sl])
            op.copy_(od_, non_blocking=True)
            ev_out[sl].record(down)
    e1.record(down)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if not torch.equal(op.to(dev), out):
        raise RuntimeError("end-to-end output differs from the device-timed step's output")
    h2d = (q.numel() + k.numel() + v.numel()) * 2
    d2h = out.numel() * 2
    del qp, kp, vp, op, slots

    # the other score backbones on the same inputs (pool + score, timed on their own)
    score_kinds = {}
    for kind, beta in (("vnorm", 0.0), ("vlog", 0.5), ("kminmax", 0.0)):
        code = bb.SCORE_KINDS[kind]
        kn = bb.bsa_score_workspace_bytes(shape, code)
        kws = torch.empty(kn, dtype=torch.uint8, device=dev)
        kp = bb.ScoreParams(beta)
        for _ in range(2):
            bb.bsa_score_ex(shape, code, kp, q, k, v, scores, st_score, kws, kn, sh)
        torch.cuda.synchronize()
        ts = []
        st_acc.zero_()
        for _ in range(5):
            flush.zero_()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            bb.bsa_score_ex(shape, code, kp, q, k, v, scores, st_score, kws, kn, sh)
            b_.record(stream)
            st_acc.bitwise_or_(st_score)
            ts.append((a, b_))
        torch.cuda.synchronize()
        if int(st_acc.item()) != 0:
            raise RuntimeError(f"score {kind}: device status {int(st_acc.item())}")
        score_kinds[kind] = {"ms": statistics.mean(a.elapsed_time(b_) for a, b_ in ts),
                             "beta": beta if kind == "vlog" else None}
        del kws
    score_kinds["mean"] = {"ms": unfused_ms["score_ms"]}

    # vertical-slash attention on the 32k vertical-slash workload (timed on its own)
    vspec = S.WORKLOADS["prefill_32k_vs"]
    vq, vk, vv = (_bf16(torch, x, dev) for x in _gen_prefill(vspec, 3001 + 1000 * rank))
    nv_, ns_ = 64, 64
    vidx = [torch.from_numpy(x).to(dev) for x in S.vs_indices(vspec, 3002 + 1000 * rank, nv_, ns_, 32)]
    vshape = bb.make_shape(vq, vk, 64, 128)
    vws_n = bb.bsa_attend_vs_workspace_bytes(vshape, nv_, ns_)
    vws = torch.empty(vws_n, dtype=torch.uint8, device=dev)
    vout = torch.empty_like(vq)
    vst = torch.zeros(1, dtype=torch.int32, device=dev)

    def run_vs():
        bb.bsa_attend_vs(vshape, vq, vk, vv, vidx[0], vidx[1], nv_, vidx[2], vidx[3], ns_,
                         1 / math.sqrt(vspec.d), vout, None, vst, vws, vws_n, sh)
    for _ in range(3):
        run_vs()
    torch.cuda.synchronize()
    ts = []
    st_acc.zero_()
    for _ in range(max(3, min(args.steps, 10))):
        flush.zero_()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run_vs()
        b_.record(stream)
        st_acc.bitwise_or_(vst)
        ts.append((a, b_))
    torch.cuda.synchronize()
    if int(st_acc.item()) != 0:
        raise RuntimeError(f"vertical-slash attend: device status {int(st_acc.item())}")
    vs_ms = statistics.mean(a.elapsed_time(b_) for a, b_ in ts)
    # visited (row tile, key block) pairs: the counts the list builder wrote into the workspace
    rows_vs = vspec.B * vspec.Hq * (vspec.N // 128)
    words = vspec.N // 64 + 1
    a256 = lambda x: (x + 255) // 256 * 256
    wl = min(vspec.N // 64, nv_ + 3 * ns_)
    off_c = 2 * a256(vspec.B * vspec.Hq * words * 8) + a256(rows_vs * wl * 4)
    visited = int(vws[off_c:off_c + rows_vs * 4].view(torch.int32).sum().item())
    vs_flops = 4.0 * 128 * 64 * vspec.d * visited
    vs_res = {"workload": "prefill_32k_vs", "n_vertical": nv_, "n_slash": ns_, "n_local": 32,
              "ms": vs_ms, "visited_block_pairs": visited,
              "visited_fraction_of_causal": visited / (vspec.B * vspec.Hq * sum(2 * t + 2 for t in range(vspec.N // 128))),
              "executed_tflops": vs_flops / (vs_ms * 1e-3) / 1e12}
    # the same workload's scores and selection (one fused call, scores not written out)
    vcfg = bb.SelectConfig(vspec.k_first, vspec.k_last, vspec.rho, vspec.gate_quantile)
    vsel = {}

    def run_vsel():
        vsel["r"] = bb.score_select(vq, vk, None, block_k=vspec.block_k, tile_q=vspec.tile_q, cfg=vcfg,
                                    want_scores=False)
    ms_c2 = time_call(run_vsel)
    if int(vsel["r"]["dev_status"].item()) != 0:
        raise RuntimeError("32k score/select: device status")
    gpu_configs = {vspec.name: {"value": _causal_score_flops(vspec) / (ms_c2 * 1e-3) / 1e12,
                                "unit": "TFLOP/s", "ms": ms_c2,
                                "scope": "scores and selection of the whole layer (bsa_score_select); "
                                         "algorithmic score flops / time"}}
    del vq, vk, vv, vws, vout, vsel

    # the tiny fp32 workload: the whole path (fp32 CUDA-core kernels)
    tspec = S.WORKLOADS["tiny_fp32_1k"]
    tq, tk, tv = (torch.from_numpy(x).to(dev) for x in S.prefill_inputs(tspec, 1001))
    tcfg = bb.SelectConfig(tspec.k_first, tspec.k_last, tspec.rho, tspec.gate_quantile)
    tres = {}

    def run_tiny():
        tres["r"] = bb.prefill(tq, tk, tv, block_k=tspec.block_k, tile_q=tspec.tile_q, cfg=tcfg)
    ms_c1 = time_call(run_tiny)
    t_out, t_sel, t_st = tres["r"]
    if int(t_st.item()) != 0 or int(t_sel["dev_status"].item()) != 0:
        raise RuntimeError("tiny fp32 prefill: device status")
    gpu_configs[tspec.name] = {"value": 4.0 * tspec.tile_q * tspec.block_k * tspec.d * float(t_sel["kv_cnt"].sum())
                               / (ms_c1 * 1e-3) / 1e12, "unit": "TFLOP/s", "ms": ms_c1,
                               "scope": "the whole path (scores and selection, attend); selected-block "
                                        "flops / time"}
    del tq, tk, tv, tres, t_out, t_sel

    # the 64k position-decay, output-aware workload: scores and selection (fused call)
    cspec = S.WORKLOADS["tpd_oam_prefill_64k"]
    cq, ck, cv = (_bf16(torch, x, dev) for x in _gen_prefill(cspec, 1004 + 1000 * rank))
    ccfg = bb.SelectConfig(cspec.k_first, cspec.k_last, cspec.rho, cspec.gate_quantile)
    cres = {}

    def run_c4():
        cres["r"] = bb.score_select(cq, ck, cv, block_k=cspec.block_k, tile_q=cspec.tile_q, cfg=ccfg,
                                    kind="vnorm", want_scores=False)
    ms_c4 = time_call(run_c4)
    if int(cres["r"]["dev_status"].item()) != 0:
        raise RuntimeError("64k score/select: device status")
    gpu_configs[cspec.name] = {"value": _causal_score_flops(cspec) / (ms_c4 * 1e-3) / 1e12,
                               "unit": "TFLOP/s", "ms": ms_c4,
                               "scope": "scores (times the value-block norms) and selection with the "
                                        "position-decay budget (bsa_score_select); algorithmic score "
                                        "flops / time"}
    del cq, ck, cv, cres

    # decode with run-time termination (timed on its own)
    dspec = S.DECODE_WORKLOADS[DECODE_WORKLOAD]
    dq, dk, dv = _gen_decode(dspec, 2005 + 1000 * rank)
    dq, dk, dv = _bf16(torch, dq, dev), _bf16(torch, dk, dev), _bf16(torch, dv, dev)
    dims = S.default_probe_dims(32)
    dshape = bb.DecodeShape(dspec.B, dspec.Hq, dspec.Hkv, dspec.L, dspec.d, dspec.block_kv, bb.BSA_BF16)
    paths["decode"] = bb.bsa_decode_path(dshape)
    if paths["decode"] != bb.BSA_PATH_TENSOR_CORES:
        raise RuntimeError("the decode workload would leave the tensor cores")
    cdims = (ctypes.c_int * len(dims))(*[int(x) for x in dims])
    dout = torch.empty_like(dq)
    used = torch.empty(dspec.B, dspec.Hkv, dtype=torch.int32, device=dev)
    dst = torch.zeros(1, dtype=torch.int32, device=dev)
    dec = {}
    # visit lists: block 0 then most recent first (every block), and a selector-shaped
    # subset of 64 blocks visited recency-first
    lists = {}
    for kind, keep in (("recency", 0), ("subset", 64)):
        lh, ch = S.decode_block_lists(dspec, 2006 + 1000 * rank, kind, keep)
        lists[kind] = (torch.from_numpy(lh).to(dev), torch.from_numpy(ch).to(dev), lh.shape[-1])
    # detector_on: the stability test runs after every block but can never pass (tau = phi = 0),
    # so the scan is as long as full_scan (test off); their difference is the detector's cost
    runs = (("terminated", 1, None, dspec.tau, dspec.phi), ("full_scan", 0, None, dspec.tau, dspec.phi),
            ("detector_on", 1, None, 0.0, 0.0),
            ("listed_recency", 1, "recency", dspec.tau, dspec.phi),
            ("listed_subset64", 1, "subset", dspec.tau, dspec.phi))
    for label, enable, lk, tau_, phi_ in runs:
        dp = bb.DecodeParams(tau_, phi_, dspec.patience, enable, len(dims), cdims)

        def run_decode():
            if lk is None:
                bb.bsa_decode(dshape, dp, dq, dk, dv, 1 / math.sqrt(dspec.d), dout, used, None, dst, sh)
            else:
                bl, bc, bw = lists[lk]
                bb.bsa_decode_list(dshape, dp, dq, dk, dv, bl, bc, bw, 1 / math.sqrt(dspec.d), dout,
                                   used, None, dst, sh)
        for _ in range(3):
            run_decode()
        torch.cuda.synchronize()
        ts = []
        st_acc.zero_()
        for _ in range(max(3, args.steps)):
            flush.zero_()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run_decode()
            b_.record(stream)
            st_acc.bitwise_or_(dst)
            ts.append((a, b_))
        torch.cuda.synchronize()
        if int(st_acc.item()) != 0:
            raise RuntimeError(f"decode {label}: device status {int(st_acc.item())}")
        ms = statistics.mean(a.elapsed_time(b_) for a, b_ in ts)
        blocks = int(used.sum().item())
        byts = blocks * dspec.block_kv * dspec.d * 2 * 2
        dec[label] = {"ms": ms, "blocks_used": blocks, "bytes": byts, "GBps": byts / ms / 1e6}
    peaks, peak_kind = _peaks()
    dec["hbm_frac_full_scan"] = dec["full_scan"]["GBps"] / peaks["hbm_gbs"]
    dec["hbm_frac_terminated"] = dec["terminated"]["GBps"] / peaks["hbm_gbs"]
    if dec["detector_on"]["blocks_used"] != dec["full_scan"]["blocks_used"]:
        raise RuntimeError("decode with tau = phi = 0 stopped early")
    dec["detector_overhead_pct"] = 100.0 * (dec["detector_on"]["ms"] / dec["full_scan"]["ms"] - 1.0)
    dec["mean_blocks_used"] = dec["terminated"]["blocks_used"] / (dspec.B * dspec.Hkv)
    dec["blocks_total"] = dspec.L // dspec.block_kv
    dec["peak_note"] = f"{peak_kind} HBM {peaks['hbm_gbs']} GB/s"

    # max over ranks
    step_ms, attend_ms, e2e_ms, total_flops = reduce_over_ranks(step_ms, attend_ms, e2e_ms, flops,
                                                                world, dev)
    if rank == 0:
        sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        sm_max = float(clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz", 1965.0))
        achieved = flops / (attend_ms * 1e-3) / 1e12
        achieved_unmasked = 4.0 * d * unmasked_pairs / (attend_ms * 1e-3) / 1e12
        traffic = None
        tp = os.path.join(ROOT, "profiles", "attend_traffic.json")
        if os.path.exists(tp):
            try:
                tj = json.load(open(tp))
                if tj.get("kernel") == "attend" and tj.get("source_sha") == _attend_sha():
                    traffic = tj["dram_bytes_per_launch"]
            except Exception:
                traffic = None
        res = {
            "metric": METRIC, "value": total_flops / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; N(0,1) plus per-block means and planted twin blocks)",
            "config": {"workload": WORKLOAD, "B": B, "Hq": Hq, "Hkv": k.shape[1], "N": N, "d": d,
                       "block_k": spec.block_k, "tile_q": spec.tile_q, "k": spec.k_first,
                       "rho": spec.rho, "gate_quantile": spec.gate_quantile,
                       "selected_blocks": sel_blocks,
                       "attend_tflop_per_step": flops / 1e12,
                       "l2": "256 MB buffer written between timed steps; inputs 1.6 GB > 126 MB L2",
                       "parallelism": f"independent problem per rank x{world}"},
            "kernel_ms": {"score_select": score_select_ms, "attend": attend_ms},
            "path_rooflines": path_rooflines(spec, score_select_ms, unfused_ms, peaks),
            "score_backbones_ms": score_kinds,
            "vertical_slash": vs_res,
            "attend_detail": {"frac_of_burst_peak": achieved / burst, "burst_peak": burst,
                              "frac_of_sustained_peak": achieved / sustained, "sustained_peak": sustained,
                              "frac_of_datasheet_dense": achieved / 2250.0,
                              "unmasked_pair_tflops": achieved_unmasked,
                              "unmasked_pairs": unmasked_pairs,
                              "step_ms_median": float(np.median(per.sum(axis=1))),
                              "attend_ms_median": float(np.median(per[:, 1])),
                              "warm_no_flush": warm},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": burst,
                         "unit": "TFLOP/s", "frac": achieved / burst, "traffic": traffic,
                         "kernel": "attend",
                         "frac_of_sustained": achieved / sustained,
                         "frac_per_clock_of_burst": (achieved / burst) * (sm_max / clocks["sm_mhz"])
                         if clocks.get("sm_mhz") else None,
                         "peak_note": f"{peak_kind} burst dense bf16 ({burst}; the timed region lasts "
                                      f"under a second); frac_of_sustained divides by the "
                                      f"{sustained} seconds-long figure, frac_per_clock_of_burst "
                                      f"rescales the achieved rate to {sm_max:.0f} MHz from the "
                                      f"sampled median SM clock"},
            "e2e": {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "note": "pinned host buffers; each step's H2D and D2H inside the timed region, "
                            "overlapping the neighbouring steps' kernels (two copy streams, two slots)"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "decode": dec,
        }
        gpu_configs[DECODE_WORKLOAD] = {"value": dec["terminated"]["GBps"], "unit": "GB/s",
                                        "ms": dec["terminated"]["ms"],
                                        "scope": "decode with termination on; KV bytes of the blocks "
                                                 "used / time"}
        gpu_configs[WORKLOAD] = {"value": res["value"], "unit": "TFLOP/s", "ms": step_ms,
                                 "scope": "the headline step"}
        res["kernel_paths"] = {k_: ("tensor cores" if v_ == bb.BSA_PATH_TENSOR_CORES else "CUDA cores")
                               for k_, v_ in paths.items()}
        res["configs"] = {name: {"gpu": g} for name, g in gpu_configs.items()}
        if world == 1 and not args.no_cpu:
            res["cpu_baseline"] = cpu_baseline(spec, seed)
            res["configs"][WORKLOAD]["cpu_baseline"] = res["cpu_baseline"]
            for name, e in cpu_config_baselines().items():
                res["configs"][name]["cpu_baseline"] = e
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def unmasked_pair_count(torch, kv_idx, kv_cnt, tile_q, block_k):
    """Number of (query row, key) pairs with key <= row inside the listed blocks: a block
    starting at key j0 in the tile whose first row is i0 contributes, over rows r < tile_q,
    clamp(a + r, 0, block_k) with a = i0 - j0 + 1 -- in closed form a ramp 1..block_k-1
    plus block_k for every row past it. kv_idx [B,Hq,n_qt,W] and kv_cnt [B,Hq,n_qt]."""
    W, n_qt = kv_idx.shape[-1], kv_idx.shape[-2]
    kvl = kv_idx.long()
    valid = torch.arange(W, device=kv_idx.device)[None, None, None, :] < kv_cnt[..., None]
    a = (torch.arange(n_qt, device=kv_idx.device) * tile_q)[None, None, :, None] - kvl * block_k + 1
    lo, hi = a.clamp(min=1), (a + tile_q - 1).clamp(max=block_k - 1)
    ramp = torch.where(lo <= hi, (lo + hi) * (hi - lo + 1) // 2, torch.zeros_like(a))
    flat = block_k * (a + tile_q - torch.maximum(a, torch.full_like(a, block_k))).clamp(min=0)
    return float(((ramp + flat) * valid).sum().item())


def path_rooflines(spec, score_select_ms, unfused_ms, peaks):
    """Scoring and selection against their rooflines, from the workload's shape.

    Scores: 2 * d * tile_q flops per (b, h, tile, causal block j <= J_t), the algorithmic count.
    The fused call (pool + score with in-kernel ranking + gate + finalize) must read Q and K and
    write kv_idx and kv_cnt; nothing else has to reach DRAM. It is reported against the burst
    tensor peak (flops) and against HBM (those bytes). The separate calls add the scores' round
    trip: bsa_score writes the causal scores, bsa_select reads the candidates back and writes
    kv_idx."""
    n_qt = spec.N // spec.tile_q
    causal = sum(((t + 1) * spec.tile_q - 1) // spec.block_k + 1 for t in range(n_qt))
    cand = sum((t * spec.tile_q) // spec.block_k for t in range(n_qt))
    heads = spec.B * spec.Hq
    W = min(spec.rho * max(spec.k_first, spec.k_last), spec.N // spec.block_k)
    score_flop = 2.0 * spec.d * spec.tile_q * causal * heads
    qk_bytes = heads * spec.N * spec.d * 2 + spec.B * spec.Hkv * spec.N * spec.d * 2
    kv_bytes = heads * n_qt * (W + 1) * 4
    fused_bytes = qk_bytes + kv_bytes
    score_bytes = qk_bytes + heads * causal * 4
    sel_bytes = heads * cand * 4 + heads * n_qt * W * 4
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    f_tflops = score_flop / (score_select_ms * 1e-3) / 1e12
    f_gbps = fused_bytes / (score_select_ms * 1e-3) / 1e9
    u_score, u_sel = unfused_ms["score_ms"], unfused_ms["select_ms"]
    return {
        "score_select": {"ms": score_select_ms, "algorithmic_tflop": score_flop / 1e12,
                         "tflops": f_tflops, "frac_tensor_burst": f_tflops / burst,
                         "bytes": fused_bytes, "GBps": f_gbps, "frac_hbm": f_gbps / hbm,
                         "note": "one bsa_score_select call: pool, score with the ranking in the "
                                 "same kernel (fp16 operands, one pass), gate, finalize; Q and K "
                                 "read, kv_idx and kv_cnt written"},
        "unfused": {"score_ms": u_score, "select_ms": u_sel,
                    "score_tflops": score_flop / (u_score * 1e-3) / 1e12,
                    "score_GBps": score_bytes / (u_score * 1e-3) / 1e9,
                    "select_GBps": sel_bytes / (u_sel * 1e-3) / 1e9,
                    "select_frac_hbm": sel_bytes / (u_sel * 1e-3) / 1e9 / hbm,
                    "note": "bsa_score (scores written) then bsa_select (candidate scores read back, "
                            "kv_idx written), same inputs and selection"},
    }


def _attend_sha():
    import hashlib
    h = hashlib.sha256()
    for f in sorted(os.listdir(os.path.join(ROOT, "block_sparse_causal_bsa_b200", "csrc"))):
        if f.startswith("attend"):
            h.update(open(os.path.join(ROOT, "block_sparse_causal_bsa_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def main_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return
    from block_sparse_causal_bsa_b200 import synthetic as S
    spec = S.WORKLOADS[WORKLOAD]
    seed = 1003
    n_tiles = 24
    cache = {}
    for i in range(args.warmup):
        cpu_sample(spec, seed, 2, rng_seed=100 + i, cache=cache)
    times, fl = [], []
    for i in range(args.steps):
        dt, f = cpu_sample(spec, seed, n_tiles, rng_seed=200 + i, cache=cache)
        times.append(dt)
        fl.append(f)
    val = sum(fl) / sum(times) / 1e12
    ms = 1e3 * sum(times) / len(times)
    cores = _blas_threads()
    res = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": WORKLOAD, "sample_tiles_per_step": n_tiles},
           "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores,
                            "host_cpus": os.cpu_count(), "kind": "oracle",
                            "sample": f"{n_tiles} random (b,h,t) tiles per step through the oracle's "
                                      "pool/score/rank/gate/attend"},
           "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        main_reference(args)
    else:
        main_gpu(args)


if __name__ == "__main__":
    main()
