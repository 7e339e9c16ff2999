"""A small case of the benchmark's kernels, sized for Nsight Compute captures.

Runs the gated prefill path (score -> select -> attend) on the gated workload
shrunk to N tokens (default 16384: Q is 134 MB, above the 126 MB L2, so DRAM
counters still mean something, while the whole case holds ~0.4 GB on the
device), then optionally the decode path on a shortened cache.

With --select-only the scores are computed once, Q, K and V are released, and
only the selection runs (--iters times): at --n 131072 --heads 16 this is the
full-length selection of half the heads (134 MB of scores, ~0.2 GB held).
With --score-select only the scoring+selection call runs (--iters times), as the
benchmark's step calls it (ranking inside the score kernel, no scores written).

    python -m block_sparse_causal_bsa_b200.profcase [--n 16384] [--heads 32] [--iters 2]
                                                    [--decode-len 8192] [--select-only]
                                                    [--score-select]
"""
from __future__ import annotations

import argparse
import ctypes
import math

import numpy as np
import torch

from . import binding as bb
from . import synthetic as S


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--n", type=int, default=16384)
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--decode-len", type=int, default=0)
    ap.add_argument("--heads", type=int, default=32)
    ap.add_argument("--select-only", action="store_true")
    ap.add_argument("--score-select", action="store_true")
    a = ap.parse_args()
    spec = S.WORKLOADS["gated_prefill_128k"].scaled(N=a.n, Hq=a.heads, Hkv=max(1, a.heads // 4))
    q, k, v = S.prefill_inputs(spec, 7)
    qd, kd, vd = _dev(q), _dev(k), _dev(v)
    cfg = bb.SelectConfig(spec.k_first, spec.k_last, spec.rho, spec.gate_quantile)
    if a.select_only:
        scores = bb.score(qd, kd, block_k=spec.block_k, tile_q=spec.tile_q)
        shape = bb.make_shape(qd, kd, spec.block_k, spec.tile_q)
        del qd, kd, vd
        torch.cuda.empty_cache()
        for _ in range(a.iters):
            sel = bb.select(scores, shape=shape, cfg=cfg)
        torch.cuda.synchronize()
        status = int(sel["dev_status"].item())
        print(f"select N={a.n} Hq={a.heads}: selected blocks {int(sel['kv_cnt'].sum())}, status {status}")
        if status:
            raise SystemExit(f"device status {status}")
        return
    if a.score_select:
        for _ in range(a.iters):
            sel = bb.score_select(qd, kd, vd, block_k=spec.block_k, tile_q=spec.tile_q, cfg=cfg,
                                  want_scores=False)
        torch.cuda.synchronize()
        status = int(sel["dev_status"].item())
        print(f"score_select N={a.n} Hq={a.heads}: selected blocks {int(sel['kv_cnt'].sum())}, status {status}")
        if status:
            raise SystemExit(f"device status {status}")
        return
    for _ in range(a.iters):
        out, sel, st = bb.prefill(qd, kd, vd, block_k=spec.block_k, tile_q=spec.tile_q, cfg=cfg)
    torch.cuda.synchronize()
    status = int(st.item()) | int(sel["dev_status"].item()) | int(sel["score_status"].item())
    print(f"prefill N={a.n}: selected blocks {int(sel['kv_cnt'].sum())}, status {status}")
    if a.decode_len:
        d = S.DECODE_WORKLOADS["decode_art_64k"].scaled(L=a.decode_len)
        dq, dk, dv = S.decode_inputs(d, 8)
        for _ in range(a.iters):
            o, used, _, st2 = bb.decode(_dev(dq), _dev(dk), _dev(dv), block_kv=d.block_kv, tau=d.tau,
                                        phi=d.phi, patience=d.patience,
                                        probe_dims=S.default_probe_dims(32))
        torch.cuda.synchronize()
        print(f"decode L={a.decode_len}: mean blocks used {float(used.float().mean()):.1f}, "
              f"status {int(st2.item())}")
        status |= int(st2.item())
    if status:
        raise SystemExit(f"device status {status}")


if __name__ == "__main__":
    main()
