"""Decode over a block list (bsa_decode_list) against the oracle.

Each (batch, KV head) visits the blocks of its list in list order ([ART] 2.4:
first block first, then e.g. most recent first, or a selector's subset). As for
the in-order decode: the stop step must equal the oracle's decision on the
GPU's own probe trace (bit-exact), the output must match attention over exactly
the visited blocks (2e-2 / 1e-3), and the oracle's own end-to-end stop step is
compared too.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_causal_bsa_b200 import binding as bb
from block_sparse_causal_bsa_b200 import synthetic as S
from oracle import bsa_oracle as O

from gpu_util import check_attend, out_rows, to_dev

pytestmark = pytest.mark.gpu


def _run(spec, seed, lists, cnt, tau, phi, patience, enable=True, expect_status=0):
    q, k, v = S.decode_inputs(spec, seed)
    dims = S.default_probe_dims(32 if spec.d == 128 else 16)
    scale = 1.0 / math.sqrt(spec.d)
    out, used, trace, st = bb.decode(to_dev(q), to_dev(k), to_dev(v), block_kv=spec.block_kv,
                                     tau=tau, phi=phi, patience=patience, enable=enable,
                                     probe_dims=dims, want_trace=True,
                                     block_list=torch.from_numpy(lists).cuda(),
                                     list_cnt=torch.from_numpy(cnt).cuda())
    torch.cuda.synchronize()
    assert int(st.item()) == expect_status
    used, trace, go = used.cpu().numpy(), trace.cpu().numpy(), out_rows(out)
    G = spec.Hq // spec.Hkv
    nb = spec.L // spec.block_kv
    agree = 0
    for b in range(spec.B):
        for g in range(spec.Hkv):
            raw = lists[b, g, :max(0, min(int(cnt[b, g]), lists.shape[-1]))]   # the list as given
            steps = O.decode_visit_steps(raw, nb)        # the oracle's visit sequence
            u = int(used[b, g])
            n = len(steps)
            exp = (O.termination_block(trace[b, g], tau, phi, patience, n_blocks=n)
                   if enable and n > 0 else n)
            assert u == exp, (b, g, u, exp)
            qg = q[b, g * G:(g + 1) * G]
            # output after the GPU's u visit steps: the shortest prefix of the raw list
            # holding u visit steps, through the oracle (which skips the bad entries itself)
            pre = next(i for i in range(len(raw) + 1) if len(O.decode_visit_steps(raw[:i], nb)) == u)
            o_ref, u_pre, _ = O.decode_group_list(qg, k[b, g], v[b, g], spec.block_kv, scale,
                                                  raw[:pre], tau, phi, patience, dims, enable=False)
            assert u_pre == u
            check_attend(go[b, g * G:(g + 1) * G], o_ref)
            _, u_ref, tr_ref = O.decode_group_list(qg, k[b, g], v[b, g], spec.block_kv, scale,
                                                   raw, tau, phi, patience, dims, enable=enable)
            agree += int(u_ref == u)
            m = min(u, u_ref)
            np.testing.assert_allclose(trace[b, g, :m], tr_ref[:m], atol=2e-3)
    return used, agree


@pytest.mark.parametrize("kind,keep", [("recency", 0), ("subset", 24)])
def test_decode_list_tensor_core(kind, keep):
    spec = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=2, L=8192)
    lists, cnt = S.decode_block_lists(spec, 1401, kind, keep)
    used, agree = _run(spec, 1402, lists, cnt, spec.tau, spec.phi, spec.patience)
    assert agree >= 0.8 * spec.B * spec.Hkv


@pytest.mark.parametrize("Hq,Hkv,d,bkv", [(4, 4, 64, 64), (8, 4, 128, 64)])
def test_decode_list_cuda_core(Hq, Hkv, d, bkv):
    spec = S.DecodeSpec("dec", B=2, Hq=Hq, Hkv=Hkv, L=2048, d=d, block_kv=bkv, tau=1e-2,
                        phi=1e-3, patience=2)
    lists, cnt = S.decode_block_lists(spec, 1403, "subset", keep=12)
    _run(spec, 1404, lists, cnt, spec.tau, spec.phi, spec.patience)


def test_decode_list_full_pass_and_limits():
    spec = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=1, L=4096)
    lists, cnt = S.decode_block_lists(spec, 1405, "subset", keep=10)
    used, _ = _run(spec, 1406, lists, cnt, 0.0, 0.0, 1)
    assert (used == 10).all()                        # never stable: every listed block
    used, _ = _run(spec, 1406, lists, cnt, float("inf"), float("inf"), 3)
    assert (used == 4).all()                         # stable every time: p + 1 steps
    used, _ = _run(spec, 1406, lists, cnt, 1e-3, 1e-4, 1, enable=False)
    assert (used == 10).all()


def test_decode_list_bad_entries_and_empty():
    spec = S.DECODE_WORKLOADS["decode_art_64k"].scaled(B=1, L=4096, Hkv=4, Hq=16)
    lists, cnt = S.decode_block_lists(spec, 1407, "subset", keep=8)
    lists[0, 0, 3] = 32                              # one past the last block
    lists[0, 1, 5] = -7
    cnt[0, 2] = 0                                    # empty list: output 0, nothing used
    cnt[0, 3] = 5                                    # entries beyond the count are ignored
    lists[0, 3, 6] = 99
    used, _ = _run(spec, 1408, lists, cnt, 0.0, 0.0, 1, expect_status=bb.BSA_DEV_BAD_INDEX)
    assert used[0].tolist() == [7, 7, 0, 5]
