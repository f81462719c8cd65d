"""The FLOP counts bench.py divides by, checked on the CPU against a direct
count over every (row, group, kept block) of small selections."""
import os
import sys
from types import SimpleNamespace

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def _direct_useful(w, ids):
    keys = 0
    for b in range(w.B):
        L = w.lens_host[b]
        for i in range(w.Sq):
            p = L - w.Sq + i
            for g in range(w.H_kv):
                for j in ids[b, i, g]:
                    if j < 0:
                        continue
                    keys += min(128, p - 128 * int(j) + 1)     # visible tokens of block j
    return keys * (w.H_q // w.H_kv) * 4 * w.D


def test_prefill_useful_flops_matches_a_direct_count():
    bench = _bench()
    rng = np.random.default_rng(3)
    for B, Sq, lens, H_q, H_kv, K in ((1, 300, [300], 8, 2, 4), (2, 64, [500, 64], 16, 4, 3),
                                     (1, 1000, [1000], 64, 8, 16)):
        w = SimpleNamespace(B=B, Sq=Sq, lens_host=lens, H_q=H_q, H_kv=H_kv, top_k=K, D=128,
                            d_idx=128)
        ids = np.full((B, Sq, H_kv, K), -1, np.int32)
        for b in range(B):
            for i in range(Sq):
                own = (lens[b] - Sq + i) // 128
                for g in range(H_kv):
                    cand = rng.permutation(own)[:K - 1] if own > 0 else np.array([], np.int64)
                    sel = np.sort(np.append(cand, own))
                    ids[b, i, g, :sel.size] = sel
        assert bench.prefill_useful_flops(w, ids) == _direct_useful(w, ids)


def test_prefill_index_flops_counts_the_causal_product():
    bench = _bench()
    w = SimpleNamespace(B=2, Sq=5, lens_host=[5, 9], H_kv=3, d_idx=128)
    # row i of sequence b sees positions 0 .. L - Sq + i
    visible = sum(L - 5 + i + 1 for L in (5, 9) for i in range(5))
    assert bench.prefill_index_flops(w) == visible * 3 * 2 * 128
