"""The parity checker itself (tests/parity.py), on the CPU: it accepts the
oracle's own results, and it rejects a wrong block score, a wrong id and a
wrong output.  The GPU tests lean on it, so a checker that let everything
through would make them meaningless."""
import numpy as np
import pytest

from parity import compare, compare_index, host_inputs
from synthetic import make_inputs


@pytest.fixture(scope="module")
def case(oracle_mod):
    w = make_inputs(B=2, Sq=3, lens=[700, 1000], H_q=8, H_kv=2, top_k=3, seed=11, device="cpu")
    a = host_inputs(w)
    ref = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"],
                                top_k=w.top_k)
    out = oracle_mod.sparse_attention(a["q"], a["k"], a["v"], ref["block_ids"], a["lens"],
                                      a["kv_offsets"], scale=w.scale)
    return w, a, ref["block_ids"], ref["block_scores"], out


def test_checker_accepts_the_oracle(oracle_mod, case):
    w, a, ids, sc, out = case
    rep = compare(oracle_mod, w, ids.copy(), sc.copy(), out.astype(np.float32), host=a)
    assert rep["near_ties"] == 0 and rep["score_err"] == 0.0


def test_checker_rejects_a_score_off_by_1e_3(oracle_mod, case):
    w, a, ids, sc, out = case
    bad = sc.copy()
    bad[1, 0, 1] += 1e-3 * max(1.0, abs(float(bad[1, 0, 1])))
    with pytest.raises(AssertionError, match="block scores"):
        compare_index(oracle_mod, w, ids, bad, host=a)


def test_checker_rejects_a_swapped_id(oracle_mod, case):
    w, a, ids, sc, out = case
    bad = ids.copy()
    r, g = 4, 1
    own = bad[r, g].max()
    cand = [j for j in range(own) if j not in bad[r, g]]
    bad[r, g, 0] = cand[0]
    bad[r, g].sort()
    with pytest.raises(AssertionError, match="block ids differ"):
        compare_index(oracle_mod, w, bad, sc, host=a)


def test_checker_rejects_a_wrong_output(oracle_mod, case):
    w, a, ids, sc, out = case
    bad = out.astype(np.float32).copy()
    bad[2, 5, 7] += 0.05
    with pytest.raises(AssertionError, match="max-abs"):
        compare(oracle_mod, w, ids, sc, bad, host=a)
