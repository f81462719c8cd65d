"""GPU parity of the fused decode step (msa_decode_step: index branch, top-k
and sparse branch in one cooperative launch) through the C ABI.

Checked against the CPU oracle with the tolerances of tests/parity.py, and
against the two-call path (msa_index_topk + msa_sparse_attention) on the same
inputs: the fused kernel scores tokens with the same fp32 arithmetic, so its
block ids and block scores must be bit-identical to the two-call path's; its
output combines the kept blocks' partial sums in another order, so it is held
to the oracle's output tolerance only.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_43_b200 as m

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fused(w, eng=None):
    eng = eng or m.MSA(batch=w.B, q_len=1, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                       num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity,
                       device=DEV)
    eng.decode_step(w.q_idx, w.k_idx, w.q, w.k, w.v, w.lens, w.kv_offsets)
    torch.cuda.synchronize()
    st = m.msa_read_device_status(eng.ws_step)
    return eng, st


def _run_and_compare(oracle_mod, w, rows=None):
    from parity import compare, run_gpu, to_host
    eng, st = _fused(w)
    assert st == 0, f"device status {st}"
    ids, sc, out = to_host(eng)
    ref, st2 = run_gpu(w)
    assert st2 == 0
    r_ids, r_sc, r_out = to_host(ref)
    np.testing.assert_array_equal(ids, r_ids)
    np.testing.assert_array_equal(sc, r_sc)
    rep = compare(oracle_mod, w, ids, sc, out, rows=rows)
    rep["vs_two_call_max_abs"] = float(np.abs(out - r_out).max())
    return rep


# (B, lens, H_q, H_kv, top_k): ragged lengths, a block-aligned length, fewer
# blocks than k, a single token, one group, 16 groups, group sizes 1..16.
CASES = [
    (3, [5000, 128, 1], 16, 2, 4),
    (2, [4096, 4097], 64, 8, 16),
    (4, [700, 2047, 129, 3000], 8, 8, 16),
    (1, [20000], 8, 1, 16),
    (2, [9000, 15000], 16, 16, 16),
    (2, [6000, 6001], 16, 4, 1),
    (1, [3 * 128 + 5], 8, 8, 16),
    (7, [300, 129000, 5, 4096, 77777, 1024, 65], 32, 4, 64),
    (3, [9000, 129, 40000], 32, 2, 16),                # groups of 16 (two n8 tiles)
    (2, [5000, 300], 128, 8, 8),                       # groups of 16, 8 groups
]


@pytest.mark.parametrize("B,lens,H_q,H_kv,top_k", CASES)
def test_decode_step_small_shapes(oracle_mod, B, lens, H_q, H_kv, top_k):
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=1, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=501 + B,
                    device=DEV, needles=3, amp=4.0)
    print((B, H_q, H_kv, top_k), _run_and_compare(oracle_mod, w))


@pytest.mark.parametrize("name", ["decode_32k", "decode_ragged", "decode_1m"])
def test_decode_step_named_workloads(oracle_mod, name):
    """The decode workloads at full size, in the configuration the benchmark
    times, every row compared."""
    from synthetic import make_workload
    w = make_workload(name, DEV)
    print(name, _run_and_compare(oracle_mod, w))


def test_decode_step_padded_cache_with_nan(oracle_mod):
    """Padded layout with NaN past each length: no padding token may reach a
    score or an output."""
    from synthetic import make_inputs
    lens = [3000, 129, 4096, 1000]
    w = make_inputs(B=4, Sq=1, lens=lens, H_q=64, H_kv=8, top_k=16, seed=8, device=DEV,
                    padded_to=4096)
    for t in (w.k_idx, w.k, w.v):
        for b, L in enumerate(lens):
            t[b * 4096 + L:(b + 1) * 4096] = float("nan")
    print(_run_and_compare(oracle_mod, w))


def test_decode_step_repeat_calls():
    """Selection bit-identical on every call; the output may differ only in
    the merge order of the kept blocks, within bf16 rounding."""
    from synthetic import make_inputs
    w = make_inputs(B=5, Sq=1, lens=[9000, 3001, 17000, 128, 40000], H_q=64, H_kv=8, top_k=16,
                    seed=22, device=DEV)
    eng, st = _fused(w)
    assert st == 0
    a = (eng.block_ids.clone(), eng.block_scores.clone(), eng.out.float().clone())
    for _ in range(3):
        _, st = _fused(w, eng)
        assert st == 0
        assert torch.equal(a[0], eng.block_ids) and torch.equal(a[1], eng.block_scores)
        assert (a[2] - eng.out.float()).abs().max().item() <= 2e-2


def test_decode_step_bad_lengths(oracle_mod):
    """A length past max_kv_len: that sequence gets -1 / -inf / NaN and the
    status word; the others are still computed correctly."""
    from parity import compare
    from synthetic import make_inputs
    w = make_inputs(B=3, Sq=1, lens=[1000, 2000, 3000], H_q=16, H_kv=2, top_k=4, seed=6,
                    device=DEV)
    eng = m.MSA(batch=3, q_len=1, max_kv_len=3000, num_q_heads=16, num_kv_heads=2, top_k=4,
                kv_capacity=w.kv_capacity, device=DEV)
    bad = torch.tensor([1000, 4000, 3000], dtype=torch.int32, device=DEV)
    eng.decode_step(w.q_idx, w.k_idx, w.q, w.k, w.v, bad, w.kv_offsets)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(eng.ws_step) == 6
    ids = eng.block_ids.cpu()
    assert (ids[1] == -1).all()
    assert torch.isnan(eng.out[1].float()).all()
    compare(oracle_mod, w, ids.numpy(), eng.block_scores.cpu().numpy(),
            eng.out.float().cpu().numpy(), rows=[0, 2])



# (B, lens, H_q, H_kv, Hi, top_k): fewer index heads than groups (bf16 keys,
# one row per index head); group g uses index head g / (H_kv / Hi).
FEWER_INDEX_HEADS = [
    (2, [4096, 300], 64, 8, 4, 16),         # the guide's 4 index heads for 8 groups
    (4, [700, 2047, 129, 3000], 16, 8, 2, 8),
    (3, [9000, 1, 20000], 16, 4, 1, 16),
]


@pytest.mark.parametrize("B,lens,H_q,H_kv,Hi,top_k", FEWER_INDEX_HEADS)
def test_decode_step_fewer_index_heads(oracle_mod, B, lens, H_q, H_kv, Hi, top_k):
    """The fused step with Hi < H_kv index heads: ids and scores bit-identical
    to msa_index_topk with the same heads, outputs against the oracle run on
    that selection."""
    from parity import compare
    from synthetic import bf16_bits, make_inputs
    w = make_inputs(B=B, Sq=1, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=61 + Hi,
                    device=DEV)
    q_idx = w.q_idx[:, :, :Hi].contiguous()
    keys = w.k_idx[:, :Hi].contiguous()
    kw = dict(batch=B, q_len=1, max_kv_len=max(lens), num_q_heads=H_q, num_kv_heads=H_kv,
              top_k=top_k, kv_capacity=w.kv_capacity, device=DEV, num_index_heads=Hi)
    fused = m.MSA(**kw)
    fused.decode_step(q_idx, keys, w.q, w.k, w.v, w.lens, w.kv_offsets)
    two = m.MSA(**kw)
    two.index_topk(q_idx, keys, w.lens, w.kv_offsets)
    two.sparse_attention(w.q, w.k, w.v, w.lens, w.kv_offsets)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(fused.ws_step) == 0
    assert two.device_status() == 0
    ids, sc = fused.block_ids.cpu().numpy(), fused.block_scores.cpu().numpy()
    assert ids.shape[2] == Hi
    np.testing.assert_array_equal(ids, two.block_ids.cpu().numpy())
    np.testing.assert_array_equal(sc, two.block_scores.cpu().numpy())
    host = dict(q_idx=bf16_bits(q_idx), k_idx=bf16_bits(keys), q=bf16_bits(w.q),
                k=bf16_bits(w.k), v=bf16_bits(w.v), lens=w.lens.cpu().numpy(),
                kv_offsets=w.kv_offsets.cpu().numpy())
    rep = compare(oracle_mod, w, ids, sc, fused.out.float().cpu().numpy(), host=host)
    print("fused fewer index heads", (B, H_q, H_kv, Hi, top_k), rep)
