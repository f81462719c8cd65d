"""GPU parity of the sparse branch's backward (dQ, dK, dV over the kept
blocks) through the C ABI against the CPU oracle's exact derivative, on the
same bf16 inputs and the same selection.

Tolerance: relative L2 <= 5e-3 (the forward's bound) and max-abs <= 2 % of
the largest reference magnitude, per gradient.  The kernel rounds P to bf16
(the operand of dV = P^T dO, and the P that dS = P (dP - Delta) is formed
from) and dS to bf16 (the operand of dK and dQ): at most 2^-9 relative each,
about 1.1e-3 RMS for round-to-nearest, about 1.6e-3 for dS's two roundings;
Delta = dO.O is taken from the recomputed bf16 output, whose error enters dS
only scaled by |O| / |v| < 1; dQ is written as bf16 (another 1.1e-3).  dK and
dV are fp32 sums of those products, so the rounding adds in quadrature to
about 2-2.5e-3 RMS, inside 5e-3.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_43_b200 as m

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL_L2 = 5e-3
MAX_ABS_FRAC = 2e-2


def _check(name, got, ref):
    got = np.asarray(got, np.float64)
    assert np.isfinite(got).all(), f"{name}: non-finite"
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(got - ref).max()
    assert err <= REL_L2, f"{name}: rel-L2 {err}"
    assert mx <= MAX_ABS_FRAC * max(np.abs(ref).max(), 1e-6), f"{name}: max-abs {mx}"
    return err


def _run(oracle_mod, w, n_idx=None, padded_nan=False):
    from synthetic import bf16_bits
    n_idx = n_idx or w.H_kv
    q_idx = w.q_idx[:, :, :n_idx].contiguous()
    k_idx = w.k_idx[:, :n_idx].contiguous()
    eng = m.MSA(batch=w.B, q_len=w.Sq, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=DEV,
                num_index_heads=n_idx)
    eng.index_topk(q_idx, k_idx, w.lens, w.kv_offsets)
    g = torch.Generator(device=DEV).manual_seed(77)
    dout = torch.randn(w.q.shape, generator=g, device=DEV).to(torch.bfloat16)
    dq = torch.empty_like(w.q)
    dk = torch.zeros(w.k.shape, dtype=torch.float32, device=DEV)
    dv = torch.zeros(w.v.shape, dtype=torch.float32, device=DEV)
    ws = m.alloc_workspace(m.msa_sparse_attention_backward_workspace_size(eng.shape), DEV)
    m.msa_sparse_attention_backward(eng.shape, w.q, w.k, w.v, eng.block_ids, w.lens,
                                    w.kv_offsets, w.scale, dout, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(ws) == 0
    ids = eng.block_ids.cpu().numpy()
    k_host, v_host = bf16_bits(w.k), bf16_bits(w.v)
    if padded_nan:
        # the oracle reads only tokens < lens; NaN padding becomes 0 in its copy
        k_host = np.where(np.isnan(w.k.float().cpu().numpy()), 0, k_host).astype(np.uint16)
        v_host = np.where(np.isnan(w.v.float().cpu().numpy()), 0, v_host).astype(np.uint16)
    rq, rk, rv = oracle_mod.sparse_attention_backward(
        bf16_bits(w.q), k_host, v_host, bf16_bits(dout), ids, w.lens.cpu().numpy(),
        w.kv_offsets.cpu().numpy(), scale=w.scale, num_index_heads=n_idx)
    gq = dq.float().cpu().numpy().reshape(rq.shape)
    gk, gv = dk.cpu().numpy(), dv.cpu().numpy()
    rep = dict(dq=_check("dq", gq, rq), dk=_check("dk", gk, rk), dv=_check("dv", gv, rv))
    # keys no row kept get no gradient at all
    untouched = (rk == 0).all(axis=-1) & (rv == 0).all(axis=-1)
    assert (gk[untouched] == 0).all() and (gv[untouched] == 0).all()
    return rep


CASES = [
    # (B, Sq, lens, H_q, H_kv, top_k)
    (1, 2048, [2048], 8, 2, 4),            # the 2k-row prefill shape
    (1, 300, [300], 8, 2, 4),              # full prefill, ragged last block
    (2, 64, [500, 64], 16, 4, 3),          # chunked prefill after a cached prefix
    (1, 1000, [1000], 64, 8, 16),          # groups of 8, every block kept
    (1, 700, [700], 32, 2, 4),             # groups of 16 (two n8 tiles)
    (3, 1, [5000, 129, 2000], 16, 2, 8),   # decode rows
    (1, 2000, [2000], 8, 8, 16),           # one head per group (7 padding heads)
]


@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,top_k", CASES)
def test_backward_matches_oracle(oracle_mod, B, Sq, lens, H_q, H_kv, top_k):
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=700 + Sq,
                    device=DEV)
    print((B, Sq, H_q, H_kv, top_k), _run(oracle_mod, w))


def test_backward_with_fewer_index_heads(oracle_mod):
    from synthetic import make_inputs
    w = make_inputs(B=1, Sq=600, lens=[600], H_q=64, H_kv=8, top_k=4, seed=71, device=DEV)
    print(_run(oracle_mod, w, n_idx=2))


def test_backward_ignores_nan_padding(oracle_mod):
    """Padded cache (offset b*4096) with NaN past each length: nothing past a
    sequence's query position may reach a gradient."""
    from synthetic import make_inputs
    lens = [1000, 300]
    w = make_inputs(B=2, Sq=300, lens=lens, H_q=16, H_kv=2, top_k=4, seed=72, device=DEV,
                    padded_to=1024)
    for t in (w.k, w.v):
        for b, L in enumerate(lens):
            t[b * 1024 + L:(b + 1) * 1024] = float("nan")
    print(_run(oracle_mod, w, padded_nan=True))


def test_backward_32k_rows_sampled(oracle_mod):
    """Groups of 8 at 32,768 rows (the 128k prefill recipe at a quarter of its
    length): dK and dV of whole key blocks, and dQ of the rows that reach
    them, against the oracle.  A row's gradient terms depend only on its own
    q, dO and kept blocks, so the rows that kept block j in group g, run
    through the oracle as single-row sequences (length = position + 1) over
    the same cache, give block j's exact dK and dV in group g."""
    from parity import oracle_rows_backward
    from synthetic import bf16_bits, make_inputs
    Sq, H_q, H_kv, G = 32768, 64, 8, 8
    w = make_inputs(B=1, Sq=Sq, lens=[Sq], H_q=H_q, H_kv=H_kv, top_k=16, seed=732, device=DEV)
    eng = m.MSA(batch=1, q_len=Sq, max_kv_len=Sq, num_q_heads=H_q, num_kv_heads=H_kv, top_k=16,
                kv_capacity=w.kv_capacity, device=DEV)
    eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets)
    g = torch.Generator(device=DEV).manual_seed(78)
    dout = torch.randn(w.q.shape, generator=g, device=DEV).to(torch.bfloat16)
    dq = torch.empty_like(w.q)
    dk = torch.zeros(w.k.shape, dtype=torch.float32, device=DEV)
    dv = torch.zeros(w.v.shape, dtype=torch.float32, device=DEV)
    ws = m.alloc_workspace(m.msa_sparse_attention_backward_workspace_size(eng.shape), DEV)
    m.msa_sparse_attention_backward(eng.shape, w.q, w.k, w.v, eng.block_ids, w.lens,
                                    w.kv_offsets, w.scale, dout, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(ws) == 0
    ids = eng.block_ids.cpu().numpy().reshape(Sq, H_kv, 16)
    qh = bf16_bits(w.q).reshape(Sq, H_q, 128)
    dh = bf16_bits(dout).reshape(Sq, H_q, 128)
    kh, vh = bf16_bits(w.k), bf16_bits(w.v)
    gq = dq.float().cpu().numpy().reshape(Sq, H_q, 128)
    gk, gv = dk.cpu().numpy(), dv.cpu().numpy()
    # the last block (its own rows only), a late block and an earlier one
    for grp, j in [(0, 255), (3, 200), (7, 150)]:
        rows = np.nonzero((ids[:, grp, :] == j).any(axis=1))[0]
        n = rows.size
        hs = slice(grp * G, (grp + 1) * G)
        rq, rk, rv = oracle_rows_backward(oracle_mod, qh[rows, hs][:, None].copy(),
                                  kh[:, grp:grp + 1].copy(), vh[:, grp:grp + 1].copy(),
                                  dh[rows, hs][:, None].copy(), ids[rows, grp][:, None, :].copy(),
                                  rows, w.scale)
        t = slice(j * 128, (j + 1) * 128)
        rep = dict(rows=n, dk=_check(f"dk[{j},{grp}]", gk[t, grp], rk[t, 0]),
                   dv=_check(f"dv[{j},{grp}]", gv[t, grp], rv[t, 0]),
                   dq=_check(f"dq[rows of {j},{grp}]", gq[rows, hs], rq.reshape(n, G, 128)))
        print(grp, j, rep)


@pytest.mark.parametrize("H_q,H_kv", [(64, 8), (16, 4)])
def test_backward_bad_lengths(oracle_mod, H_q, H_kv):
    """A sequence whose length is out of range: the call raises the status
    word, writes NaN into that sequence's dq and leaves its keys' dk, dv
    alone; the other sequence's gradients still match the oracle."""
    from synthetic import bf16_bits, make_inputs
    w = make_inputs(B=2, Sq=300, lens=[600, 900], H_q=H_q, H_kv=H_kv, top_k=4, seed=74,
                    device=DEV)
    eng = m.MSA(batch=2, q_len=300, max_kv_len=900, num_q_heads=H_q, num_kv_heads=H_kv, top_k=4,
                kv_capacity=w.kv_capacity, device=DEV)
    eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets)
    g = torch.Generator(device=DEV).manual_seed(79)
    dout = torch.randn(w.q.shape, generator=g, device=DEV).to(torch.bfloat16)
    dq = torch.empty_like(w.q)
    dk = torch.zeros(w.k.shape, dtype=torch.float32, device=DEV)
    dv = torch.zeros(w.v.shape, dtype=torch.float32, device=DEV)
    ws = m.alloc_workspace(m.msa_sparse_attention_backward_workspace_size(eng.shape), DEV)
    bad = torch.tensor([600, 5000], dtype=torch.int32, device=DEV)     # 5000 > max_kv_len
    m.msa_sparse_attention_backward(eng.shape, w.q, w.k, w.v, eng.block_ids, bad, w.kv_offsets,
                                    w.scale, dout, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(ws) == 6
    gq = dq.float().cpu().numpy()
    assert np.isnan(gq[1]).all() and np.isfinite(gq[0]).all()
    offs = w.kv_offsets.cpu().numpy()
    gk, gv = dk.cpu().numpy(), dv.cpu().numpy()
    assert (gk[offs[1]:] == 0).all() and (gv[offs[1]:] == 0).all()
    ids = eng.block_ids.cpu().numpy()
    rq, rk, rv = oracle_mod.sparse_attention_backward(
        bf16_bits(w.q)[:1], bf16_bits(w.k), bf16_bits(w.v), bf16_bits(dout)[:1], ids[:1],
        np.array([600], np.int32), offs[:1], scale=w.scale)
    _check("dq", gq[0].reshape(rq.shape), rq)
    _check("dk", gk, rk)
    _check("dv", gv, rv)
