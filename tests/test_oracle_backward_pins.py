"""Pins for the oracle's backward of the sparse branch (dQ, dK, dV over the
kept keys; the index branch's selection passes no gradient).

MSA is trained natively (cloud.tencent.com article, section 五: the index
branch gives the selection, the sparse branch computes exactly on the
selected region); the pages give no gradient formulas, so the oracle's
backward is the exact derivative of its forward.  It is pinned against torch
autograd in float64 (dense causal attention when every block is kept, and
attention restricted by an explicit kept-key mask built from the ids),
closed-form sums (softmax weights sum to 1, so per group sum_t dV_t = sum
dO and sum_t dK_t = 0), constant values (zero dQ and dK) and the index-head
map.
"""
import numpy as np
import pytest
import torch

from synthetic import bf16_bits, make_inputs


def _np(w):
    return dict(q_idx=bf16_bits(w.q_idx), k_idx=bf16_bits(w.k_idx), q=bf16_bits(w.q),
                k=bf16_bits(w.k), v=bf16_bits(w.v), lens=w.lens.numpy(),
                kv_offsets=w.kv_offsets.numpy())


def _f64(bits):
    return torch.from_numpy((bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64))


def _dout(w, seed):
    g = torch.Generator().manual_seed(seed)
    d = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
    return bf16_bits(d)


def _autograd(w, a, dout_bits, ids, n_idx):
    """torch autograd (float64) of attention restricted to the kept keys:
    mask[i, t] = t <= p_i and block(t) in the ids of row i's index head."""
    G = w.H_q // w.H_kv
    T = a["k"].shape[0]
    k = _f64(a["k"]).requires_grad_(True)
    v = _f64(a["v"]).requires_grad_(True)
    q = _f64(a["q"]).requires_grad_(True)
    dout = _f64(dout_bits)
    ids = ids.reshape(w.B, w.Sq, n_idx, -1)
    loss = 0.0
    for b in range(w.B):
        L = w.lens_host[b]
        off = int(a["kv_offsets"][b])
        pos = torch.arange(w.Sq) + (L - w.Sq)
        for g in range(w.H_kv):
            gi = g // (w.H_kv // n_idx)
            kept = torch.zeros(w.Sq, L, dtype=torch.bool)
            for i in range(w.Sq):
                for j in ids[b, i, gi]:
                    if j >= 0:
                        kept[i, w.block * int(j):min(L, w.block * (int(j) + 1))] = True
            mask = kept & (torch.arange(L)[None, :] <= pos[:, None])
            kg, vg = k[off:off + L, g], v[off:off + L, g]
            for hh in range(G):
                h = g * G + hh
                s = (q[b, :, h] @ kg.T) * w.scale
                s = s.masked_fill(~mask, float("-inf"))
                o = torch.softmax(s, dim=-1) @ vg
                loss = loss + (o * dout[b, :, h]).sum()
    loss.backward()
    return (q.grad.reshape(w.B * w.Sq, w.H_q, -1).numpy(), k.grad.numpy(), v.grad.numpy())


def _run(oracle_mod, w, a, top_k, dout_bits, n_idx=None):
    n_idx = n_idx or w.H_kv
    qi = np.ascontiguousarray(a["q_idx"][:, :, :n_idx])
    ki = np.ascontiguousarray(a["k_idx"][:, :n_idx])
    ids = oracle_mod.index_topk(qi, ki, a["lens"], a["kv_offsets"], block=w.block,
                                top_k=top_k)["block_ids"]
    dq, dk, dv = oracle_mod.sparse_attention_backward(a["q"], a["k"], a["v"], dout_bits, ids,
                                                      a["lens"], a["kv_offsets"], block=w.block,
                                                      scale=w.scale, num_index_heads=n_idx)
    return ids, dq, dk, dv


CASES = [
    # (B, Sq, lens, H_q, H_kv, D, block, top_k)
    (1, 40, [40], 4, 2, 16, 8, 8),        # every block kept: dense causal attention
    (2, 9, [30, 25], 4, 1, 8, 4, 3),      # chunked prefill, real selection
    (1, 300, [300], 8, 2, 32, 32, 4),     # ragged last block, real selection
    (2, 1, [70, 33], 6, 3, 16, 8, 3),     # decode rows
]


@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,D,block,top_k", CASES)
def test_backward_equals_autograd_on_the_kept_keys(oracle_mod, B, Sq, lens, H_q, H_kv, D, block,
                                                   top_k):
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=31 + Sq,
                    device="cpu", D=D, d_idx=D, block=block)
    a = _np(w)
    dout = _dout(w, 5)
    ids, dq, dk, dv = _run(oracle_mod, w, a, top_k, dout)
    rq, rk, rv = _autograd(w, a, dout, ids, w.H_kv)
    np.testing.assert_allclose(dq, rq, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dk, rk, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dv, rv, rtol=1e-9, atol=1e-12)


def test_backward_closed_form_sums(oracle_mod):
    """sum_t P_t = 1 per (row, head): per group, the dV rows add up to the sum
    of that group's dO, and the dK rows to zero (sum_t dZ_t = 0)."""
    w = make_inputs(B=2, Sq=20, lens=[200, 20], H_q=8, H_kv=2, top_k=3, seed=40, device="cpu",
                    D=16, d_idx=16, block=16)
    a = _np(w)
    dout = _dout(w, 6)
    _, dq, dk, dv = _run(oracle_mod, w, a, 3, dout)
    do = _f64(dout).numpy()
    for g in range(2):
        np.testing.assert_allclose(dv[:, g].sum(0), do[:, :, 4 * g:4 * g + 4].sum((0, 1, 2)),
                                   rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(dk[:, g].sum(0), 0.0, atol=1e-10)


def test_constant_values_have_no_query_or_key_gradient(oracle_mod):
    w = make_inputs(B=1, Sq=33, lens=[80], H_q=4, H_kv=2, top_k=2, seed=41, device="cpu",
                    D=16, d_idx=16, block=16)
    w.v[:] = 0.75
    a = _np(w)
    _, dq, dk, dv = _run(oracle_mod, w, a, 2, _dout(w, 7))
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12
    assert np.abs(dv).max() > 0.1


def test_backward_with_fewer_index_heads_equals_replicated_ids(oracle_mod):
    w = make_inputs(B=1, Sq=24, lens=[150], H_q=8, H_kv=4, top_k=3, seed=42, device="cpu",
                    D=16, d_idx=16, block=16)
    a = _np(w)
    dout = _dout(w, 8)
    ids2, dq2, dk2, dv2 = _run(oracle_mod, w, a, 3, dout, n_idx=2)
    ids4 = np.ascontiguousarray(np.repeat(ids2.reshape(24, 2, 3), 2, axis=1))
    dq4, dk4, dv4 = oracle_mod.sparse_attention_backward(a["q"], a["k"], a["v"], dout, ids4,
                                                         a["lens"], a["kv_offsets"], block=16,
                                                         scale=w.scale)
    np.testing.assert_array_equal(dq2, dq4)
    np.testing.assert_array_equal(dk2, dk4)
    np.testing.assert_array_equal(dv2, dv4)


def test_oracle_rows_helper_matches_full_oracle(oracle_mod):
    """oracle_rows_backward (tests/parity.py), whose split single-row calls
    the 32k-row GPU test uses, gives the same dQ, dK and dV as one
    oracle call on the whole prefill (checked on the CPU here, no GPU used)."""
    from parity import host_inputs, oracle_rows_backward
    Sq, H_q = 700, 8
    w = make_inputs(B=1, Sq=Sq, lens=[Sq], H_q=H_q, H_kv=1, top_k=3, seed=41, device="cpu")
    a = host_inputs(w)
    ids = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"],
                                top_k=w.top_k)["block_ids"]
    dout = bf16_bits(torch.randn(w.q.shape, generator=torch.Generator().manual_seed(4))
                     .to(torch.bfloat16))
    rq, rk, rv = oracle_mod.sparse_attention_backward(a["q"], a["k"], a["v"], dout, ids, a["lens"],
                                                      a["kv_offsets"], scale=w.scale)
    sq, sk, sv = oracle_rows_backward(oracle_mod, a["q"].reshape(Sq, 1, H_q, 128), a["k"],
                                      a["v"], dout.reshape(Sq, 1, H_q, 128),
                                      ids.reshape(Sq, 1, -1), np.arange(Sq), w.scale, parts=4)
    assert np.allclose(sq.reshape(rq.shape), rq, rtol=1e-12, atol=1e-12)
    assert np.allclose(sk, rk, rtol=1e-10, atol=1e-12)
    assert np.allclose(sv, rv, rtol=1e-10, atol=1e-12)
