"""Pins for the CPU oracle: each test checks the oracle against something other
than itself (a library attention routine, brute force, a closed form or an
invariant), chosen so that a dropped term, a wrong sign or index, a transposed
operand, a missing scale or a reversed tie rule fails at least one of them.

The method (MiniMax Sparse Attention, per the cloud.tencent.com article,
sections 二 and 六, and the mlqm.cn guide's configuration passage): one index
query per GQA group, dotted with each visible index key, max-pooled per block,
top-k blocks (own block kept, ties to the lower id), then exact softmax
attention over the kept blocks, shared by the group's heads.
"""
import math

import numpy as np
import pytest
import torch

from synthetic import bf16_bits, make_inputs


def _np_inputs(w):
    return dict(q_idx=bf16_bits(w.q_idx), k_idx=bf16_bits(w.k_idx), q=bf16_bits(w.q),
                k=bf16_bits(w.k), v=bf16_bits(w.v), lens=w.lens.numpy(),
                kv_offsets=w.kv_offsets.numpy())


def _f64(bits):
    return torch.from_numpy(bits.astype(np.uint32) << 16).view(torch.float32).double()


def _sdpa_rows(w, mask_fn):
    """Attention through torch's own scaled_dot_product_attention in float64,
    with a caller-given boolean mask [Sq, L] per sequence (True = attend).
    Returns [B*Sq, H_q, D]."""
    a = _np_inputs(w)
    G = w.H_q // w.H_kv
    outs = []
    for b in range(w.B):
        L = w.lens_host[b]
        off = int(a["kv_offsets"][b])
        q = _f64(a["q"][b]).permute(1, 0, 2)                         # [H_q, Sq, D]
        k = _f64(a["k"][off:off + L]).permute(1, 0, 2).repeat_interleave(G, 0)
        v = _f64(a["v"][off:off + L]).permute(1, 0, 2).repeat_interleave(G, 0)
        pos = torch.arange(w.Sq) + (L - w.Sq)
        mask = mask_fn(pos[:, None], torch.arange(L)[None, :])
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                              scale=w.scale)
        outs.append(o.permute(1, 0, 2))
    return torch.cat(outs, 0).numpy()


def _oracle_run(oracle_mod, w, top_k, **kw):
    a = _np_inputs(w)
    sel = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"],
                                block=w.block, top_k=top_k, want_all_scores=True)
    out, ws = oracle_mod.sparse_attention(a["q"], a["k"], a["v"], sel["block_ids"], a["lens"],
                                          a["kv_offsets"], block=w.block, scale=w.scale,
                                          want_wsum=True)
    return sel, out, ws


SMALL = [
    # (B, Sq, lens, H_q, H_kv, D, block)
    (1, 40, [40], 4, 2, 16, 8),          # prefill, 5 blocks
    (2, 1, [37, 64], 6, 3, 16, 8),       # decode, ragged (37 is not block-aligned)
    (2, 9, [30, 25], 4, 1, 8, 4),        # chunked prefill: last 9 rows of each sequence
    (1, 300, [300], 8, 2, 128, 128),     # method's own dims, ragged last block
]


@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,D,block", SMALL)
def test_p1_full_selection_equals_dense_causal_attention(oracle_mod, B, Sq, lens, H_q, H_kv,
                                                        D, block):
    """P1: when k >= number of blocks every visible block is kept, so MSA's
    sparse branch must equal plain causal attention (library routine)."""
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=1, seed=11, device="cpu",
                    D=D, d_idx=D, block=block)
    k_big = max(-(-L // block) for L in lens)
    sel, out, _ = _oracle_run(oracle_mod, w, k_big)
    ref = _sdpa_rows(w, lambda p, t: t <= p)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    assert (sel["block_ids"] >= -1).all()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_p2_selection_equals_brute_force_sort(oracle_mod, seed):
    """P2: on tiny inputs the kept set equals a brute-force full sort of every
    block score (numpy scores, Python sort on (-score, id)), own block forced."""
    B, Sq, L, H_kv, D, blk, K = 1, 61, 61, 2, 16, 4, 5
    w = make_inputs(B=B, Sq=Sq, lens=[L], H_q=2, H_kv=H_kv, top_k=K, seed=seed, device="cpu",
                    D=D, d_idx=D, block=blk)
    a = _np_inputs(w)
    sel = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"], block=blk,
                                top_k=K)
    qi = _f64(a["q_idx"][0]).numpy()          # [Sq, H_kv, D]
    ki = _f64(a["k_idx"]).numpy()             # [L, H_kv, D]
    for i in range(Sq):
        for g in range(H_kv):
            s = ki[:, g, :] @ qi[i, g, :]
            nb = i // blk + 1
            S = [max(s[t] for t in range(j * blk, min((j + 1) * blk, i + 1))) for j in range(nb)]
            own = nb - 1
            if nb <= K:
                want = list(range(nb))
            else:
                ranked = sorted(range(own), key=lambda j: (-S[j], j))
                want = sorted([own] + ranked[:K - 1])
            got = [x for x in sel["block_ids"][i, g] if x >= 0]
            assert got == want, (i, g, got, want)
            np.testing.assert_array_equal(sel["block_scores"][i, g, :len(want)],
                                          np.float32([S[j] for j in want]))


def test_p2_exact_ties_go_to_lower_block_id(oracle_mod):
    """P2 (ties): three bit-identical blocks tie for the best score; with two
    free slots the two lowest ids win, whatever their order in memory."""
    D, blk, K = 16, 4, 3
    L = 10 * blk
    w = make_inputs(B=1, Sq=1, lens=[L], H_q=1, H_kv=1, top_k=K, seed=5, device="cpu",
                    D=D, d_idx=D, block=blk)
    qn = w.q_idx[0, 0, 0].float()
    qn = qn / qn.norm()
    hot = (8.0 * qn).to(torch.bfloat16)
    for j in (7, 2, 5):
        w.k_idx[j * blk:(j + 1) * blk, 0, :] = hot
    a = _np_inputs(w)
    sel = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"], block=blk,
                                top_k=K)
    assert sel["block_ids"][0, 0].tolist() == [2, 5, 9]
    b = sel["boundary"][0, 0]
    assert b[0] == b[1]  # the cut falls inside the tie


def test_p3_planted_needles_are_selected(oracle_mod):
    """P3: needle blocks whose index keys are 16*q_idx/|q_idx| + N(0, 0.1)
    score about 16|q_idx| (~16 sigma above a random block max), so with
    #needles <= k-1 every needle must be kept."""
    L = 64 * 128
    w = make_inputs(B=2, Sq=1, lens=[L, L - 77], H_q=4, H_kv=2, top_k=16, seed=9, device="cpu",
                    needles=15, amp=16.0)
    a = _np_inputs(w)
    sel = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"], top_k=16)
    for b in range(2):
        own = (w.lens_host[b] - 1) // 128
        want = sorted(w.needle_blocks[b] + [own])
        for g in range(2):
            assert sel["block_ids"][b, g].tolist() == want


def test_p4_softmax_weights_sum_to_one(oracle_mod):
    """P4: the normalised weights of every (row, head) sum to 1; with V set to
    one-hot rows e_(t mod D) the output itself sums to 1."""
    D, blk = 16, 8
    w = make_inputs(B=2, Sq=20, lens=[50, 33], H_q=4, H_kv=2, top_k=3, seed=3, device="cpu",
                    D=D, d_idx=D, block=blk)
    eye = torch.eye(D, dtype=torch.bfloat16)
    for t in range(w.v.shape[0]):
        w.v[t, :, :] = eye[t % D]
    sel, out, ws = _oracle_run(oracle_mod, w, 3)
    np.testing.assert_allclose(ws, 1.0, atol=1e-12)
    np.testing.assert_allclose(out.sum(-1), 1.0, atol=1e-12)
    assert (out >= 0).all()


def test_p5_constant_values_give_that_constant(oracle_mod):
    """P5: if every value row is the same vector c, the output is c."""
    D, blk = 16, 8
    w = make_inputs(B=1, Sq=30, lens=[30], H_q=4, H_kv=2, top_k=2, seed=4, device="cpu",
                    D=D, d_idx=D, block=blk)
    c = torch.linspace(-3, 3, D).to(torch.bfloat16)
    w.v[:] = c
    _, out, _ = _oracle_run(oracle_mod, w, 2)
    np.testing.assert_allclose(out, np.broadcast_to(c.double().numpy(), out.shape), atol=1e-12)


def test_p6_top1_is_block_diagonal_causal_attention(oracle_mod):
    """P6: with k = 1 only the own block is kept, so MSA equals causal
    attention restricted to the query's own block (library routine + mask)."""
    D, blk = 16, 8
    w = make_inputs(B=1, Sq=45, lens=[45], H_q=4, H_kv=2, top_k=1, seed=6, device="cpu",
                    D=D, d_idx=D, block=blk)
    sel, out, _ = _oracle_run(oracle_mod, w, 1)
    ref = _sdpa_rows(w, lambda p, t: (t <= p) & (t // blk == p // blk))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    for i in range(45):
        assert sel["block_ids"][i, :, 0].tolist() == [i // blk] * 2


def test_p7_scaling_index_query_doubles_scores(oracle_mod):
    """P7: q_idx -> 2*q_idx (exact in bf16) doubles every block score exactly
    and keeps the selection (the index score is linear in q_idx)."""
    w = make_inputs(B=1, Sq=1, lens=[40 * 128 + 5], H_q=2, H_kv=2, top_k=16, seed=7,
                    device="cpu")
    a = _np_inputs(w)
    s1 = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"])
    q2 = bf16_bits((w.q_idx.float() * 2).to(torch.bfloat16))
    s2 = oracle_mod.index_topk(q2, a["k_idx"], a["lens"], a["kv_offsets"])
    np.testing.assert_array_equal(s1["block_ids"], s2["block_ids"])
    np.testing.assert_array_equal(2 * s1["block_scores"], s2["block_scores"])


def test_p8_swapping_two_blocks_swaps_their_ids(oracle_mod):
    """P8: exchanging the contents (k_idx, K, V) of a kept and a dropped
    non-own block exchanges their ids and leaves the output unchanged."""
    blk = 128
    w = make_inputs(B=1, Sq=1, lens=[30 * blk + 3], H_q=2, H_kv=1, top_k=4, seed=8, device="cpu")
    sel, out, _ = _oracle_run(oracle_mod, w, 4)
    kept = [j for j in sel["block_ids"][0, 0].tolist() if j != 30]
    dropped = [j for j in range(30) if j not in kept]
    ja, jb = kept[0], dropped[0]
    for name in ("k_idx", "k", "v"):
        t = getattr(w, name)
        tmp = t[ja * blk:(ja + 1) * blk].clone()
        t[ja * blk:(ja + 1) * blk] = t[jb * blk:(jb + 1) * blk]
        t[jb * blk:(jb + 1) * blk] = tmp
    sel2, out2, _ = _oracle_run(oracle_mod, w, 4)
    want = sorted([jb if j == ja else j for j in sel["block_ids"][0, 0].tolist()])
    assert sel2["block_ids"][0, 0].tolist() == want
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Sq,L", [(1, 1000), (77, 77), (5, 130)])
def test_p9_block_score_is_brute_force_max_of_token_scores(oracle_mod, Sq, L):
    """P9: every visible block score equals the max of the per-token dot
    products over that block's visible tokens (t <= p), computed by numpy."""
    w = make_inputs(B=1, Sq=Sq, lens=[L], H_q=2, H_kv=2, top_k=16, seed=12, device="cpu")
    a = _np_inputs(w)
    sel = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"],
                                want_all_scores=True)
    qi = _f64(a["q_idx"][0]).numpy()
    ki = _f64(a["k_idx"]).numpy()
    for i in range(Sq):
        p = L - Sq + i
        for g in range(2):
            s = ki[:p + 1, g, :] @ qi[i, g, :]
            nb = p // 128 + 1
            want = np.array([s[j * 128:(j + 1) * 128].max() for j in range(nb)])
            got = sel["all_scores"][i, g]
            np.testing.assert_allclose(got[:nb], want, rtol=0, atol=1e-9)
            assert np.isneginf(got[nb:]).all()


def test_decode_row_equals_last_prefill_row(oracle_mod):
    """Decode (Sq=1, query at position L-1) equals the last row of a prefill
    over the same sequence."""
    L = 700
    wp = make_inputs(B=1, Sq=L, lens=[L], H_q=4, H_kv=2, top_k=3, seed=13, device="cpu")
    selp, outp, _ = _oracle_run(oracle_mod, wp, 3)
    a = _np_inputs(wp)
    qd = a["q"][:, -1:]
    qid = a["q_idx"][:, -1:]
    seld = oracle_mod.index_topk(qid, a["k_idx"], a["lens"], a["kv_offsets"], top_k=3)
    outd = oracle_mod.sparse_attention(qd, a["k"], a["v"], seld["block_ids"], a["lens"],
                                       a["kv_offsets"], scale=wp.scale)
    np.testing.assert_array_equal(seld["block_ids"][0], selp["block_ids"][L - 1])
    np.testing.assert_allclose(outd[0], outp[L - 1], rtol=0, atol=1e-13)


def test_padded_layout_equals_packed_and_ignores_padding(oracle_mod):
    """Padded caches (offset b*L_max) give the packed result; the padding
    beyond each length (filled with NaN) is never read."""
    lens = [300, 129, 512]
    wk = make_inputs(B=3, Sq=1, lens=lens, H_q=4, H_kv=2, top_k=2, seed=14, device="cpu")
    wp = make_inputs(B=3, Sq=1, lens=lens, H_q=4, H_kv=2, top_k=2, seed=14, device="cpu",
                     padded_to=512)
    for name in ("k_idx", "k", "v"):
        src, dst = getattr(wk, name), getattr(wp, name)
        dst.fill_(float("nan"))
        for b, L in enumerate(lens):
            dst[b * 512:b * 512 + L] = src[int(wk.kv_offsets[b]):int(wk.kv_offsets[b]) + L]
    wp.q_idx.copy_(wk.q_idx)
    wp.q.copy_(wk.q)
    s1, o1, _ = _oracle_run(oracle_mod, wk, 2)
    s2, o2, _ = _oracle_run(oracle_mod, wp, 2)
    np.testing.assert_array_equal(s1["block_ids"], s2["block_ids"])
    np.testing.assert_array_equal(o1, o2)
    assert np.isfinite(o2).all()


def test_short_sequence_keeps_every_block_and_pads(oracle_mod):
    """With no more visible blocks than k, all are kept; the rest is -1/-inf."""
    w = make_inputs(B=1, Sq=1, lens=[3 * 128 + 1], H_q=2, H_kv=1, top_k=16, seed=15,
                    device="cpu")
    a = _np_inputs(w)
    sel = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"])
    assert sel["block_ids"][0, 0].tolist() == [0, 1, 2, 3] + [-1] * 12
    assert np.isneginf(sel["block_scores"][0, 0, 4:]).all()
    assert np.isfinite(sel["block_scores"][0, 0, :4]).all()


def test_invalid_lengths_are_rejected(oracle_mod):
    w = make_inputs(B=1, Sq=4, lens=[10], H_q=2, H_kv=1, top_k=2, seed=1, device="cpu", D=8,
                    d_idx=8, block=4)
    a = _np_inputs(w)
    bad = np.array([3], np.int32)     # fewer tokens than query rows
    with pytest.raises(ValueError):
        oracle_mod.index_topk(a["q_idx"], a["k_idx"], bad, a["kv_offsets"], block=4, top_k=2)


def test_hand_worked_decode_example(oracle_mod):
    """A worked decode example derived by hand (tests/golden/hand_worked_decode.json):
    block size 2, head dim 2, seven tokens; the expected ids, scores and the
    closed-form outputs are written out in the fixture's derivation."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_decode.json")
    g = json.load(open(path))

    def bits(x):
        return bf16_bits(torch.tensor(x, dtype=torch.float32).to(torch.bfloat16))

    q_idx = bits(g["q_idx"]).reshape(1, 1, 1, 2)
    k_idx = bits(g["k_idx"]).reshape(7, 1, 2)
    q = bits(g["q"]).reshape(1, 1, 2, 2)
    k = bits(g["k"]).reshape(7, 1, 2)
    v = bits(g["v"]).reshape(7, 1, 2)
    lens = np.array(g["lens"], np.int32)
    offs = np.zeros(1, np.int64)
    e = g["expect"]
    s2 = oracle_mod.index_topk(q_idx, k_idx, lens, offs, block=2, top_k=2)
    s3 = oracle_mod.index_topk(q_idx, k_idx, lens, offs, block=2, top_k=3)
    assert s2["block_ids"][0, 0].tolist() == e["k2_ids"]
    assert s2["block_scores"][0, 0].tolist() == e["k2_scores"]
    assert s3["block_ids"][0, 0].tolist() == e["k3_ids"]
    assert s3["block_scores"][0, 0].tolist() == e["k3_scores"]
    out = oracle_mod.sparse_attention(q, k, v, s2["block_ids"], lens, offs, block=2,
                                      scale=g["scale"])
    want = [[eval(expr, {"e": math.e}) for expr in row] for row in e["k2_out_closed_form"]]
    np.testing.assert_allclose(out[0], np.array(want), rtol=0, atol=1e-14)
