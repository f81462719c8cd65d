"""Pins for the oracle's index-branch variants: fewer index heads than GQA
groups, index keys shared by every index head, and FP8 E4M3 index keys with
one fp32 scale per key row.

The mlqm.cn guide's configuration sets sparse_num_index_heads = 4 while the
cloud.tencent.com article (section 二) describes one index query per group;
the pages say nothing more, so the oracle reads index heads as partitioning
the groups into contiguous sets.  Each pin below ties a variant to something
outside the code path it tests: the FP8 format's published values and torch's
own E4M3 converter, a numpy brute force, a library attention routine, or an
exact equivalence with the already pinned one-head-per-group path.
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
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _e4m3_bytes(shape, seed):
    """Seeded E4M3 bytes, NaN codes (S.1111.111) excluded."""
    rng = np.random.default_rng(seed)
    b = rng.integers(0, 256, size=shape, dtype=np.uint8)
    b[(b & 0x7F) == 0x7F] ^= 0x01
    return b


# Values of the OCP 8-bit floating-point specification's E4M3 encoding.
E4M3_SPEC = {
    0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3C: 1.5,
    0x40: 2.0, 0x77: 240.0, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0,
}


def test_e4m3_decoding_matches_format_definition(oracle_mod):
    for code, val in E4M3_SPEC.items():
        got = oracle_mod.e4m3_to_float(code)
        assert got == val and np.signbit(got) == np.signbit(val), (hex(code), got, val)
    assert np.isnan(oracle_mod.e4m3_to_float(0x7F)) and np.isnan(oracle_mod.e4m3_to_float(0xFF))
    # every code against torch's own E4M3 converter
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle_mod.e4m3_to_float(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def _brute_block_scores(qi, keys, lens, offs, Sq, block, kh_of):
    """numpy float64: max over the visible tokens of each block of q . key."""
    B, _, H, D = qi.shape
    res = {}
    for b in range(B):
        L = int(lens[b])
        for i in range(Sq):
            p = L - Sq + i
            for g in range(H):
                s = keys[int(offs[b]):int(offs[b]) + p + 1, kh_of(g)] @ qi[b, i, g]
                nb = p // block + 1
                res[(b, i, g)] = np.array([s[j * block:min((j + 1) * block, p + 1)].max()
                                           for j in range(nb)])
    return res


def _check_scores(sel, brute, B, Sq, H, rtol=1e-13):
    for (b, i, g), ref in brute.items():
        got = sel["all_scores"][b * Sq + i, g, :ref.shape[0]]
        np.testing.assert_allclose(got, ref, rtol=rtol, atol=1e-300)


@pytest.mark.parametrize("Sq,lens", [(1, [300, 77]), (40, [40, 61])])
def test_shared_keys_scores_equal_brute_force(oracle_mod, Sq, lens):
    """Shared keys: every index head dots the token's single key row."""
    w = make_inputs(B=2, Sq=Sq, lens=lens, H_q=8, H_kv=4, top_k=3, seed=70 + Sq, device="cpu",
                    D=16, d_idx=16, block=8)
    a = _np(w)
    shared = np.ascontiguousarray(a["k_idx"][:, :1, :])
    sel = oracle_mod.index_topk(a["q_idx"], shared, a["lens"], a["kv_offsets"], block=8, top_k=3,
                                want_all_scores=True)
    brute = _brute_block_scores(_f64(a["q_idx"]), _f64(shared), a["lens"], a["kv_offsets"], Sq, 8,
                                lambda g: 0)
    _check_scores(sel, brute, 2, Sq, 4)


def test_shared_keys_equal_per_head_keys_replicated(oracle_mod):
    """Shared keys are the per-head method with every head's key row equal."""
    w = make_inputs(B=2, Sq=24, lens=[200, 24], H_q=8, H_kv=4, top_k=4, seed=71, device="cpu",
                    D=32, d_idx=32, block=16)
    a = _np(w)
    shared = np.ascontiguousarray(a["k_idx"][:, :1, :])
    rep = np.ascontiguousarray(np.repeat(shared, 4, axis=1))
    s1 = oracle_mod.index_topk(a["q_idx"], shared, a["lens"], a["kv_offsets"], block=16, top_k=4)
    s2 = oracle_mod.index_topk(a["q_idx"], rep, a["lens"], a["kv_offsets"], block=16, top_k=4)
    np.testing.assert_array_equal(s1["block_ids"], s2["block_ids"])
    np.testing.assert_array_equal(s1["block_scores"], s2["block_scores"])
    # and the selections differ between index heads (the query still matters)
    assert not np.array_equal(s1["block_ids"][:, 0], s1["block_ids"][:, 1])


@pytest.mark.parametrize("key_heads", [1, 4])
def test_fp8_keys_scores_equal_brute_force(oracle_mod, key_heads):
    """score = row scale * (q . decoded key), decoded by torch's E4M3 converter."""
    w = make_inputs(B=2, Sq=5, lens=[90, 37], H_q=8, H_kv=4, top_k=3, seed=72, device="cpu",
                    D=16, d_idx=16, block=8)
    a = _np(w)
    T = a["k_idx"].shape[0]
    k8 = _e4m3_bytes((T, key_heads, 16), seed=5)
    rng = np.random.default_rng(6)
    scale = rng.uniform(0.01, 3.0, size=(T, key_heads)).astype(np.float32)
    sel = oracle_mod.index_topk(a["q_idx"], k8, a["lens"], a["kv_offsets"], block=8, top_k=3,
                                want_all_scores=True, k_scale=scale)
    dec = torch.from_numpy(k8).view(torch.float8_e4m3fn).double().numpy()
    keys = dec * scale.astype(np.float64)[:, :, None]
    brute = _brute_block_scores(_f64(a["q_idx"]), keys, a["lens"], a["kv_offsets"], 5, 8,
                                (lambda g: 0) if key_heads == 1 else (lambda g: g))
    _check_scores(sel, brute, 2, 5, 4, rtol=1e-12)


def test_fp8_keys_at_scale_one_equal_bf16_keys_of_the_decoded_values(oracle_mod):
    """Every E4M3 value is exact in bf16, so FP8 keys with scale 1 and bf16
    keys holding the decoded values must give identical ids and scores; a
    power-of-two scale multiplies every score exactly and keeps the ids."""
    w = make_inputs(B=1, Sq=30, lens=[300], H_q=8, H_kv=2, top_k=4, seed=73, device="cpu",
                    D=32, d_idx=32, block=16)
    a = _np(w)
    T = a["k_idx"].shape[0]
    k8 = _e4m3_bytes((T, 2, 32), seed=7)
    dec = torch.from_numpy(k8).view(torch.float8_e4m3fn).float()
    kb = bf16_bits(dec.to(torch.bfloat16))
    assert np.array_equal(_f64(kb), dec.double().numpy())          # exact in bf16
    one = np.ones((T, 2), np.float32)
    s8 = oracle_mod.index_topk(a["q_idx"], k8, a["lens"], a["kv_offsets"], block=16, top_k=4,
                               k_scale=one)
    sb = oracle_mod.index_topk(a["q_idx"], kb, a["lens"], a["kv_offsets"], block=16, top_k=4)
    np.testing.assert_array_equal(s8["block_ids"], sb["block_ids"])
    np.testing.assert_array_equal(s8["block_scores"], sb["block_scores"])
    s4 = oracle_mod.index_topk(a["q_idx"], k8, a["lens"], a["kv_offsets"], block=16, top_k=4,
                               k_scale=one * 4.0)
    np.testing.assert_array_equal(s4["block_ids"], s8["block_ids"])
    np.testing.assert_array_equal(s4["block_scores"], s8["block_scores"] * 4.0)


def test_fewer_index_heads_equal_the_selection_replicated_over_groups(oracle_mod):
    """Two index heads for four groups: groups {0,1} use head 0, {2,3} head 1
    (contiguous).  Replicating each head's ids over its groups and running the
    one-head-per-group path must give the same outputs bit for bit."""
    w = make_inputs(B=2, Sq=20, lens=[260, 40], H_q=8, H_kv=4, top_k=3, seed=74, device="cpu",
                    D=16, d_idx=16, block=16)
    a = _np(w)
    qi2 = np.ascontiguousarray(a["q_idx"][:, :, :2])
    ki2 = np.ascontiguousarray(a["k_idx"][:, :2])
    sel = oracle_mod.index_topk(qi2, ki2, a["lens"], a["kv_offsets"], block=16, top_k=3)
    ids2 = sel["block_ids"]                                           # [R, 2, k]
    assert not np.array_equal(ids2[:, 0], ids2[:, 1])
    out2 = oracle_mod.sparse_attention(a["q"], a["k"], a["v"], ids2, a["lens"], a["kv_offsets"],
                                       block=16, num_index_heads=2)
    ids4 = np.ascontiguousarray(np.repeat(ids2, 2, axis=1))          # group g -> head g // 2
    out4 = oracle_mod.sparse_attention(a["q"], a["k"], a["v"], ids4, a["lens"], a["kv_offsets"],
                                       block=16)
    np.testing.assert_array_equal(out2, out4)
    # the interleaved map (g -> g % 2) would differ
    ids_bad = np.ascontiguousarray(np.tile(ids2, (1, 2, 1)))
    bad = oracle_mod.sparse_attention(a["q"], a["k"], a["v"], ids_bad, a["lens"], a["kv_offsets"],
                                      block=16)
    assert not np.allclose(out2, bad)


def test_fewer_index_heads_with_every_block_kept_is_dense_attention(oracle_mod):
    """P1 for the variant: k >= blocks keeps everything, whatever the index
    heads, so the output is causal attention (torch's library routine)."""
    w = make_inputs(B=1, Sq=48, lens=[48], H_q=8, H_kv=4, top_k=6, seed=75, device="cpu",
                    D=16, d_idx=16, block=8)
    a = _np(w)
    qi1 = np.ascontiguousarray(a["q_idx"][:, :, :1])
    shared = np.ascontiguousarray(a["k_idx"][:, :1])
    sel = oracle_mod.index_topk(qi1, shared, a["lens"], a["kv_offsets"], block=8, top_k=6)
    out = oracle_mod.sparse_attention(a["q"], a["k"], a["v"], sel["block_ids"], a["lens"],
                                      a["kv_offsets"], block=8, num_index_heads=1)
    q = torch.from_numpy(_f64(a["q"][0])).permute(1, 0, 2)
    k = torch.from_numpy(_f64(a["k"])).permute(1, 0, 2).repeat_interleave(2, 0)
    v = torch.from_numpy(_f64(a["v"])).permute(1, 0, 2).repeat_interleave(2, 0)
    mask = torch.arange(48)[None, :] <= torch.arange(48)[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                           scale=1 / 4.0).permute(1, 0, 2)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
