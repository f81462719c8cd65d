"""GPU parity of the index-branch variants through the C ABI: fewer index
heads than groups, index keys shared by every index head, and FP8 E4M3 index
keys with per-row scales, in decode and prefill, each against the CPU oracle on the same
bytes with the tolerances of tests/parity.py.  The sparse branch runs on the
variant's selection (group g uses index head g / (H_kv / Hi))."""
import numpy as np
import pytest
import torch

import block_sparse_attention_43_b200 as m

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _variant(w, Hi, fmt, seed):
    """q_idx of Hi index heads and index keys in format fmt, built from w."""
    from synthetic import bf16_bits, quantize_e4m3_rows
    shared = fmt in (m.INDEX_KEYS_BF16_SHARED, m.INDEX_KEYS_FP8_SHARED)
    q_idx = w.q_idx[:, :, :Hi].contiguous()
    keys = w.k_idx[:, :1 if shared else Hi].contiguous()
    host = dict(q_idx=bf16_bits(q_idx), q=bf16_bits(w.q), k=bf16_bits(w.k), v=bf16_bits(w.v),
                lens=w.lens.cpu().numpy(), kv_offsets=w.kv_offsets.cpu().numpy())
    scale = None
    if fmt in (m.INDEX_KEYS_FP8, m.INDEX_KEYS_FP8_SHARED):
        keys, scale = quantize_e4m3_rows(keys)
        host["k_idx"] = keys.cpu().numpy()
        host["k_scale"] = scale.cpu().numpy()
    else:
        host["k_idx"] = bf16_bits(keys)
    return q_idx, keys, scale, host


def _run(w, Hi, fmt, seed):
    from parity import compare
    q_idx, keys, scale, host = _variant(w, Hi, fmt, seed)
    eng = m.MSA(batch=w.B, q_len=w.Sq, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=DEV,
                num_index_heads=Hi, index_key_format=fmt)
    eng.index_topk(q_idx, keys, w.lens, w.kv_offsets, k_idx_scale=scale)
    eng.sparse_attention(w.q, w.k, w.v, w.lens, w.kv_offsets)
    torch.cuda.synchronize()
    assert eng.device_status() == 0
    ids, sc, out = eng.block_ids.cpu().numpy(), eng.block_scores.cpu().numpy(), \
        eng.out.float().cpu().numpy()
    assert ids.shape[2] == Hi
    return compare(_oracle(), w, ids, sc, out, host=host)


_ORACLE = []


def _oracle():
    if not _ORACLE:
        import oracle
        _ORACLE.append(oracle)
    return _ORACLE[0]


FORMATS = {"bf16": 0, "bf16_shared": 1, "fp8": 2, "fp8_shared": 3}

DECODE = [
    # (B, lens, H_q, H_kv, Hi, top_k)
    (3, [5000, 129, 20000], 64, 8, 8, 16),
    (2, [4096, 300], 64, 8, 4, 16),         # the guide's 4 index heads for 8 groups
    (4, [700, 2047, 129, 3000], 16, 8, 2, 8),
    (1, [9000], 32, 16, 16, 16),            # 16 index heads (two n8 tiles)
    (2, [1500, 7], 8, 1, 1, 4),
]


@pytest.mark.parametrize("fmt", list(FORMATS))
@pytest.mark.parametrize("B,lens,H_q,H_kv,Hi,top_k", DECODE)
def test_decode_variants(oracle_mod, fmt, B, lens, H_q, H_kv, Hi, top_k):
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=1, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=900 + B,
                    device=DEV, needles=2, amp=4.0)
    rep = _run(w, Hi, FORMATS[fmt], 1)
    print(fmt, (B, H_kv, Hi), rep)


PREFILL = [
    # (B, Sq, lens, H_q, H_kv, Hi, top_k): tensor-core index path (E4M3 keys
    # widened to bf16 in the workspace, row scales applied to the scores)
    (1, 1000, [1000], 64, 8, 4, 16),        # block-outer attention path (groups of 8)
    (2, 300, [700, 300], 16, 4, 1, 4),      # row attention path, one index head
    (1, 2000, [2000], 64, 8, 8, 8),
]


@pytest.mark.parametrize("fmt", list(FORMATS))
@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,Hi,top_k", PREFILL)
def test_prefill_variants(oracle_mod, fmt, B, Sq, lens, H_q, H_kv, Hi, top_k):
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=950 + Sq,
                    device=DEV)
    rep = _run(w, Hi, FORMATS[fmt], 2)
    print(fmt, (B, Sq, H_kv, Hi), rep)


def test_decode_shared_fp8_queries_outside_f16(oracle_mod):
    """Shared E4M3 keys take f16 products when a sequence's index queries are
    f16 values.  Sequence 0's queries here are scaled by 2^17 (exact in bf16,
    beyond f16's range), so its warps widen the codes to bf16 instead;
    sequence 1 keeps the f16 form.  Both must match the oracle."""
    from synthetic import make_inputs
    w = make_inputs(B=2, Sq=1, lens=[6000, 3000], H_q=64, H_kv=8, top_k=16, seed=77, device=DEV,
                    needles=2, amp=4.0)
    w.q_idx[0] *= 2.0 ** 17
    assert w.q_idx[0].float().abs().max().item() > 65504.0
    print(_run(w, 8, FORMATS["fp8_shared"], 3))
