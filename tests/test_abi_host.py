"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/msa.h declares, sizes workspaces, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_msa_build", os.path.join(ROOT, "block_sparse_attention_43_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import block_sparse_attention_43_b200 as mod
    return mod


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"MSA_API\s+[\w\s\*]*?\b(msa_\w+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(m):
    decl = _declared()
    assert {"msa_index_topk", "msa_sparse_attention"} <= decl
    lib = ctypes.CDLL(m.LIB_PATH)
    for name in decl:
        assert hasattr(lib, name), name
    assert decl == set(m.EXPORTS)


def _shape(m, **kw):
    base = dict(batch=4, q_len=1, max_kv_len=1 << 20, num_q_heads=64, num_kv_heads=8, top_k=16,
                kv_capacity=4 << 20)
    base.update(kw)
    return m.make_shape(**base)


def test_workspace_sizes(m):
    s = _shape(m)
    nb = (1 << 20) // 128
    assert m.msa_index_topk_workspace_size(s) == 256 + 4 * 8 * nb * 4
    assert m.msa_sparse_attention_workspace_size(s) > 256
    assert m.msa_index_topk_workspace_size(_shape(m, head_dim=64)) == 0
    assert m.msa_index_topk_workspace_size(_shape(m, num_q_heads=63)) == 0
    assert m.msa_sparse_attention_workspace_size(_shape(m, top_k=65)) == 0


def _call_index(m, s, ptrs, ws=0x100000, wsb=1 << 40):
    P = ctypes.c_void_p
    return m.lib.msa_index_topk(ctypes.byref(s), *[P(x) for x in ptrs], P(ws), wsb, None)


def test_bad_arguments_are_rejected_before_launch(m):
    s = _shape(m)
    good = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000]
    assert _call_index(m, s, [0] + good[1:]) == 1                 # null q_idx
    assert _call_index(m, s, [0x10001] + good[1:]) == 7           # misaligned q_idx
    assert _call_index(m, s, good, ws=0x100010) == 3              # misaligned workspace
    assert _call_index(m, s, good, wsb=100) == 3                  # short workspace
    assert _call_index(m, _shape(m, block_size=64), good) == 2
    assert _call_index(m, _shape(m, num_kv_heads=3, num_q_heads=9), good) == 2
    assert _call_index(m, _shape(m, q_len=0), good) == 1
    assert _call_index(m, _shape(m, q_len=10, max_kv_len=5), good) == 1
    P = ctypes.c_void_p
    r = m.lib.msa_sparse_attention(ctypes.byref(s), P(0x10000), P(0x20000), P(0x30000),
                                   P(0x40000), P(0x50000), P(0x60000), ctypes.c_float(float("nan")),
                                   P(0x70000), P(0x100000), 1 << 40, None)
    assert r == 1
    assert m.lib.msa_read_device_status(None, None) == 1


def test_status_strings(m):
    for code in range(8):
        assert m.msa_status_string(code).startswith(m.STATUS_NAMES[code])
    assert m.msa_status_string(99) == "MSA_ERR_UNKNOWN"


def test_paged_and_append_arguments_are_checked(m):
    P = ctypes.c_void_p
    s = _shape(m, kv_capacity=4 << 20)
    args = [P(0x10000), P(0x20000), P(0x30000)]
    tail = [P(0x60000), P(0x70000), P(0x100000), 1 << 40, None]
    # pages_per_seq * 128 < max_kv_len
    assert m.lib.msa_index_topk_paged(ctypes.byref(s), *args, P(0x40000), 8, *tail) == 1
    # pool not a whole number of pages
    bad = _shape(m, kv_capacity=(4 << 20) + 5)
    assert m.lib.msa_index_topk_paged(ctypes.byref(bad), *args, P(0x40000), 8192, *tail) == 1
    # null page table
    assert m.lib.msa_index_topk_paged(ctypes.byref(s), *args, None, 8192, *tail) == 1
    # kv_append needs exactly one of kv_offsets / page_table
    ptrs = [P(0x10000)] * 4
    caches = [P(0x20000)] * 3
    assert m.lib.msa_kv_append(ctypes.byref(s), 1, *ptrs[:3], P(0x30000), None, None, 0, *caches,
                               None, None) == 1
    assert m.lib.msa_kv_append(ctypes.byref(s), 1, *ptrs[:3], P(0x30000), P(0x40000),
                               P(0x50000), 8192, *caches, None, None) == 1
    assert m.lib.msa_kv_append(ctypes.byref(s), 0, *ptrs[:3], P(0x30000), P(0x40000), None, 0,
                               *caches, None, None) == 1


def test_index_variant_shapes_are_checked(m):
    P = ctypes.c_void_p
    nb = (1 << 20) // 128
    # 4 index heads for 8 groups: block scores per index head
    assert m.msa_index_topk_workspace_size(_shape(m, num_index_heads=4)) == 256 + 4 * 4 * nb * 4
    assert m.msa_index_topk_workspace_size(_shape(m, num_index_heads=3)) == 0     # does not divide 8
    assert m.msa_index_topk_workspace_size(_shape(m, num_index_heads=16)) == 0    # more heads than groups
    assert m.msa_index_topk_workspace_size(_shape(m, index_key_format=4)) == 0
    assert m.msa_sparse_attention_workspace_size(_shape(m, num_index_heads=2)) > 256
    good = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000]
    # E4M3 formats go through msa_index_topk_fp8, bf16 formats through msa_index_topk
    assert _call_index(m, _shape(m, index_key_format=m.INDEX_KEYS_FP8), good) == 2
    s = _shape(m, index_key_format=m.INDEX_KEYS_BF16_SHARED)
    args = [P(x) for x in (0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000)]
    assert m.lib.msa_index_topk_fp8(ctypes.byref(s), *args, P(0x100000), 1 << 40, None) == 1
    s8 = _shape(m, index_key_format=m.INDEX_KEYS_FP8_SHARED)
    assert m.lib.msa_index_topk_fp8(ctypes.byref(s8), P(0x10000), P(0x20000), None,
                                    *args[3:], P(0x100000), 1 << 40, None) == 1  # no scales
    assert m.lib.msa_index_topk_fp8(ctypes.byref(s8), P(0x10000), P(0x20000), P(0x30002),
                                    *args[3:], P(0x100000), 1 << 40, None) == 7  # misaligned scales
    # prefill on E4M3 keys: the workspace also holds a bf16 copy of every key row
    cap = 4 << 20
    assert m.msa_index_topk_workspace_size(_shape(m, q_len=64, index_key_format=m.INDEX_KEYS_FP8)) \
        == 256 + cap * 8 * 128 * 2
    assert m.msa_index_topk_workspace_size(
        _shape(m, q_len=64, index_key_format=m.INDEX_KEYS_FP8_SHARED)) == 256 + cap * 128 * 2


def test_decode_step_rejects_unsupported_shapes(m):
    """q_len > 1, shared or E4M3 index keys: the workspace query returns 0
    and the call returns MSA_ERR_UNSUPPORTED.  Fewer index heads than groups
    (bf16, one key row per index head) and groups of 16 heads are
    accepted."""
    for kw in (dict(q_len=2), dict(index_key_format=m.INDEX_KEYS_BF16_SHARED),
               dict(index_key_format=m.INDEX_KEYS_FP8)):
        base = dict(batch=1, q_len=1, max_kv_len=1000, num_q_heads=16, num_kv_heads=2, top_k=4,
                    kv_capacity=1000)
        base.update(kw)
        s = m.make_shape(**base)
        assert m.msa_decode_step_workspace_size(s) == 0
        fake = [0x1000] * 7
        assert m.lib.msa_decode_step(ctypes.byref(s), *fake, 0.1, 0x1000, 0x1000, 0x1000,
                                     0x100000, 1 << 40, None) == 2
    ok = m.make_shape(batch=3, q_len=1, max_kv_len=1000, num_q_heads=16, num_kv_heads=2,
                      top_k=4, kv_capacity=3000)
    assert m.msa_decode_step_workspace_size(ok) > 256
    fewer = m.make_shape(batch=3, q_len=1, max_kv_len=1000, num_q_heads=16, num_kv_heads=2,
                         top_k=4, kv_capacity=3000, num_index_heads=1)
    assert m.msa_decode_step_workspace_size(fewer) > 256
    g16 = m.make_shape(batch=3, q_len=1, max_kv_len=1000, num_q_heads=32, num_kv_heads=2,
                       top_k=4, kv_capacity=3000)
    assert m.msa_decode_step_workspace_size(g16) > 256
    # paged: a pool that is not whole pages, or a table row too short for max_kv_len
    for cap, pps in ((3000, 8), (3072, 7)):
        s = m.make_shape(batch=3, q_len=1, max_kv_len=1000, num_q_heads=16, num_kv_heads=2,
                         top_k=4, kv_capacity=cap)
        assert m.lib.msa_decode_step_paged(ctypes.byref(s), *([0x1000] * 7), pps, 0.1, 0x1000,
                                           0x1000, 0x1000, 0x100000, 1 << 40, None) == 1


def test_block_count_bound(m):
    """batch x ceil(max_kv_len / 128) must stay below 2^31 (work units are
    counted in 32 bits; sequences may share cache rows, so the pool size does
    not bound it)."""
    big = m.make_shape(batch=4096, q_len=1, max_kv_len=1 << 27, num_q_heads=64, num_kv_heads=8,
                       top_k=16, kv_capacity=1 << 27)
    assert m.msa_index_topk_workspace_size(big) == 0
    assert m.msa_decode_step_workspace_size(big) == 0
    ok = m.make_shape(batch=4096, q_len=1, max_kv_len=(1 << 26) - 128, num_q_heads=64,
                      num_kv_heads=8, top_k=16, kv_capacity=1 << 27)
    assert m.msa_index_topk_workspace_size(ok) > 0


def test_backward_workspace_layout(m):
    """The backward's workspace is the forward's, then per (row, head) the
    recomputed output (256 B), log-sum-exp and Delta (4 B each) and the fp32
    dQ sum (512 B), each region rounded to 256 B, then the backward's own
    bucket lists -- except with groups of 8 on the block-outer prefill path,
    whose forward items are reused and add nothing."""
    up = lambda x: (x + 255) // 256 * 256
    for H_q, H_kv, Sq in ((64, 8, 4096), (8, 2, 2048), (64, 8, 1)):
        s = m.make_shape(batch=2, q_len=Sq, max_kv_len=8192, num_q_heads=H_q, num_kv_heads=H_kv,
                         top_k=16, kv_capacity=16384)
        fwd = m.msa_sparse_attention_workspace_size(s)
        bwd = m.msa_sparse_attention_backward_workspace_size(s)
        pairs = 2 * Sq * H_q
        regions = up(pairs * 256) + 2 * up(pairs * 4) + up(pairs * 512)
        if H_q // H_kv == 8 and Sq > 1:
            assert bwd == up(fwd) + regions
        else:
            assert bwd > up(fwd) + regions
