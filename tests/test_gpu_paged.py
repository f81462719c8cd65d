"""Paged KV caches and KV append through the C ABI.

Paging only changes where a 128-token block lives, so on the same tokens the
paged calls must give bit-identical ids and scores to the packed calls, and
identical outputs wherever the kernel's summation order is fixed (decode and
the per-row kernel; the block-outer prefill path adds partials with atomics
and may differ in the last bf16 bit); the paged outputs are also compared
with the oracle directly.  Page padding past each length
is filled with NaN: it must never reach an output."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def m():
    assert torch.cuda.is_available(), "needs a CUDA device"
    import block_sparse_attention_43_b200 as mod
    return mod


def _paged_copy(w, seed=0, spare=3):
    """Scatter the packed caches of w into shuffled 128-token pages."""
    nb = [(L + 127) // 128 for L in w.lens_host]
    pps = max(nb)
    n_pages = sum(nb) + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)
    table = torch.full((w.B, pps), -1, dtype=torch.int32)
    pools = {}
    for name in ("k_idx", "k", "v"):
        src = getattr(w, name)
        pools[name] = torch.full((n_pages * 128,) + tuple(src.shape[1:]), float("nan"),
                                 dtype=src.dtype, device=src.device)
    used = 0
    for b, L in enumerate(w.lens_host):
        off = int(w.kv_offsets[b])
        for j in range(nb[b]):
            pg = int(perm[used])
            used += 1
            table[b, j] = pg
            n = min(128, L - 128 * j)
            for name in ("k_idx", "k", "v"):
                pools[name][pg * 128:pg * 128 + n] = getattr(w, name)[off + 128 * j:off + 128 * j + n]
    # unused table slots point at a spare page (never read: past each length)
    table[table < 0] = int(perm[-1])
    return pools, table.to(w.k.device), n_pages


def _run_both(m, w):
    from parity import run_gpu, to_host
    packed, st = run_gpu(w)
    assert st == 0
    pools, table, n_pages = _paged_copy(w)
    shape = m.make_shape(batch=w.B, q_len=w.Sq, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                         num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=n_pages * 128)
    sel = (w.B, w.Sq, w.H_kv, w.top_k)
    ids = torch.empty(sel, dtype=torch.int32, device=DEV)
    sc = torch.empty(sel, dtype=torch.float32, device=DEV)
    out = torch.empty_like(packed.out)
    ws_i = m.alloc_workspace(m.msa_index_topk_workspace_size(shape), DEV)
    ws_a = m.alloc_workspace(m.msa_sparse_attention_workspace_size(shape), DEV)
    m.msa_index_topk_paged(shape, w.q_idx, pools["k_idx"], w.lens, table, ids, sc, ws_i)
    m.msa_sparse_attention_paged(shape, w.q, pools["k"], pools["v"], ids, w.lens, table, w.scale,
                                 out, ws_a)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(ws_i) == 0 and m.msa_read_device_status(ws_a) == 0
    return to_host(packed), (ids.cpu().numpy(), sc.cpu().numpy(), out.float().cpu().numpy())


CASES = [
    # (B, Sq, lens, H_q, H_kv, top_k)
    (3, 1, [5000, 129, 20000], 64, 8, 16),      # decode
    (2, 1, [4096, 300], 16, 4, 4),              # decode, group of 4
    (1, 1000, [1000], 64, 8, 16),               # prefill, block-outer path, partial last page
    (2, 200, [777, 200], 8, 2, 3),              # prefill, group of 4 (row kernel)
]


@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,top_k", CASES)
def test_paged_equals_packed_and_oracle(m, oracle_mod, B, Sq, lens, H_q, H_kv, top_k):
    from parity import compare
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=600 + Sq,
                    device=DEV, needles=2 if Sq == 1 else 0)
    (pi, ps, po), (gi, gs, go) = _run_both(m, w)
    np.testing.assert_array_equal(gi, pi)
    np.testing.assert_array_equal(gs, ps)
    if Sq > 1 and H_q // H_kv == 8:
        # The block-outer prefill path adds partial outputs with atomics, so the
        # fp32 summation order (and at most the last bf16 bit) varies by run.
        np.testing.assert_allclose(go, po, rtol=0, atol=4e-3)
    else:
        np.testing.assert_array_equal(go, po)
    compare(oracle_mod, w, gi, gs, go)


def test_bad_page_number_sets_status(m):
    from synthetic import make_inputs
    w = make_inputs(B=2, Sq=1, lens=[1000, 600], H_q=16, H_kv=2, top_k=4, seed=9, device=DEV)
    pools, table, n_pages = _paged_copy(w)
    table[1, 2] = n_pages + 50                   # outside the pool
    shape = m.make_shape(batch=2, q_len=1, max_kv_len=1000, num_q_heads=16, num_kv_heads=2,
                         top_k=4, kv_capacity=n_pages * 128)
    ids = torch.empty((2, 1, 2, 4), dtype=torch.int32, device=DEV)
    sc = torch.empty((2, 1, 2, 4), dtype=torch.float32, device=DEV)
    ws = m.alloc_workspace(m.msa_index_topk_workspace_size(shape), DEV)
    m.msa_index_topk_paged(shape, w.q_idx, pools["k_idx"], w.lens, table, ids, sc, ws)
    assert m.msa_read_device_status(ws) == 6


@pytest.mark.parametrize("paged", [False, True])
def test_kv_append_then_decode(m, paged):
    """Caches holding L-1 tokens + msa_kv_append of the last token equal the
    full caches, and the decode step on them gives the same result."""
    from parity import run_gpu, to_host
    from synthetic import make_inputs
    lens = [3000, 129, 777]
    w = make_inputs(B=3, Sq=1, lens=lens, H_q=16, H_kv=2, top_k=4, seed=31, device=DEV)
    full = to_host(run_gpu(w)[0])
    if paged:
        pools, table, n_pages = _paged_copy(w)
        caches = {k: v.clone() for k, v in pools.items()}
        cap = n_pages * 128
    else:
        caches = {k: getattr(w, k).clone() for k in ("k_idx", "k", "v")}
        table, cap = None, w.kv_capacity
    new = {}
    for name in ("k_idx", "k", "v"):
        new[name] = torch.stack([getattr(w, name)[int(w.kv_offsets[b]) + L - 1]
                                 for b, L in enumerate(lens)]).unsqueeze(1).contiguous()
        # wipe the last token in the caches
        for b, L in enumerate(lens):
            if paged:
                t = L - 1
                row = int(table[b, t // 128]) * 128 + t % 128
            else:
                row = int(w.kv_offsets[b]) + L - 1
            caches[name][row] = 0
    shape = m.make_shape(batch=3, q_len=1, max_kv_len=max(lens), num_q_heads=16, num_kv_heads=2,
                         top_k=4, kv_capacity=cap)
    short = (w.lens - 1).contiguous()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    m.msa_kv_append(shape, new["k_idx"], new["k"], new["v"], short, caches["k_idx"], caches["k"],
                    caches["v"], kv_offsets=None if paged else w.kv_offsets,
                    page_table=table if paged else None, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    if paged:
        for name in ("k_idx", "k", "v"):
            a, b_ = caches[name], pools[name]
            assert torch.equal(torch.nan_to_num(a.float()), torch.nan_to_num(b_.float()))
        return
    for name in ("k_idx", "k", "v"):
        assert torch.equal(caches[name], getattr(w, name))
    w.k_idx, w.k, w.v = caches["k_idx"], caches["k"], caches["v"]
    again = to_host(run_gpu(w)[0])
    for x, y in zip(full, again):
        np.testing.assert_array_equal(x, y)


def test_kv_append_past_max_len_is_refused(m):
    from synthetic import make_inputs
    w = make_inputs(B=1, Sq=1, lens=[256], H_q=8, H_kv=1, top_k=2, seed=3, device=DEV)
    shape = m.make_shape(batch=1, q_len=1, max_kv_len=256, num_q_heads=8, num_kv_heads=1, top_k=2,
                         kv_capacity=w.kv_capacity)
    before = w.k.clone()
    new = torch.ones((1, 1, 1, 128), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    m.msa_kv_append(shape, new, new, new, w.lens, w.k_idx, w.k, w.v, kv_offsets=w.kv_offsets,
                    device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    assert torch.equal(w.k, before)


@pytest.mark.parametrize("B,lens,H_q,H_kv,top_k", [
    (3, [5000, 129, 20000], 64, 8, 16),
    (2, [4096, 300], 16, 4, 4),
])
def test_fused_decode_step_paged_equals_packed(m, oracle_mod, B, lens, H_q, H_kv, top_k):
    """msa_decode_step_paged on shuffled pages (NaN page padding) gives the
    packed msa_decode_step's ids, scores and outputs bit for bit."""
    from parity import compare
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=1, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=650 + B,
                    device=DEV, needles=2)
    eng = m.MSA(batch=B, q_len=1, max_kv_len=max(lens), num_q_heads=H_q, num_kv_heads=H_kv,
                top_k=top_k, kv_capacity=w.kv_capacity, device=DEV)
    eng.decode_step(w.q_idx, w.k_idx, w.q, w.k, w.v, w.lens, w.kv_offsets)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(eng.ws_step) == 0
    pools, table, n_pages = _paged_copy(w)
    shape = m.make_shape(batch=B, q_len=1, max_kv_len=max(lens), num_q_heads=H_q,
                         num_kv_heads=H_kv, top_k=top_k, kv_capacity=n_pages * 128)
    ids = torch.empty_like(eng.block_ids)
    sc = torch.empty_like(eng.block_scores)
    out = torch.empty_like(eng.out)
    ws = m.alloc_workspace(m.msa_decode_step_workspace_size(shape), DEV)
    m.msa_decode_step_paged(shape, w.q_idx, pools["k_idx"], w.q, pools["k"], pools["v"], w.lens,
                            table, w.scale, ids, sc, out, ws)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(ws) == 0
    assert torch.equal(ids, eng.block_ids) and torch.equal(sc, eng.block_scores)
    assert torch.equal(out, eng.out)
    compare(oracle_mod, w, ids.cpu().numpy(), sc.cpu().numpy(), out.float().cpu().numpy())
