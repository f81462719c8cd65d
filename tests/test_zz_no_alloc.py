"""msa_index_topk_static: the index branch for callers that cannot allocate
device memory or pass a workspace (plugin hosts that hand over only inputs and
outputs, processes whose device memory belongs to another allocator, loops
that must not stall on cudaMalloc).  Its scratch is the library's own fixed
device array, so this test checks, through the C ABI, that two calls in a row
give the same block ids and scores as msa_index_topk with a caller workspace
(ids exactly, scores within the parity tolerance) for decode rows and for
prefill rows (which need only the array's header), and that a decode shape
too large for the array is refused.  The file is named to be collected
last."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_static_scratch_index_matches_workspace_path():
    assert torch.cuda.is_available(), "needs a CUDA device"
    import block_sparse_attention_43_b200 as msa
    from parity import SCORE_REL
    from synthetic import make_inputs

    lens = [70000, 4097, 131072, 12345]
    w = make_inputs(B=4, Sq=1, lens=lens, H_q=64, H_kv=8, top_k=16, seed=77, device="cuda",
                    needles=4, amp=4.0)
    shape = msa.make_shape(batch=4, q_len=1, max_kv_len=max(lens), num_q_heads=64,
                           num_kv_heads=8, top_k=16, kv_capacity=w.kv_capacity)
    sel = (4, 1, 8, 16)
    ids_ref = torch.empty(sel, dtype=torch.int32, device="cuda")
    sc_ref = torch.empty(sel, dtype=torch.float32, device="cuda")
    ws = msa.alloc_workspace(msa.msa_index_topk_workspace_size(shape), "cuda")
    msa.msa_index_topk(shape, w.q_idx, w.k_idx, w.lens, w.kv_offsets, ids_ref, sc_ref, ws)
    torch.cuda.synchronize()
    ids_ref, sc_ref = ids_ref.cpu().numpy(), sc_ref.cpu().numpy()

    for _ in range(2):   # two calls in a row share the same static scratch
        ids = torch.full(sel, -7, dtype=torch.int32, device="cuda")
        sc = torch.full(sel, 7.0, dtype=torch.float32, device="cuda")
        stream = torch.cuda.current_stream()
        rc = msa.lib.msa_index_topk_static(
            ctypes.byref(shape), ctypes.c_void_p(w.q_idx.data_ptr()),
            ctypes.c_void_p(w.k_idx.data_ptr()), ctypes.c_void_p(w.lens.data_ptr()),
            ctypes.c_void_p(w.kv_offsets.data_ptr()), ctypes.c_void_p(ids.data_ptr()),
            ctypes.c_void_p(sc.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        assert rc == 0, msa.msa_status_string(rc)
        torch.cuda.synchronize()
        ids, sc = ids.cpu().numpy(), sc.cpu().numpy()
        np.testing.assert_array_equal(ids, ids_ref)
        fin = np.isfinite(sc_ref)
        np.testing.assert_array_equal(np.isfinite(sc), fin)
        lim = SCORE_REL * np.maximum(np.abs(sc_ref[fin].astype(np.float64)), 1.0)
        assert (np.abs(sc[fin].astype(np.float64) - sc_ref[fin]) <= lim).all()

    # Too many decode block scores for the fixed array: refused before any launch.
    big = msa.make_shape(batch=64, q_len=1, max_kv_len=1 << 20, num_q_heads=64, num_kv_heads=8,
                         top_k=16, kv_capacity=w.kv_capacity)
    rc = msa.lib.msa_index_topk_static(ctypes.byref(big), *([ctypes.c_void_p(16)] * 6), None)
    assert rc == 3   # MSA_ERR_WORKSPACE


def _call_static(msa, shape, q_idx, k_idx, lens, offs, ids, sc):
    stream = torch.cuda.current_stream()
    return msa.lib.msa_index_topk_static(
        ctypes.byref(shape), ctypes.c_void_p(q_idx.data_ptr()), ctypes.c_void_p(k_idx.data_ptr()),
        ctypes.c_void_p(lens.data_ptr()), ctypes.c_void_p(offs.data_ptr()),
        ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
        ctypes.c_void_p(stream.cuda_stream))


def test_static_scratch_prefill_rows_match_workspace_path():
    """q_len > 1: the selection runs inside the tensor-core kernel, so the
    static path uses only the array's header; two calls in a row must still
    equal msa_index_topk with a caller workspace."""
    assert torch.cuda.is_available(), "needs a CUDA device"
    import block_sparse_attention_43_b200 as msa
    from parity import SCORE_REL
    from synthetic import make_inputs

    lens = [1000, 1500]
    Sq = 600
    w = make_inputs(B=2, Sq=Sq, lens=lens, H_q=16, H_kv=2, top_k=4, seed=78, device="cuda")
    shape = msa.make_shape(batch=2, q_len=Sq, max_kv_len=max(lens), num_q_heads=16,
                           num_kv_heads=2, top_k=4, kv_capacity=w.kv_capacity)
    assert msa.msa_index_topk_workspace_size(shape) == 256
    sel = (2, Sq, 2, 4)
    ids_ref = torch.empty(sel, dtype=torch.int32, device="cuda")
    sc_ref = torch.empty(sel, dtype=torch.float32, device="cuda")
    ws = msa.alloc_workspace(msa.msa_index_topk_workspace_size(shape), "cuda")
    msa.msa_index_topk(shape, w.q_idx, w.k_idx, w.lens, w.kv_offsets, ids_ref, sc_ref, ws)
    torch.cuda.synchronize()
    ids_ref, sc_ref = ids_ref.cpu().numpy(), sc_ref.cpu().numpy()
    for _ in range(2):
        ids = torch.full(sel, -7, dtype=torch.int32, device="cuda")
        sc = torch.full(sel, 7.0, dtype=torch.float32, device="cuda")
        rc = _call_static(msa, shape, w.q_idx, w.k_idx, w.lens, w.kv_offsets, ids, sc)
        assert rc == 0, msa.msa_status_string(rc)
        torch.cuda.synchronize()
        ids, sc = ids.cpu().numpy(), sc.cpu().numpy()
        np.testing.assert_array_equal(ids, ids_ref)
        fin = np.isfinite(sc_ref)
        np.testing.assert_array_equal(np.isfinite(sc), fin)
        lim = SCORE_REL * np.maximum(np.abs(sc_ref[fin].astype(np.float64)), 1.0)
        assert (np.abs(sc[fin].astype(np.float64) - sc_ref[fin]) <= lim).all()

    # E4M3 index keys are not taken by the static entry (nothing is launched).
    fp8 = msa.make_shape(batch=2, q_len=Sq, max_kv_len=max(lens), num_q_heads=16,
                         num_kv_heads=2, top_k=4, kv_capacity=w.kv_capacity,
                         index_key_format=msa.INDEX_KEYS_FP8)
    rc = msa.lib.msa_index_topk_static(ctypes.byref(fp8), *([ctypes.c_void_p(16)] * 6), None)
    assert rc == 2   # MSA_ERR_UNSUPPORTED
