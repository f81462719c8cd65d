"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element on the same seeded inputs (tolerances in tests/parity.py)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def msa_lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import block_sparse_attention_43_b200 as m   # raises if libmsa.so is missing
    return m


def _run_and_compare(oracle_mod, w, rows=None):
    from parity import compare, run_gpu, to_host
    m, st = run_gpu(w)
    assert st == 0, f"device status {st}"
    ids, sc, out = to_host(m)
    return compare(oracle_mod, w, ids, sc, out, rows=rows)


# (B, lens, H_q, H_kv, top_k): ragged, block-aligned, shorter than k blocks,
# a single token, one group, 16 groups, group sizes 1..16.
DECODE_CASES = [
    (3, [5000, 128, 1], 16, 2, 4),
    (2, [4096, 4097], 64, 8, 16),
    (4, [700, 2047, 129, 3000], 8, 8, 16),
    (1, [20000], 8, 1, 16),
    (2, [9000, 15000], 16, 16, 16),
    (5, [1500, 333, 4096, 8191, 260], 32, 2, 16),
    (2, [6000, 6001], 16, 4, 1),
    (1, [3 * 128 + 5], 8, 8, 16),
]


@pytest.mark.parametrize("B,lens,H_q,H_kv,top_k", DECODE_CASES)
def test_decode_small_shapes(msa_lib, oracle_mod, B, lens, H_q, H_kv, top_k):
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=1, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=101 + B,
                    device=DEV, needles=3, amp=4.0)
    _run_and_compare(oracle_mod, w)


def test_decode_padded_cache(msa_lib, oracle_mod):
    """Padded layout (offset b*L_max) with NaN padding past each length."""
    from synthetic import make_inputs
    lens = [3000, 129, 4096, 1000]
    w = make_inputs(B=4, Sq=1, lens=lens, H_q=64, H_kv=8, top_k=16, seed=7, device=DEV,
                    padded_to=4096)
    for t in (w.k_idx, w.k, w.v):
        for b, L in enumerate(lens):
            t[b * 4096 + L:(b + 1) * 4096] = float("nan")
    _run_and_compare(oracle_mod, w)


PREFILL_CASES = [
    (1, 300, [300], 8, 2, 4),        # full prefill, ragged last block
    (2, 64, [500, 64], 16, 4, 3),    # chunked prefill: last 64 rows; a 64-token sequence
    (1, 1024, [1024], 8, 8, 16),     # k >= blocks everywhere
    (1, 777, [2000], 16, 2, 5),      # prefill continuing a cached prefix
]


@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,top_k", PREFILL_CASES)
def test_prefill_small_shapes(msa_lib, oracle_mod, B, Sq, lens, H_q, H_kv, top_k):
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=300 + Sq,
                    device=DEV)
    _run_and_compare(oracle_mod, w)


# Groups of 8 heads take the block-outer tensor-core prefill path.
PREFILL_G8_CASES = [
    (1, 1000, [1000], 64, 8, 16),     # every block kept (k >= blocks), ragged last block
    (1, 4000, [4000], 16, 2, 8),      # real selection
    (2, 700, [3000, 700], 16, 2, 4),  # unaligned chunk after a cached prefix + a full prefill
    (1, 20000, [20000], 8, 1, 16),    # one group, three 8192-row bucket ranges
]


@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,top_k", PREFILL_G8_CASES)
def test_prefill_block_outer_path(msa_lib, oracle_mod, B, Sq, lens, H_q, H_kv, top_k):
    from parity import sample_rows
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=400 + Sq,
                    device=DEV)
    rows = None if B * Sq <= 4000 else sample_rows(B * Sq, 3000, seed=5)
    rep = _run_and_compare(oracle_mod, w, rows=rows)
    print("prefill g8", (B, Sq, H_q, H_kv, top_k), rep)


# top-k above 16 takes the index kernel's longer row lists (32, 64 slots) and
# the block-outer attention with up to 64 kept blocks per row.
PREFILL_LARGE_K_CASES = [
    (1, 6000, [6000], 16, 2, 32),      # 47 blocks, 32 kept
    (2, 4500, [9000, 4500], 16, 2, 64),  # chunk after a cached prefix (71 blocks) + 36 blocks
    (1, 3000, [3000], 8, 2, 17),       # list of 32 slots, row attention path (groups of 4)
]


@pytest.mark.parametrize("B,Sq,lens,H_q,H_kv,top_k", PREFILL_LARGE_K_CASES)
def test_prefill_large_top_k(msa_lib, oracle_mod, B, Sq, lens, H_q, H_kv, top_k):
    from parity import sample_rows
    from synthetic import make_inputs
    w = make_inputs(B=B, Sq=Sq, lens=lens, H_q=H_q, H_kv=H_kv, top_k=top_k, seed=500 + top_k,
                    device=DEV)
    rep = _run_and_compare(oracle_mod, w, rows=sample_rows(B * Sq, 600, seed=6))
    print("prefill large k", (B, Sq, H_q, H_kv, top_k), rep)


def _flag_count(eng):
    """(row, head) pairs the block-outer prefill path handed to its exact
    fp32 pass (a count the kernels keep in the workspace header)."""
    return int(eng.ws_attn[4:8].view(torch.int32).item())


def test_prefill_large_logit_block_takes_exact_path(msa_lib, oracle_mod):
    """A kept non-own block whose keys are 40x larger: its logits dwarf the
    own block's, so its partial outputs are far beyond the fp16 sum's range;
    those (row, head) pairs must go through the exact fp32 pass."""
    from synthetic import make_inputs
    from parity import compare, run_gpu, to_host
    w = make_inputs(B=1, Sq=640, lens=[640], H_q=16, H_kv=2, top_k=5, seed=33, device=DEV)
    w.k[128:256].mul_(40.0)
    m, st = run_gpu(w)
    assert st == 0
    assert _flag_count(m) > 0, "the exact pass was not exercised"
    rep = compare(oracle_mod, w, *to_host(m))
    print("large logits", rep, "flagged", _flag_count(m))


def test_prefill_sharp_logits_take_exact_path(msa_lib, oracle_mod):
    """Queries 6x larger in one sequence (logits with a standard deviation
    of 6): for rows whose own block holds few keys, another kept block's
    maximum beats the own block's by far more than the fp16 sum allows, so
    those (row, head) pairs take the exact pass; the outputs stay O(1)."""
    from synthetic import make_inputs
    from parity import compare, run_gpu, to_host
    w = make_inputs(B=2, Sq=1024, lens=[1024, 1024], H_q=16, H_kv=2, top_k=4, seed=34, device=DEV)
    w.q[0].mul_(6.0)
    m, st = run_gpu(w)
    assert st == 0
    n = _flag_count(m)
    assert n > 0, "the exact pass was not exercised"
    rep = compare(oracle_mod, w, *to_host(m))
    print("sharp logits", rep, "flagged", n)


@pytest.mark.parametrize("name", ["prefill_2k", "decode_32k", "decode_ragged", "decode_1m"])
def test_named_workload_full_parity(msa_lib, oracle_mod, name):
    """The workloads at full size, every row compared."""
    from synthetic import make_workload
    w = make_workload(name, DEV)
    rep = _run_and_compare(oracle_mod, w)
    print(name, rep)


def test_prefill_128k_index_sampled_rows(msa_lib, oracle_mod):
    """128k-token prefill, index branch at full size on the GPU (tcgen05
    path), 4096 seeded rows plus block-edge rows checked against the oracle."""
    import block_sparse_attention_43_b200 as m
    from parity import compare_index, sample_rows
    from synthetic import bf16_bits, make_workload
    w = make_workload("prefill_128k", DEV)
    eng = m.MSA(batch=1, q_len=w.Sq, max_kv_len=w.Sq, num_q_heads=w.H_q, num_kv_heads=w.H_kv,
                top_k=w.top_k, kv_capacity=w.kv_capacity, device=DEV)
    eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets)
    assert m.msa_read_device_status(eng.ws_index) == 0
    host = dict(q_idx=bf16_bits(w.q_idx), k_idx=bf16_bits(w.k_idx), lens=w.lens.cpu().numpy(),
                kv_offsets=w.kv_offsets.cpu().numpy())
    rows = sample_rows(w.Sq, 4096, seed=2)
    _, _, rep = compare_index(oracle_mod, w, eng.block_ids.cpu().numpy(),
                              eng.block_scores.cpu().numpy(), rows=rows, host=host)
    print("prefill_128k index", rep)


def test_prefill_128k_full_path_sampled_rows(msa_lib, oracle_mod):
    """128k-token prefill, both stages at full size on the GPU, in the launch
    configuration the benchmark times; 4096 seeded rows plus block-edge rows
    compared with the oracle (ids, scores, outputs)."""
    from parity import compare, run_gpu, sample_rows, to_host
    from synthetic import make_workload
    w = make_workload("prefill_128k", DEV)
    m, st = run_gpu(w)
    assert st == 0, f"device status {st}"
    rows = sample_rows(w.Sq, 4096, seed=2)
    rep = compare(oracle_mod, w, *to_host(m), rows=rows)
    print("prefill_128k", rep)


def test_repeat_calls_are_bit_identical(msa_lib):
    from parity import run_gpu, to_host
    from synthetic import make_inputs
    w = make_inputs(B=3, Sq=1, lens=[9000, 3001, 17000], H_q=64, H_kv=8, top_k=16, seed=21,
                    device=DEV)
    a = to_host(run_gpu(w)[0])
    b = to_host(run_gpu(w)[0])
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_bad_lengths_set_device_status(msa_lib):
    """lens beyond max_kv_len or past kv_capacity: the kernels' own range
    checks skip the sequence, write -1/-inf/NaN and raise the status word."""
    import block_sparse_attention_43_b200 as m
    from synthetic import make_inputs
    w = make_inputs(B=3, Sq=1, lens=[1000, 2000, 3000], H_q=16, H_kv=2, top_k=4, seed=5,
                    device=DEV)
    eng = m.MSA(batch=3, q_len=1, max_kv_len=3000, num_q_heads=16, num_kv_heads=2, top_k=4,
                kv_capacity=w.kv_capacity, device=DEV)
    bad = torch.tensor([1000, 4000, 3000], dtype=torch.int32, device=DEV)    # 4000 > max
    eng.index_topk(w.q_idx, w.k_idx, bad, w.kv_offsets)
    assert m.msa_read_device_status(eng.ws_index) == 6
    ids = eng.block_ids.cpu()
    assert (ids[1] == -1).all() and (ids[0, 0, :, 0] >= 0).all()
    eng.sparse_attention(w.q, w.k, w.v, bad, w.kv_offsets)
    assert m.msa_read_device_status(eng.ws_attn) == 6
    out = eng.out.float().cpu()
    assert torch.isnan(out[1]).all() and torch.isfinite(out[0]).all()
    # Offsets running past the cache.
    offs = w.kv_offsets.clone()
    offs[2] = w.kv_capacity - 10
    eng.index_topk(w.q_idx, w.k_idx, w.lens, offs)
    assert m.msa_read_device_status(eng.ws_index) == 6
    # A clean call clears the word again.
    eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets)
    assert m.msa_read_device_status(eng.ws_index) == 0


def test_bad_lengths_prefill_path(msa_lib):
    """The block-outer prefill path (groups of 8) reports an out-of-range
    length the same way: status word raised, NaN output for that sequence,
    the other sequence finite."""
    import block_sparse_attention_43_b200 as m
    from synthetic import make_inputs
    w = make_inputs(B=2, Sq=300, lens=[600, 900], H_q=64, H_kv=8, top_k=4, seed=6, device=DEV)
    eng = m.MSA(batch=2, q_len=300, max_kv_len=900, num_q_heads=64, num_kv_heads=8, top_k=4,
                kv_capacity=w.kv_capacity, device=DEV)
    eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets)
    bad = torch.tensor([600, 5000], dtype=torch.int32, device=DEV)     # 5000 > max_kv_len
    eng.sparse_attention(w.q, w.k, w.v, bad, w.kv_offsets)
    assert m.msa_read_device_status(eng.ws_attn) == 6
    out = eng.out.float().cpu()
    assert torch.isnan(out[1]).all() and torch.isfinite(out[0]).all()
