"""The bounded device waits, made to run out on purpose.

Every wait inside the kernels gives up after a limit, records
MSA_ERR_DEVICE_TIMEOUT in the workspace status word, lets the copies it
issued land and returns; nothing traps.  Here msa_set_wait_controls shortens
the limit to 1 ms and makes one kernel wait on something that never happens
(an mbarrier nobody arrives on, a flag nobody sets).  Each test checks that
the call returns at once, that the status word reports the timeout, and that
the next call on the same workspace, with the controls cleared, returns
MSA_OK with results equal to the CPU oracle's."""
import time

import pytest
import torch

import block_sparse_attention_43_b200 as m

pytestmark = pytest.mark.gpu
DEV = "cuda"
LIMIT_NS = 1_000_000


@pytest.fixture
def controls():
    yield m.msa_set_wait_controls
    m.msa_set_wait_controls(0, m.STALL_NONE)


def _workload():
    from synthetic import make_inputs
    return make_inputs(B=3, Sq=1, lens=[9000, 700, 40000], H_q=64, H_kv=8, top_k=16, seed=91,
                       device=DEV)


def _timed(fn):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fn()
    torch.cuda.synchronize()
    return time.perf_counter() - t0


def test_index_decode_wait_gives_up_and_next_call_is_clean(oracle_mod, controls):
    from parity import compare, to_host
    w = _workload()
    eng = m.MSA(batch=w.B, q_len=1, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=DEV)
    controls(LIMIT_NS, m.STALL_INDEX_DECODE)
    dt = _timed(lambda: eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets))
    assert m.msa_read_device_status(eng.ws_index) == 5, "expected MSA_ERR_DEVICE_TIMEOUT"
    assert dt < 1.0, f"a 1 ms wait limit took {dt:.3f} s to give up"

    controls(0, m.STALL_NONE)
    eng.forward(w.q_idx, w.k_idx, w.q, w.k, w.v, w.lens, w.kv_offsets)
    torch.cuda.synchronize()
    assert eng.device_status() == 0
    compare(oracle_mod, w, *to_host(eng))


def test_decode_step_flag_wait_gives_up_and_next_call_is_clean(oracle_mod, controls):
    from parity import compare, to_host
    w = _workload()
    eng = m.MSA(batch=w.B, q_len=1, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=DEV)
    controls(LIMIT_NS, m.STALL_DECODE_STEP)
    dt = _timed(lambda: eng.decode_step(w.q_idx, w.k_idx, w.q, w.k, w.v, w.lens, w.kv_offsets))
    assert m.msa_read_device_status(eng.ws_step) == 5, "expected MSA_ERR_DEVICE_TIMEOUT"
    assert dt < 1.0, f"a 1 ms wait limit took {dt:.3f} s to give up"

    controls(0, m.STALL_NONE)
    eng.decode_step(w.q_idx, w.k_idx, w.q, w.k, w.v, w.lens, w.kv_offsets)
    torch.cuda.synchronize()
    assert m.msa_read_device_status(eng.ws_step) == 0
    compare(oracle_mod, w, *to_host(eng))
