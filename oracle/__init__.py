"""CPU oracle for MiniMax Sparse Attention (MSA) -- TEST INFRASTRUCTURE ONLY.

This package wraps ``msa_oracle.c``: a plain, slow, double-precision C
restatement of the method (index branch: one index query per GQA group, plain
dot product with every visible index key, block max-pool over 128-token
blocks, top-k with the own block kept and ties to the lower id; sparse branch:
exact softmax attention over the kept blocks, shared by the group's heads).
Index-branch variants: fewer index heads than groups (contiguous sets of
groups share one index head's selection), index keys shared by every index
head, and FP8 E4M3 index keys with one fp32 scale per key row.  The sparse
branch's backward (dQ, dK, dV over the kept keys) is here too.
The sources are the cloud.tencent.com MSA article, sections 二 and 六, and the
mlqm.cn guide's configuration-file passage.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never imports, links
or calls it, and this package imports nothing from the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_SO = os.path.join(_HERE, "libmsa_oracle.so")
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_int64
        lib.oracle_index_topk.argtypes = [I, I, I, I, I, I, P, P, P, P, L, P, L, P, P, P, I, P, I]
        lib.oracle_index_topk.restype = I
        lib.oracle_sparse_attention.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, L,
                                                ctypes.c_double, P, L, P, P, I]
        lib.oracle_sparse_attention.restype = I
        lib.oracle_index_topk_ex.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, L, P, L, P, P,
                                             P, I, P, I]
        lib.oracle_index_topk_ex.restype = I
        lib.oracle_sparse_attention_ex.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, P, L,
                                                   ctypes.c_double, P, L, P, P, I]
        lib.oracle_sparse_attention_ex.restype = I
        lib.oracle_sparse_attention_backward.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, P,
                                                         P, L, ctypes.c_double, P, P, P, I]
        lib.oracle_sparse_attention_backward.restype = I
        lib.oracle_e4m3_to_double.argtypes = [I]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def e4m3_to_float(x: int) -> float:
    """Value of one FP8 E4M3 byte (OCP E4M3FN: bias 7, no infinities)."""
    return _load().oracle_e4m3_to_double(int(x))


def index_topk(q_idx, k_idx, lens, kv_offsets, *, block=128, top_k=16, rows=None,
               want_all_scores=False, n_threads=None, k_scale=None):
    """Index branch.  Shapes: q_idx [B,Sq,H,D] (bf16 bits as uint16; H index
    heads), k_idx [T,KH,D] (packed caches; KH = H, one key per index head, or
    KH = 1, one key per token shared by every index head): uint16 bf16 bits,
    or uint8 FP8 E4M3 bytes together with k_scale [T,KH] float32 (score =
    scale * dot).  lens [B] int32, kv_offsets [B] int64.
    ``rows`` selects flattened query rows r = b*Sq + i (default: all).
    Returns dict(block_ids [R,H,k] int32, block_scores [R,H,k] float32,
    boundary [R,H,2] float64, and all_scores [R,H,nb_max] if asked)."""
    q_idx = _c(q_idx, np.uint16)
    fp8 = np.asarray(k_idx).dtype == np.uint8
    k_idx = _c(k_idx, np.uint8 if fp8 else np.uint16)
    lens = _c(lens, np.int32)
    kv_offsets = _c(kv_offsets, np.int64)
    B, Sq, H_kv, D = q_idx.shape
    T, KH = k_idx.shape[:2]
    assert k_idx.shape[2] == D and KH in (1, H_kv)
    if fp8:
        assert k_scale is not None
        k_scale = _c(k_scale, np.float32)
        assert k_scale.shape == (T, KH)
    else:
        assert k_scale is None
    rows_a = None if rows is None else _c(rows, np.int64)
    R = B * Sq if rows_a is None else rows_a.shape[0]
    ids = np.empty((R, H_kv, top_k), np.int32)
    sc = np.empty((R, H_kv, top_k), np.float32)
    bnd = np.empty((R, H_kv, 2), np.float64)
    nb_max = int((int(lens.max()) + block - 1) // block)
    allsc = np.empty((R, H_kv, nb_max), np.float64) if want_all_scores else None
    rc = _load().oracle_index_topk_ex(B, Sq, H_kv, KH, D, block, top_k, _ptr(q_idx),
                                      None if fp8 else _ptr(k_idx), _ptr(k_idx) if fp8 else None,
                                      _ptr(k_scale), _ptr(lens), _ptr(kv_offsets), T,
                                      _ptr(rows_a), R, _ptr(ids), _ptr(sc), _ptr(allsc), nb_max,
                                      _ptr(bnd), n_threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_index_topk rejected its input (code {rc})")
    res = dict(block_ids=ids, block_scores=sc, boundary=bnd)
    if want_all_scores:
        res["all_scores"] = allsc
    return res


def sparse_attention(q, k, v, block_ids, lens, kv_offsets, *, block=128, scale=None,
                     rows=None, want_wsum=False, n_threads=None, num_index_heads=None):
    """Sparse branch.  Shapes: q [B,Sq,H_q,D], k/v [T,H_kv,D] (uint16 bf16 bits),
    block_ids [B*Sq, n_idx, k] (indexed by the flattened row r, whatever rows
    are requested; n_idx = num_index_heads, default H_kv; group g uses index
    head g // (H_kv // n_idx)).  Returns out [R,H_q,D] float64 (and wsum
    [R,H_q])."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    lens = _c(lens, np.int32)
    kv_offsets = _c(kv_offsets, np.int64)
    B, Sq, H_q, D = q.shape
    T, H_kv, _ = k.shape
    n_idx = H_kv if num_index_heads is None else int(num_index_heads)
    ids = _c(block_ids, np.int32).reshape(B * Sq, n_idx, -1)
    top_k = ids.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    rows_a = None if rows is None else _c(rows, np.int64)
    R = B * Sq if rows_a is None else rows_a.shape[0]
    out = np.empty((R, H_q, D), np.float64)
    ws = np.empty((R, H_q), np.float64) if want_wsum else None
    rc = _load().oracle_sparse_attention_ex(B, Sq, H_q, H_kv, n_idx, D, block, top_k, _ptr(q),
                                            _ptr(k), _ptr(v), _ptr(ids), _ptr(lens),
                                            _ptr(kv_offsets), T, float(scale), _ptr(rows_a), R,
                                            _ptr(out), _ptr(ws), n_threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_sparse_attention rejected its input (code {rc})")
    return (out, ws) if want_wsum else out


def sparse_attention_backward(q, k, v, dout, block_ids, lens, kv_offsets, *, block=128,
                              scale=None, num_index_heads=None, n_threads=None):
    """Backward of the sparse branch.  Shapes as sparse_attention, plus dout
    [B,Sq,H_q,D] (uint16 bf16 bits).  Returns (dq [B*Sq,H_q,D], dk [T,H_kv,D],
    dv [T,H_kv,D]), float64; dk/dv are zero on keys no row kept.  Each thread
    owns whole (sequence, group) jobs and adds into dk/dv without locks, so
    with n_threads > 1 the sequences must not share cache rows."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    dout = _c(dout, np.uint16)
    lens = _c(lens, np.int32)
    kv_offsets = _c(kv_offsets, np.int64)
    B, Sq, H_q, D = q.shape
    T, H_kv, _ = k.shape
    assert dout.shape == q.shape
    n_idx = H_kv if num_index_heads is None else int(num_index_heads)
    ids = _c(block_ids, np.int32).reshape(B * Sq, n_idx, -1)
    top_k = ids.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dq = np.empty((B * Sq, H_q, D), np.float64)
    dk = np.zeros((T, H_kv, D), np.float64)
    dv = np.zeros((T, H_kv, D), np.float64)
    rc = _load().oracle_sparse_attention_backward(B, Sq, H_q, H_kv, n_idx, D, block, top_k,
                                                  _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(ids),
                                                  _ptr(lens), _ptr(kv_offsets), T, float(scale),
                                                  _ptr(dq), _ptr(dk), _ptr(dv),
                                                  n_threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_sparse_attention_backward rejected its input (code {rc})")
    return dq, dk, dv
