"""Shared parity checks: the CUDA library (through its C ABI) against the CPU
oracle on the same seeded inputs.

Tolerances (written here, used by every GPU test):
  - block ids: bit-exact, except at a near tie, where the oracle's last kept
    and first dropped non-own block scores differ by <= 1e-5 relative; there
    the kept sets may differ in that one slot, and the outputs are compared
    with the oracle run on the GPU's own selection;
  - block scores: |gpu - oracle| <= 1e-5 * |q_idx| * max |k_idx| (the norm
    of the row's index query times the largest key norm in that block, scaled
    keys for E4M3).  A block score is one 128-term dot product; a dot's
    rounding error is relative to the sum of its terms' magnitudes, which
    Cauchy-Schwarz bounds by that product, not to the dot itself, which may
    be near zero.  The scores of ids that both sides kept are compared on
    every row, near ties included;
  - outputs (bf16): max-abs <= 2e-2 and relative L2 <= 5e-3 against the
    oracle's double result.
"""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_attention_43_b200 as msa
from synthetic import bf16_bits

NEAR_TIE_REL = 1e-5
SCORE_REL = 1e-5
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 5e-3


def run_gpu(w, *, stream=None):
    """Both stages through the C ABI on the workload's device tensors."""
    m = msa.MSA(batch=w.B, q_len=w.Sq, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=w.q.device)
    m.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets, stream)
    m.sparse_attention(w.q, w.k, w.v, w.lens, w.kv_offsets, stream=stream)
    torch.cuda.synchronize()
    st = m.device_status()
    return m, st


def host_inputs(w):
    return dict(q_idx=bf16_bits(w.q_idx), k_idx=bf16_bits(w.k_idx), q=bf16_bits(w.q),
                k=bf16_bits(w.k), v=bf16_bits(w.v), lens=w.lens.cpu().numpy(),
                kv_offsets=w.kv_offsets.cpu().numpy())


def compare_index(oracle_mod, w, gpu_ids, gpu_scores, rows=None, host=None):
    """Block ids and scores of `rows` (flattened b*Sq+i; None = all) against
    the oracle's index branch.  Returns (rows, gpu ids of those rows, report)."""
    a = host if host is not None else host_inputs(w)
    R = w.B * w.Sq
    H = a["q_idx"].shape[2]                    # index heads (k_idx may be shared or E4M3)
    rows_a = np.arange(R, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    ref = oracle_mod.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["kv_offsets"],
                                block=w.block, top_k=w.top_k, rows=rows_a,
                                k_scale=a.get("k_scale"))
    g_ids = gpu_ids.reshape(R, H, w.top_k)[rows_a]
    g_sc = gpu_scores.reshape(R, H, w.top_k)[rows_a]
    o_ids, o_sc, bnd = ref["block_ids"], ref["block_scores"], ref["boundary"]

    same = (g_ids == o_ids).all(axis=-1)
    ties = 0
    for r, g in zip(*np.nonzero(~same)):
        last_in, first_out = bnd[r, g]
        gap = abs(last_in - first_out)
        tol = NEAR_TIE_REL * max(abs(last_in), abs(first_out))
        assert np.isfinite(first_out) and gap <= tol, (
            f"block ids differ at row {rows_a[r]} group {g}: gpu {g_ids[r, g].tolist()} "
            f"oracle {o_ids[r, g].tolist()} (boundary {last_in} vs {first_out})")
        diff = set(g_ids[r, g].tolist()) ^ set(o_ids[r, g].tolist())
        assert len(diff) == 2, (rows_a[r], g, diff)
        ties += 1
    # Scores of the ids both sides kept (on near-tie rows too: every kept id
    # the two selections share).
    eq = (g_ids[..., :, None] == o_ids[..., None, :]) & (o_ids[..., None, :] >= 0)
    m = eq.any(-1)                             # [R, H, k] over the gpu's slots
    o_matched = np.take_along_axis(o_sc, eq.argmax(-1), axis=-1)
    err = np.abs(g_sc[m].astype(np.float64) - o_matched[m].astype(np.float64))
    scale = _score_scale(a, w, rows_a, g_ids)
    lim = SCORE_REL * scale[m]
    assert (err <= lim).all(), f"block scores off by up to {err.max()} (limit {lim[err > lim].min()})"
    assert (g_sc[~(o_ids >= 0) & same[..., None]] == -np.inf).all()
    return rows_a, g_ids, dict(rows=len(rows_a), near_ties=ties,
                               score_err=float(err.max()) if err.size else 0.0)


def _key_rows(a, rows):
    """Index keys of token rows `rows` (any shape) as float64 [..., KH, D],
    E4M3 codes decoded and multiplied by their row scale."""
    k = a["k_idx"][rows]
    if k.dtype == np.uint8:
        dec = torch.from_numpy(np.ascontiguousarray(k)).view(torch.float8_e4m3fn).double().numpy()
        return dec * a["k_scale"][rows][..., None].astype(np.float64)
    return (k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _score_scale(a, w, rows_a, ids):
    """|q_idx| * (largest key norm in the block) for every (row, index head,
    slot) of `ids` ([R, H, k], -1 = empty); the natural scale of a block
    score's rounding error."""
    q = a["q_idx"]
    B, Sq, H = q.shape[:3]
    KH = a["k_idx"].shape[1]
    qf = (q.reshape(B * Sq, H, -1)[rows_a].astype(np.uint32) << 16).view(np.float32)
    qn = np.linalg.norm(qf.astype(np.float64), axis=-1)            # [R, H]
    lens = np.asarray(a["lens"], np.int64)
    offs = np.asarray(a["kv_offsets"], np.int64)
    b_of = rows_a // Sq
    hh = np.broadcast_to(np.arange(H)[None, :, None], ids.shape)
    bb = np.broadcast_to(b_of[:, None, None], ids.shape)
    kh = hh if KH > 1 else np.zeros_like(hh)
    valid = ids >= 0
    trip = np.stack([bb[valid], np.asarray(ids)[valid].astype(np.int64), kh[valid]], axis=1)
    uniq, inv = np.unique(trip, axis=0, return_inverse=True)
    kmax = np.zeros(len(uniq))
    for c0 in range(0, len(uniq), 512):
        u = uniq[c0:c0 + 512]
        t = np.arange(w.block)[None, :] + w.block * u[:, 1:2]       # token positions
        ok = t < lens[u[:, 0]][:, None]
        rows_t = np.where(ok, offs[u[:, 0]][:, None] + t, offs[u[:, 0]][:, None])
        kr = _key_rows(a, rows_t)                                     # [n, 128, KH, D]
        kr = np.take_along_axis(kr, u[:, 2][:, None, None, None], axis=2)[:, :, 0]
        kn = np.linalg.norm(kr, axis=-1)                              # [n, 128]
        kmax[c0:c0 + 512] = np.where(ok, kn, 0.0).max(axis=1)
    out = np.zeros(ids.shape)
    out[valid] = kmax[inv.reshape(-1)] * np.broadcast_to(qn[..., None], ids.shape)[valid]
    return out


def compare(oracle_mod, w, gpu_ids, gpu_scores, gpu_out, rows=None, host=None):
    """Checks one run (ids, scores, outputs) against the oracle on `rows`.
    Returns a small report dict; raises AssertionError on a mismatch."""
    a = host if host is not None else host_inputs(w)
    R = w.B * w.Sq
    rows_a, g_ids, rep = compare_index(oracle_mod, w, gpu_ids, gpu_scores, rows=rows, host=a)

    # Outputs: oracle attention on the GPU's own selection (identical to the
    # oracle's except at near ties).
    H = a["q_idx"].shape[2]
    full_ids = np.full((R, H, w.top_k), -1, np.int32)
    full_ids[rows_a] = g_ids
    o_out = oracle_mod.sparse_attention(a["q"], a["k"], a["v"], full_ids, a["lens"],
                                        a["kv_offsets"], block=w.block, scale=w.scale, rows=rows_a,
                                        num_index_heads=H)
    g_out = gpu_out.reshape(R, w.H_q, w.D)[rows_a].astype(np.float64)
    assert np.isfinite(g_out).all(), "non-finite output"
    d = np.abs(g_out - o_out)
    max_abs = float(d.max())
    rel_l2 = float(np.linalg.norm(g_out - o_out) / max(np.linalg.norm(o_out), 1e-30))
    assert max_abs <= OUT_MAX_ABS, f"max-abs {max_abs}"
    assert rel_l2 <= OUT_REL_L2, f"rel-L2 {rel_l2}"
    rep.update(max_abs=max_abs, rel_l2=rel_l2)
    return rep


def sample_rows(n, count, seed):
    """`count` seeded distinct rows of [0, n) plus the block-edge rows."""
    g = np.random.default_rng(seed)
    pick = set(g.choice(n, size=min(count, n), replace=False).tolist())
    pick |= {x for x in (0, 1, 127, 128, 129, 2047, 2048, n - 1) if 0 <= x < n}
    return np.array(sorted(pick), np.int64)


def to_host(m):
    ids = m.block_ids.cpu().numpy()
    sc = m.block_scores.cpu().numpy()
    out = m.out.float().cpu().numpy()
    return ids, sc, out


def oracle_rows_backward(oracle_mod, q, k, v, dout, ids, pos, scale, parts=8):
    """Backward of independent rows (row i at position pos[i]) over one shared
    cache: each row is its own single-row sequence at offset 0.  The oracle's
    threads each own whole (sequence, group) jobs and assume sequences do not
    share cache rows, so the rows go in `parts` single-threaded calls on
    separate outputs, run side by side, and the dK, dV parts are summed."""
    from concurrent.futures import ThreadPoolExecutor
    n = len(pos)
    cuts = np.linspace(0, n, parts + 1).astype(int)

    def one(a, b):
        return oracle_mod.sparse_attention_backward(
            q[a:b], k, v, dout[a:b], ids[a:b], (pos[a:b] + 1).astype(np.int32),
            np.zeros(b - a, np.int64), scale=scale, n_threads=1)

    with ThreadPoolExecutor(parts) as ex:
        res = list(ex.map(lambda ab: one(*ab), [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]))
    return (np.concatenate([r[0] for r in res]), sum(r[1] for r in res), sum(r[2] for r in res))
