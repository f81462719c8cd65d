"""Benchmark of the MSA hot path on B200: one step = the whole decode path
(index score + block max-pool, top-k, sparse attention with split-K merge)
for one batch, through the C ABI; a decode run also times the same decode
step as one fused cooperative launch, the decode step on the index-branch
variants (fewer index heads, shared index keys, E4M3 index keys), the sparse
branch's backward on the 2k-row prefill, and one
128k-token prefill (index GEMM + fused top-k, sparse attention) as
sub-objects.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode_1m]
                    [--impl msa|reference] [--no-cpu-baseline] [--no-e2e]
                    [--no-prefill] [--no-fused] [--no-variants] [--no-backward]
                    [--prefill-steps S]
                    [--prefill-len N]

Prints ONE JSON line (rank 0).  N > 1 runs under torchrun: every rank runs
its own independent batch (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSA decode HBM GB/s (% of 8 TB/s) & prefill sparse-attn TFLOP/s, 128k/1M"
DOMINANT = "index_score_maxpool_decode"
DOMINANT_SRC = os.path.join(ROOT, "block_sparse_attention_43_b200", "csrc", "index_decode.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode_1m",
                    choices=["decode_1m", "decode_32k", "decode_ragged", "prefill_128k",
                             "prefill_2k"])
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill_128k measurement attached to a decode run")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the index-branch variant measurement attached to a decode run")
    ap.add_argument("--no-fused", action="store_true",
                    help="skip the single-launch decode step attached to a decode run")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the sparse-branch backward measurement attached to a decode run")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other four workloads attached to a decode_1m run")
    ap.add_argument("--cpu-rows", type=int, default=4096,
                    help="query rows of the prefill_128k oracle sample (CPU baseline)")
    ap.add_argument("--prefill-steps", type=int, default=5)
    ap.add_argument("--prefill-len", type=int, default=None,
                    help="override the prefill length (profiling captures of a smaller case)")
    ap.add_argument("--decode-len", type=int, default=None,
                    help="override the decode context length (profiling captures of a smaller case)")
    ap.add_argument("--backward-rows", type=int, default=None,
                    help="only time the backward on the prefill_128k recipe at this many rows "
                         "(profiling captures); prints its JSON object")
    return ap.parse_args()


# ----------------------------------------------------------------------------- bytes
def decode_step_bytes(w, ids_host):
    """Bytes the decode path must move per step: every index key of every
    sequence, the valid tokens of the kept K/V blocks, q, q_idx, out, ids and
    scores."""
    lens = np.asarray(w.lens_host, np.int64)
    k_idx = int(lens.sum()) * w.H_kv * w.d_idx * 2
    kv = 0
    ids = ids_host.reshape(w.B, w.H_kv, w.top_k)
    for b in range(w.B):
        L = int(lens[b])
        for g in range(w.H_kv):
            for j in ids[b, g]:
                if j >= 0:
                    kv += min(128, L - 128 * int(j))
    kv *= w.D * 2 * 2
    small = w.B * w.H_q * w.D * 2 * 2 + w.B * w.H_kv * w.d_idx * 2 + w.B * w.H_kv * w.top_k * 8
    return k_idx + kv + small, k_idx


def index_kernel_bytes(w):
    lens = np.asarray(w.lens_host, np.int64)
    nb = (lens + 127) // 128
    return int(lens.sum()) * w.H_kv * w.d_idx * 2 + w.B * w.H_kv * w.d_idx * 2 + int(nb.sum()) * w.H_kv * 4


def prefill_useful_flops(w, ids_host):
    """Useful sparse-branch FLOPs: 4*D per (row, head, visible kept key)."""
    ids = ids_host.reshape(w.B, w.Sq, w.H_kv, w.top_k).astype(np.int64)
    keys = 0
    for b in range(w.B):
        L = w.lens_host[b]
        p = np.arange(w.Sq, dtype=np.int64) + (L - w.Sq)
        own = p // 128
        idb = ids[b]
        vis = np.where(idb == own[:, None, None], (p % 128 + 1)[:, None, None], 128)
        keys += int((vis * (idb >= 0)).sum())
    return keys * (w.H_q // w.H_kv) * 4 * w.D


def prefill_index_flops(w):
    """Index-branch FLOPs of the causal product: 2*d_idx per (row, group, visible token)."""
    f = 0
    for b in range(w.B):
        L = w.lens_host[b]
        p = np.arange(w.Sq, dtype=np.int64) + (L - w.Sq)
        f += int((p + 1).sum())
    return f * w.H_kv * 2 * w.d_idx


def measure_prefill(name, dev, steps, warmup, seq_len=None):
    """Times msa_index_topk + msa_sparse_attention on a prefill workload;
    per-kernel times come from the library's CUDA-event trace."""
    import block_sparse_attention_43_b200 as msa
    from synthetic import WORKLOADS, make_inputs, make_workload
    if seq_len is None:
        w = make_workload(name, dev)
    else:
        c = WORKLOADS[name]
        w = make_inputs(B=c["B"], Sq=seq_len, lens=[seq_len] * c["B"], H_q=c["H_q"],
                        H_kv=c["H_kv"], top_k=c["top_k"], seed=c["seed"], device=dev,
                        name=f"{name}@{seq_len}")
    stream = torch.cuda.Stream(device=dev)
    eng = msa.MSA(batch=w.B, q_len=w.Sq, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                  num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=dev)

    def step():
        eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets, stream)
        eng.sparse_attention(w.q, w.k, w.v, w.lens, w.kv_offsets, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    st = eng.device_status(stream)
    if st != 0:
        raise RuntimeError(f"prefill device status {msa.STATUS_NAMES.get(st, st)}")
    # (row, head) pairs the block-outer path handed to its exact fp32 pass
    # (a count the kernels keep in the attention workspace header)
    flagged = int(eng.ws_attn[4:8].view(torch.int32).item()) if w.H_q // w.H_kv == 8 else 0
    useful = prefill_useful_flops(w, eng.block_ids.cpu().numpy())
    idx_flops = prefill_index_flops(w)
    msa.msa_trace_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    trace = msa.msa_trace_read()
    msa.msa_trace_enable(False)
    ms_step = ev0.elapsed_time(ev1) / steps
    per = {}
    for n, t in trace:
        per[n] = per.get(n, 0.0) + t / steps
    idx_ms = sum(t for n, t in per.items() if n.startswith("index_"))
    att_ms = sum(t for n, t in per.items() if n.startswith("prefill_") or n.startswith("sparse_"))
    res = {"workload": w.name, "rows": w.B * w.Sq, "H_q": w.H_q, "H_kv": w.H_kv,
           "top_k": w.top_k, "ms_per_step": ms_step,
           "sparse_attn_useful_tflop": useful / 1e12,
           "sparse_attn_ms": att_ms, "sparse_attn_tflops": useful / (att_ms / 1e3) / 1e12,
           "index_tflop": idx_flops / 1e12, "index_ms": idx_ms,
           "index_tflops": idx_flops / (idx_ms / 1e3) / 1e12,
           "kernel_ms": per, "gpu_launches_per_step": len(trace) / steps,
           "exact_pass_row_heads": flagged}
    del eng, w
    torch.cuda.empty_cache()
    return res


def measure_backward(name, dev, steps, warmup, seq_len=None):
    """Times one msa_sparse_attention_backward call (the forward recomputed
    for the log-sum-exp, Delta, buckets, the block-outer kernel and the dQ
    conversion) on a prefill workload's own selection, with CUDA events on
    its stream; per-kernel times come from the library's trace.  Useful
    FLOPs: 10*D per (row, head, visible kept key) -- the five products
    S = QK^T, dP = dO V^T, dV += P^T dO, dK += dS^T Q, dQ += dS K."""
    import block_sparse_attention_43_b200 as msa
    from synthetic import WORKLOADS, make_inputs, make_workload
    if seq_len is None:
        w = make_workload(name, dev)
    else:
        c = WORKLOADS[name]
        w = make_inputs(B=c["B"], Sq=seq_len, lens=[seq_len] * c["B"], H_q=c["H_q"],
                        H_kv=c["H_kv"], top_k=c["top_k"], seed=c["seed"], device=dev,
                        name=f"{name}@{seq_len}")
    eng = msa.MSA(batch=w.B, q_len=w.Sq, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                  num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=dev)
    stream = torch.cuda.Stream(device=dev)
    eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets, stream)
    g = torch.Generator(device=dev).manual_seed(1)
    dout = torch.randn(w.q.shape, generator=g, device=dev).to(torch.bfloat16)
    dq = torch.empty_like(w.q)
    dk = torch.zeros(w.k.shape, dtype=torch.float32, device=dev)
    dv = torch.zeros(w.v.shape, dtype=torch.float32, device=dev)
    ws = msa.alloc_workspace(msa.msa_sparse_attention_backward_workspace_size(eng.shape), dev)

    def step():
        msa.msa_sparse_attention_backward(eng.shape, w.q, w.k, w.v, eng.block_ids, w.lens,
                                          w.kv_offsets, w.scale, dout, dq, dk, dv, ws, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    st = msa.msa_read_device_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"backward device status {msa.STATUS_NAMES.get(st, st)}")
    ids = eng.block_ids.cpu().numpy()
    fwd_useful = prefill_useful_flops(w, ids)             # 4*D per (row, head, key)
    useful = fwd_useful * 10 // 4
    kept = int((ids >= 0).sum()) * (w.H_q // w.H_kv)      # (row, head, kept block)
    msa.msa_trace_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    trace = msa.msa_trace_read()
    msa.msa_trace_enable(False)
    ms = ev0.elapsed_time(ev1) / steps
    per = {}
    for n, t in trace:
        per[n] = per.get(n, 0.0) + t / steps
    blocks_ms = per.get("backward_blocks", float("nan"))
    _, tf_burst, _, kind = measured_peaks()
    tflops = useful / (ms / 1e3) / 1e12
    res = {"workload": w.name, "rows": w.B * w.Sq, "H_q": w.H_q, "H_kv": w.H_kv, "top_k": w.top_k,
           "ms": ms, "useful_tflop": useful / 1e12, "tflops": tflops,
           "frac_of_bf16_burst": tflops / tf_burst,
           "kernels_ms": {k: round(v, 4) for k, v in sorted(per.items())},
           "blocks_kernel": {"ms": blocks_ms,
                             "tflops": useful / (blocks_ms / 1e3) / 1e12,
                             "frac_of_bf16_burst": useful / (blocks_ms / 1e3) / 1e12 / tf_burst},
           "dq_reduction_bytes": kept * w.D * 4,
           "note": "ms covers the whole call, the forward recompute included; useful FLOPs "
                   "count the backward's five products only",
           "peak_kind": kind}
    del eng, w, ws
    torch.cuda.empty_cache()
    return res


def _variant_keys(w, Hi, fmt, msa):
    """Index queries / keys of an index-branch variant, built from w's tensors
    (per-head keys are the first Hi groups' keys; shared keys the first
    group's; E4M3 codes quantised per key row in chunks)."""
    from synthetic import quantize_e4m3_rows
    shared = fmt in (msa.INDEX_KEYS_BF16_SHARED, msa.INDEX_KEYS_FP8_SHARED)
    q_idx = w.q_idx[:, :, :Hi].contiguous()
    src = w.k_idx[:, :1 if shared else Hi]
    if fmt in (msa.INDEX_KEYS_BF16, msa.INDEX_KEYS_BF16_SHARED):
        return q_idx, src.contiguous(), None
    T = src.shape[0]
    codes = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    scale = torch.empty(src.shape[:2], dtype=torch.float32, device=src.device)
    step = 1 << 20
    for t0 in range(0, T, step):
        c, s = quantize_e4m3_rows(src[t0:t0 + step])
        codes[t0:t0 + step] = c
        scale[t0:t0 + step] = s
    return q_idx, codes, scale


def measure_index_variants(w, dev, steps, warmup):
    """Decode step (index + top-k + sparse attention) on the index-branch
    variants: the guide's 4 index heads for 8 groups (bf16 keys per head),
    keys shared by the index heads (bf16, E4M3) and E4M3 keys per head.
    Index bytes = keys (+ row scales) + index queries + block scores."""
    import block_sparse_attention_43_b200 as msa
    peak, _, _, kind = measured_peaks()
    lens = np.asarray(w.lens_host, np.int64)
    nb = int(((lens + 127) // 128).sum())
    ntok = int(lens.sum())
    cases = [("4_index_heads_bf16", 4, msa.INDEX_KEYS_BF16),
             ("shared_keys_bf16", w.H_kv, msa.INDEX_KEYS_BF16_SHARED),
             ("per_head_keys_fp8", w.H_kv, msa.INDEX_KEYS_FP8),
             ("shared_keys_fp8", w.H_kv, msa.INDEX_KEYS_FP8_SHARED)]
    out = {}
    stream = torch.cuda.Stream(device=dev)
    for name, Hi, fmt in cases:
        q_idx, keys, scale = _variant_keys(w, Hi, fmt, msa)
        eng = msa.MSA(batch=w.B, q_len=1, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                      num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=dev,
                      num_index_heads=Hi, index_key_format=fmt)

        def step():
            eng.index_topk(q_idx, keys, w.lens, w.kv_offsets, stream, k_idx_scale=scale)
            eng.sparse_attention(w.q, w.k, w.v, w.lens, w.kv_offsets, stream=stream)

        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        st = eng.device_status(stream)
        if st != 0:
            raise RuntimeError(f"{name}: device status {msa.STATUS_NAMES.get(st, st)}")
        msa.msa_trace_enable(True)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        trace = msa.msa_trace_read()
        msa.msa_trace_enable(False)
        per = {}
        for n, t in trace:
            per[n] = per.get(n, 0.0) + t / steps
        idx_name = [n for n in per if n.startswith("index_score_maxpool_decode")][0]
        kh = keys.shape[1]
        key_bytes = ntok * kh * w.d_idx * keys.element_size() + (ntok * kh * 4 if scale is not None else 0)
        idx_bytes = key_bytes + w.B * Hi * w.d_idx * 2 + nb * Hi * 4
        gbs = idx_bytes / (per[idx_name] / 1e3) / 1e9
        fused_ms = None
        if fmt == msa.INDEX_KEYS_BF16:
            # the same step as one launch (msa_decode_step takes bf16 keys, one row per index head)
            for _ in range(warmup):
                eng.decode_step(q_idx, keys, w.q, w.k, w.v, w.lens, w.kv_offsets, stream)
            torch.cuda.synchronize()
            st = msa.msa_read_device_status(eng.ws_step, stream)
            if st != 0:
                raise RuntimeError(f"{name} fused: device status {msa.STATUS_NAMES.get(st, st)}")
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                eng.decode_step(q_idx, keys, w.q, w.k, w.v, w.lens, w.kv_offsets, stream)
            e1.record(stream)
            torch.cuda.synchronize()
            fused_ms = e0.elapsed_time(e1) / steps
        out[name] = {"index_heads": Hi, "key_rows_per_token": kh,
                     "fused_step_ms": fused_ms,
                     "key_dtype": "e4m3" if scale is not None else "bf16",
                     "ms_per_step": ev0.elapsed_time(ev1) / steps, "kernel_ms": per,
                     "index_bytes": idx_bytes, "index_gbs": gbs, "index_frac_of_hbm": gbs / peak,
                     "peak_kind": kind}
        del eng, q_idx, keys, scale
        torch.cuda.empty_cache()
    return out


def measure_decode_fused(w, dev, steps, warmup, step_bytes, ref_ids):
    """The same decode step as one cooperative launch (msa_decode_step:
    index scores, top-k and sparse attention fused); GB/s on the same
    algorithmic bytes as the two-call step, and whether its block ids equal
    the two-call path's."""
    import block_sparse_attention_43_b200 as msa
    peak, _, _, kind = measured_peaks()
    stream = torch.cuda.Stream(device=dev)
    eng = msa.MSA(batch=w.B, q_len=1, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                  num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=dev)

    def step():
        eng.decode_step(w.q_idx, w.k_idx, w.q, w.k, w.v, w.lens, w.kv_offsets, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    st = msa.msa_read_device_status(eng.ws_step, stream)
    if st != 0:
        raise RuntimeError(f"decode_step: device status {msa.STATUS_NAMES.get(st, st)}")
    same = bool(np.array_equal(eng.block_ids.cpu().numpy(), ref_ids))
    msa.msa_trace_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    trace = msa.msa_trace_read()
    msa.msa_trace_enable(False)
    ker = [t for n, t in trace if n == "decode_fused_step"]
    ms = ev0.elapsed_time(ev1) / steps
    kms = float(np.mean(ker)) if ker else float("nan")
    gbs = step_bytes / (ms / 1e3) / 1e9
    tr = kernel_traffic("decode_fused_step",
                        os.path.join(ROOT, "block_sparse_attention_43_b200", "csrc", "decode_fused.cu"))
    traffic = None if tr is None else tr["dram_bytes_per_unit"] * (step_bytes / tr["bytes_per_unit_basis"])
    res = {"entry": "msa_decode_step", "ms_per_step": ms, "kernel_ms": kms, "traffic": traffic,
           "algorithmic_bytes": step_bytes,
           "launches_per_step": len(trace) / steps, "gbs": gbs, "frac_of_hbm": gbs / peak,
           "kernel_gbs": step_bytes / (kms / 1e3) / 1e9, "peak_kind": kind,
           "ids_equal_two_call": same}
    del eng
    torch.cuda.empty_cache()
    return res


def measure_decode_config(name, dev, steps, warmup, with_cpu=True):
    """One decode workload at full size: the two-call step (index + top-k,
    sparse attention) timed with CUDA events, the dominant kernel's roofline
    from the library's trace, the same step as one fused launch, and the
    oracle on every sequence of the workload as the CPU baseline."""
    import block_sparse_attention_43_b200 as msa
    from synthetic import make_workload
    w = make_workload(name, dev)
    stream = torch.cuda.Stream(device=dev)
    eng = msa.MSA(batch=w.B, q_len=1, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                  num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=dev)

    def step():
        eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets, stream)
        eng.sparse_attention(w.q, w.k, w.v, w.lens, w.kv_offsets, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    st = eng.device_status(stream)
    if st != 0:
        raise RuntimeError(f"{name}: device status {msa.STATUS_NAMES.get(st, st)}")
    ids_host = eng.block_ids.cpu().numpy()
    step_bytes, kidx_bytes = decode_step_bytes(w, ids_host)
    msa.msa_trace_enable(True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    trace = msa.msa_trace_read()
    msa.msa_trace_enable(False)
    ms = ev0.elapsed_time(ev1) / steps
    per = {}
    for n, t in trace:
        per[n] = per.get(n, 0.0) + t / steps
    dom = [t for n, t in trace if n == DOMINANT]
    dom_ms = float(np.mean(dom))
    peak, _, _, kind = measured_peaks()
    kb = index_kernel_bytes(w)
    gbs = step_bytes / (ms / 1e3) / 1e9
    fused = measure_decode_fused(w, dev, steps, warmup, step_bytes, ids_host)
    cpu = None
    if with_cpu:
        c_gbs, dt, used, note = oracle_sample(w, seqs=range(w.B))
        cpu = {"value": c_gbs, "unit": "GB/s", "cores": host_cores(), "threads_used": used,
               "kind": "oracle", "sample": note, "seconds": dt}
    lens = w.lens_host
    res = {"workload": name, "batch": w.B,
           "context": lens[0] if len(set(lens)) == 1 else
           {"min": min(lens), "max": max(lens), "total": int(sum(lens))},
           "H_q": w.H_q, "H_kv": w.H_kv, "top_k": w.top_k,
           "ms_per_step": ms, "value": gbs, "unit": "GB/s", "pct_of_8TBps": 100.0 * gbs / 8000.0,
           "frac_of_hbm": gbs / peak, "step_bytes": step_bytes, "index_key_bytes": kidx_bytes,
           "tokens_per_s": w.B / (ms / 1e3),
           "l2": "inputs larger than L2 (index keys %.2f GiB)" % (kidx_bytes / 2**30),
           "roofline": {"bound": "hbm", "kernel": DOMINANT, "achieved": kb / (dom_ms / 1e3) / 1e9,
                        "peak": peak, "peak_kind": kind, "unit": "GB/s",
                        "frac": kb / (dom_ms / 1e3) / 1e9 / peak, "algorithmic_bytes": kb,
                        "avg_launch_ms": dom_ms, "traffic": None},
           "kernel_ms": per, "gpu_launches_per_step": len(trace) / steps,
           "decode_step_fused": fused, "cpu_baseline": cpu}
    tr = kernel_traffic()
    if tr is not None:
        res["roofline"]["traffic"] = tr["dram_bytes_per_unit"] * (kb / tr["bytes_per_unit_basis"])
    del eng, w
    torch.cuda.empty_cache()
    return res


def measure_prefill_config(name, dev, steps, warmup, with_cpu=True, cpu_rows=4096):
    """One prefill workload at full size (index GEMM with fused top-k, then
    the sparse branch), its sparse branch's roofline on useful FLOPs, and the
    oracle on a seeded row sample as the CPU baseline."""
    from synthetic import make_workload
    r = measure_prefill(name, dev, steps, warmup)
    _, tf_burst, tf_sus, kind = measured_peaks()
    r["value"] = r["sparse_attn_tflops"]
    r["unit"] = "TFLOP/s"
    r["tokens_per_s"] = r["rows"] / (r["ms_per_step"] / 1e3)
    r["roofline"] = {"bound": "tensor", "kernel": "sparse branch (prefill_* kernels)",
                     "achieved": r["sparse_attn_tflops"], "peak": tf_burst,
                     "peak_kind": kind + " burst", "unit": "TFLOP/s",
                     "frac": r["sparse_attn_tflops"] / tf_burst,
                     "sparse_attn_frac_of_burst": r["sparse_attn_tflops"] / tf_burst,
                     "index_frac_of_burst": r["index_tflops"] / tf_burst,
                     "peak_burst": tf_burst, "peak_sustained": tf_sus, "traffic": None}
    r["cpu_baseline"] = None
    if with_cpu:
        w = make_workload(name, dev)
        rps, dt, used, n, note, _ = oracle_prefill_sample(w, cpu_rows)
        full = w.B * w.Sq
        r["cpu_baseline"] = {"value": rps, "unit": "query rows/s", "cores": host_cores(),
                             "threads_used": used, "kind": "oracle", "sample": note,
                             "seconds": dt, "sample_rows": n,
                             "extrapolated_full_seconds": dt * full / n if n < full else dt,
                             "extrapolation": "linear in rows" if n < full else "none (all rows)"}
        r["gpu_rows_per_s"] = full / (r["ms_per_step"] / 1e3)
        del w
        torch.cuda.empty_cache()
    return r


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- helpers
def measured_peaks():
    """(HBM GB/s, bf16 burst TFLOP/s, bf16 sustained TFLOP/s, source)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_traffic(name=DOMINANT, src=DOMINANT_SRC):
    """Per-launch DRAM bytes of a kernel from its last ncu capture, or None
    when the kernel source changed since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE)).get(name)
    if not d:
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if d.get("source_sha256") != h:
        return None
    return d


def dist_setup(args):
    if args.gpus > 1 or "RANK" in os.environ:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ.get("RANK", 0))
        local = int(os.environ.get("LOCAL_RANK", 0))
        world = int(os.environ.get("WORLD_SIZE", 1))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, rank, local, world
    return None, 0, 0, 1


def max_over_ranks(dist, x, device):
    """The slowest rank's value (every rank calls this, in the same order)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(dist, world, units_per_rank, seconds_local, device):
    """Whole-job throughput: every rank's units over the slowest rank's time.
    Returns (units per second, slowest seconds)."""
    slow = max_over_ranks(dist, seconds_local, device)
    return units_per_rank * world / slow, slow


def host_cores():
    """Cores this process may run on (sched_getaffinity)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- CPU oracle leg
def oracle_sample(w, seqs=(0,)):
    """The oracle, as it stands, on sequences `seqs` of a decode workload
    (index branch over all their index keys + sparse branch), on the host's
    cores.  Returns (GB/s of those sequences' algorithmic bytes, seconds,
    threads the oracle could keep busy, note)."""
    import oracle
    from synthetic import bf16_bits
    seqs = list(seqs)
    lens_l, offs_l, sl = [], [], []
    acc = 0
    for b in seqs:
        L = w.lens_host[b]
        off = int(w.kv_offsets[b])
        sl.append(slice(off, off + L))
        lens_l.append(L)
        offs_l.append(acc)
        acc += L
    cat = lambda t: np.concatenate([bf16_bits(t[x]) for x in sl]) if len(sl) > 1 else bf16_bits(t[sl[0]])
    q_idx = bf16_bits(w.q_idx[seqs])
    q = bf16_bits(w.q[seqs])
    k_idx, k, v = cat(w.k_idx), cat(w.k), cat(w.v)
    lens = np.array(lens_l, np.int32)
    offs = np.array(offs_l, np.int64)
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    sel = oracle.index_topk(q_idx, k_idx, lens, offs, top_k=w.top_k, n_threads=threads)
    oracle.sparse_attention(q, k, v, sel["block_ids"], lens, offs, n_threads=threads)
    dt = time.perf_counter() - t0
    nbytes = int(lens.sum()) * w.H_kv * w.d_idx * 2
    ids = sel["block_ids"].reshape(len(seqs), w.H_kv, w.top_k)
    kv = sum(min(128, lens_l[i] - 128 * int(j)) for i in range(len(seqs)) for j in ids[i].ravel()
             if j >= 0) * w.D * 4
    gbs = (nbytes + kv) / dt / 1e9
    # The oracle spreads (row, group) jobs over threads: a decode row has
    # H_kv index jobs and H_q attention jobs.
    used = min(threads, len(seqs) * w.H_kv)
    what = f"sequence 0 of {w.name} ({lens_l[0]} tokens" if seqs == [0] and w.B > 1 else \
        f"all {len(seqs)} sequences of {w.name} ({int(lens.sum())} tokens"
    return gbs, dt, used, what + f", all {w.H_kv} groups, both stages)"


def oracle_prefill_sample(w, n_rows=4096, seed=2):
    """The oracle, as it stands, on a seeded sample of a prefill workload's
    query rows (uniform without replacement plus the block-edge rows), both
    stages.  Returns (rows/s, seconds, threads, sample rows, note); the whole
    prefill's oracle time is extrapolated linearly from the sample (a uniform
    row sample has the mean per-row cost)."""
    import oracle
    from synthetic import bf16_bits
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import sample_rows
    R = w.B * w.Sq
    rows = sample_rows(R, min(n_rows, R), seed) if n_rows < R else np.arange(R, dtype=np.int64)
    a = dict(q_idx=bf16_bits(w.q_idx), k_idx=bf16_bits(w.k_idx), q=bf16_bits(w.q),
             k=bf16_bits(w.k), v=bf16_bits(w.v), lens=w.lens.cpu().numpy(),
             offs=w.kv_offsets.cpu().numpy())
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    sel = oracle.index_topk(a["q_idx"], a["k_idx"], a["lens"], a["offs"], top_k=w.top_k,
                            rows=rows, n_threads=threads)
    ids = np.full((R, w.H_kv, w.top_k), -1, np.int32)
    ids[rows] = sel["block_ids"]
    oracle.sparse_attention(a["q"], a["k"], a["v"], ids, a["lens"], a["offs"], scale=w.scale,
                            rows=rows, n_threads=threads)
    dt = time.perf_counter() - t0
    # useful sparse-branch FLOPs of the sampled rows (4*D per row, head, visible kept key)
    ids_s = sel["block_ids"].astype(np.int64)
    b_of = rows // w.Sq
    p = rows % w.Sq + (np.asarray(w.lens_host)[b_of] - w.Sq)
    vis = np.where(ids_s == (p // 128)[:, None, None], (p % 128 + 1)[:, None, None], 128)
    useful = int((vis * (ids_s >= 0)).sum()) * (w.H_q // w.H_kv) * 4 * w.D
    used = min(threads, len(rows) * w.H_kv)
    note = (f"{len(rows)} of {R} query rows of {w.name} (seeded uniform sample + block-edge rows), "
            f"all {w.H_kv} groups, both stages" if len(rows) < R else
            f"all {R} query rows of {w.name}, both stages")
    return len(rows) / dt, dt, used, len(rows), note, useful


def run_reference(args):
    dist, rank, local, world = dist_setup(args)
    if rank != 0:
        return
    from synthetic import make_workload
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = make_workload(args.workload, dev)
    prefill = args.workload.startswith("prefill")
    unit = "TFLOP/s" if prefill else "GB/s"
    vals = []
    for i in range(args.warmup + args.steps):
        if prefill:
            # a bounded row sample per step (rows/s scale linearly with rows)
            _, dt, used, _, note, useful = oracle_prefill_sample(w, min(args.cpu_rows, 256), seed=2 + i)
            v = useful / dt / 1e12
        else:
            v, dt, used, note = oracle_sample(w)
        if i >= args.warmup:
            vals.append((v, dt))
    gbs = float(np.mean([v[0] for v in vals]))
    ms = float(np.mean([v[1] for v in vals])) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": gbs, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample": note},
            "cpu_baseline": {"value": gbs, "unit": unit, "cores": host_cores(),
                             "threads_used": used, "kind": "oracle", "sample": note},
            "e2e": {"value": gbs, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main arm
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.backward_rows is not None:
        torch.cuda.set_device(0)
        r = measure_backward("prefill_128k", torch.device("cuda", 0), args.steps, max(args.warmup, 1),
                             seq_len=args.backward_rows)
        print(json.dumps(r), flush=True)
        return
    if args.workload.startswith("prefill"):
        return run_prefill_headline(args)
    import block_sparse_attention_43_b200 as msa
    from synthetic import make_workload

    dist, rank, local, world = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.decode_len is None:
        w = make_workload(args.workload, dev)
    else:
        from synthetic import WORKLOADS, make_inputs
        c = WORKLOADS[args.workload]
        w = make_inputs(B=c["B"], Sq=1, lens=[args.decode_len] * c["B"], H_q=c["H_q"],
                        H_kv=c["H_kv"], top_k=c["top_k"], seed=c["seed"], device=dev,
                        name=f"{args.workload}@{args.decode_len}", needles=c.get("needles", 0),
                        amp=c.get("amp", 4.0))
    if world > 1:
        # independent batch per rank: perturb q so ranks differ
        w.q_idx.mul_(1.0 + 0.001 * rank)
    stream = torch.cuda.Stream(device=dev)
    eng = msa.MSA(batch=w.B, q_len=1, max_kv_len=max(w.lens_host), num_q_heads=w.H_q,
                  num_kv_heads=w.H_kv, top_k=w.top_k, kv_capacity=w.kv_capacity, device=dev)
    torch.cuda.synchronize()

    def step():
        eng.index_topk(w.q_idx, w.k_idx, w.lens, w.kv_offsets, stream)
        eng.sparse_attention(w.q, w.k, w.v, w.lens, w.kv_offsets, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    status = eng.device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {msa.STATUS_NAMES.get(status, status)} after warm-up")
    ids_host = eng.block_ids.cpu().numpy()
    step_bytes, kidx_bytes = decode_step_bytes(w, ids_host)

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    msa.msa_trace_enable(True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms_total = ev0.elapsed_time(ev1)
    trace = msa.msa_trace_read()
    msa.msa_trace_enable(False)
    clk = clocks.stop()

    kb = index_kernel_bytes(w)
    head_cfg = {"workload": args.workload, "batch": w.B, "context": max(w.lens_host),
                "H_q": w.H_q, "H_kv": w.H_kv, "top_k": w.top_k}
    launches = len(trace)
    dom = [t for n, t in trace if n == DOMINANT]
    dom_ms = float(np.mean(dom)) if dom else float("nan")
    shares = {}
    for n, t in trace:
        shares[n] = shares.get(n, 0.0) + t

    rate, slow_s = whole_job_rate(dist, world, step_bytes * args.steps, ms_total / 1e3, dev)
    ms_step = slow_s * 1e3 / args.steps
    value = rate / 1e9

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(w, eng, stream, args, step_bytes, world, dist)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, dt, used, note = oracle_sample(w)
        cpu = {"value": gbs, "unit": "GB/s", "cores": host_cores(), "threads_used": used,
               "kind": "oracle", "sample": note, "seconds": dt}

    fused = None
    if not args.no_fused and world == 1:
        fused = measure_decode_fused(w, dev, max(20, args.steps // 4), 5, step_bytes, ids_host)
        fused["two_call_ms_per_step"] = ms_step

    variants = None
    if not args.no_variants and world == 1:
        variants = measure_index_variants(w, dev, 20, 3)

    backward = None
    if not args.no_backward and world == 1:
        # the 128k prefill recipe at 32,768 rows (the largest backward that
        # keeps the default run short) and the 2k-row prefill
        big = measure_backward("prefill_128k", dev, 5, 2, seq_len=32768)
        _, tf_burst, _, kind = measured_peaks()
        big["roofline"] = {"bound": "tensor", "kernel": "whole backward call (forward recompute included)",
                           "achieved": big["tflops"], "peak": tf_burst, "peak_kind": kind + " burst",
                           "unit": "TFLOP/s", "frac": big["frac_of_bf16_burst"]}
        backward = big                                  # headline: the 32k-row case
        backward["prefill_2k"] = measure_backward("prefill_2k", dev, 20, 3)

    prefill = None
    configs = None
    if world == 1 and (not args.no_prefill or not args.no_configs):
        del eng
        del w
        torch.cuda.empty_cache()
    if not args.no_prefill and world == 1:
        prefill = measure_prefill_config("prefill_128k", dev, args.prefill_steps, 2,
                                         with_cpu=not args.no_cpu_baseline,
                                         cpu_rows=args.cpu_rows)
    if not args.no_configs and world == 1:
        configs = {}
        for name in ("decode_32k", "decode_ragged"):
            configs[name] = measure_decode_config(name, dev, 100, 10,
                                                  with_cpu=not args.no_cpu_baseline)
        configs["prefill_2k"] = measure_prefill_config("prefill_2k", dev, 50, 5,
                                                       with_cpu=not args.no_cpu_baseline)

    peak, _, _, peak_kind = measured_peaks()
    achieved = kb / (dom_ms / 1e3) / 1e9
    if configs is not None:
        # all five workloads side by side (the headline's own figures first)
        configs = {"decode_1m": {"workload": args.workload, "ms_per_step": ms_step, "value": value,
                                 "unit": "GB/s", "pct_of_8TBps": 100.0 * value / 8000.0,
                                 "frac_of_hbm": value / peak, "tokens_per_s": head_cfg["batch"] / (ms_step / 1e3),
                                 "roofline_frac": achieved / peak, "cpu_baseline": cpu,
                                 "detail": "the headline fields of this line"},
                   **configs, "prefill_128k": prefill}
    tr = kernel_traffic()
    traffic = None
    if tr is not None:
        traffic = tr["dram_bytes_per_unit"] * (kb / tr["bytes_per_unit_basis"])
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**head_cfg, "block": 128,
                       "step_bytes": step_bytes, "index_key_bytes": kidx_bytes,
                       "pct_of_8TBps": 100.0 * value / world / 8000.0,
                       "l2": "inputs larger than L2 (index keys %.1f GiB per GPU)" % (kidx_bytes / 2**30),
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": {"bound": "hbm", "kernel": DOMINANT, "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "algorithmic_bytes": kb,
                         "avg_launch_ms": dom_ms},
            "kernel_ms": {k: v / args.steps for k, v in shares.items()},
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "prefill_128k": prefill,
            "configs": configs,
            "decode_step_fused": fused,
            "index_variants": variants,
            "prefill_backward": backward,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_prefill_headline(args):
    """--workload prefill_*: the step is one full prefill (index + sparse
    branch); the value is the sparse branch's useful TFLOP/s."""
    dist, rank, local, world = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    clocks = ClockSampler(dev.index)
    clocks.start()
    r = measure_prefill(args.workload, dev, args.steps, max(args.warmup, 1), args.prefill_len)
    clk = clocks.stop()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.prefill_len is None:
        from synthetic import make_workload
        w = make_workload(args.workload, dev)
        rps, dt, used, n, note, useful = oracle_prefill_sample(w, args.cpu_rows)
        cpu = {"value": useful / dt / 1e12, "unit": "TFLOP/s", "rows_per_s": rps,
               "cores": host_cores(), "threads_used": used, "kind": "oracle", "sample": note,
               "seconds": dt, "sample_rows": n,
               "extrapolated_full_seconds": dt * r["rows"] / n}
        del w
    _, tf_burst, tf_sus, kind = measured_peaks()
    if rank == 0:
        line = {"metric": METRIC, "value": r["sparse_attn_tflops"], "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": r["workload"], "rows": r["rows"], "H_q": r["H_q"],
                           "H_kv": r["H_kv"], "top_k": r["top_k"],
                           "l2": "inputs larger than L2"},
                "roofline": {"bound": "tensor", "kernel": "prefill_attn_kv_outer",
                             "achieved": r["sparse_attn_tflops"], "peak": tf_burst,
                             "peak_kind": kind + " burst", "unit": "TFLOP/s",
                             "frac": r["sparse_attn_tflops"] / tf_burst, "traffic": None},
                "prefill": r, "clocks": clk, "gpu_launches": int(r["gpu_launches_per_step"] * args.steps),
                "e2e": None, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_e2e(w, eng, stream, args, step_bytes, world, dist):
    """Same step through the public API from pinned host buffers, as a decode
    server runs it: per step ONE host->device copy brings the new query (q,
    q_idx) and the new token's k_idx/k/v rows, `msa_kv_append` writes that
    token at position L-1 of every sequence's resident cache, the two calls
    run, and ONE device->host copy returns out + block ids + block scores
    (packed into one device buffer), then the host waits for it."""
    import block_sparse_attention_43_b200 as msa
    B = w.B
    dev = w.q.device
    pos = [int(w.kv_offsets[b]) + w.lens_host[b] - 1 for b in range(B)]
    rows = {n: torch.stack([getattr(w, n)[p] for p in pos]).unsqueeze(1) for n in ("k_idx", "k", "v")}
    parts = [w.q, w.q_idx, rows["k_idx"], rows["k"], rows["v"]]
    h_in = torch.cat([t.reshape(-1).cpu() for t in parts]).pin_memory()
    d_in = torch.empty_like(h_in, device=dev)
    views, o = [], 0
    for t in parts:
        views.append(d_in[o:o + t.numel()].view(t.shape))
        o += t.numel()
    d_q, d_qi, d_kidx, d_k, d_v = views
    lens_prev = (w.lens - 1).contiguous()       # kv_append writes at lens[b] + 0
    # outputs packed into one device buffer: out (bf16) | ids (int32) | scores (fp32)
    n_out = eng.out.numel() * 2
    n_ids = eng.block_ids.numel() * 4
    d_res = torch.empty(n_out + 2 * n_ids, dtype=torch.uint8, device=dev)
    out_v = d_res[:n_out].view(torch.bfloat16).view(eng.out.shape)
    ids_v = d_res[n_out:n_out + n_ids].view(torch.int32).view(eng.block_ids.shape)
    sc_v = d_res[n_out + n_ids:].view(torch.float32).view(eng.block_scores.shape)
    h_res = torch.empty(d_res.shape, dtype=torch.uint8).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    h2d = h_in.numel() * h_in.element_size()
    d2h = h_res.numel()

    def one():
        with torch.cuda.stream(stream):
            d_in.copy_(h_in, non_blocking=True)
            msa.msa_kv_append(eng.shape, d_kidx, d_k, d_v, lens_prev, w.k_idx, w.k, w.v,
                              kv_offsets=w.kv_offsets, device_status=status, stream=stream)
            msa.msa_index_topk(eng.shape, d_qi, w.k_idx, w.lens, w.kv_offsets, ids_v, sc_v,
                               eng.ws_index, stream)
            msa.msa_sparse_attention(eng.shape, d_q, w.k, w.v, ids_v, w.lens, w.kv_offsets,
                                     eng.softmax_scale, out_v, eng.ws_attn, stream)
            h_res.copy_(d_res, non_blocking=True)
        stream.synchronize()

    for _ in range(max(3, args.warmup // 4)):
        one()
    if int(status.item()) != 0 or msa.msa_read_device_status(eng.ws_attn, stream) != 0:
        raise RuntimeError("e2e: device status set")
    n = max(10, args.steps // 4)
    if dist is not None:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(n):
        one()
    rate, dt = whole_job_rate(dist, world, step_bytes, (time.perf_counter() - t0) / n, w.q.device)
    return {"value": rate / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": dt * 1e3, "steps": n,
            "copies_per_step": {"h2d": 1, "d2h": 1}}


if __name__ == "__main__":
    main()
