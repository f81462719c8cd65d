"""Seeded input generator for the five MSA workloads.

Layouts (token-major, head dim innermost):
    q_idx  [B, Sq, H_kv, d_idx] bf16   one index query per GQA group
    k_idx  [T, H_kv, d_idx]     bf16   packed: sequence b owns tokens
                                        kv_offsets[b] .. kv_offsets[b]+lens[b]-1
    q      [B, Sq, H_q, D]      bf16
    k, v   [T, H_kv, D]         bf16   packed like k_idx
    lens   [B] int32, kv_offsets [B] int64

Values are i.i.d. N(0, 1) drawn with torch's counter-based generator on the
target device, rounded to bf16 (round-to-nearest-even).  "Needle" blocks are
planted by overwriting a block's index keys with amp * q_idx/|q_idx| + N(0, 0.1)
(per group), as the decode workloads describe.  Needle positions and ragged
lengths come from a CPU generator so they do not depend on the device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BLOCK = 128
HEAD_DIM = 128
INDEX_DIM = 128

# The five workloads, named by what they are.
WORKLOADS = {
    "prefill_2k": dict(mode="prefill", B=1, n=2048, H_q=8, H_kv=2, top_k=4, seed=0),
    "decode_32k": dict(mode="decode", B=8, L=32768, H_q=64, H_kv=8, top_k=16, seed=1),
    "prefill_128k": dict(mode="prefill", B=1, n=131072, H_q=64, H_kv=8, top_k=16, seed=2),
    "decode_1m": dict(mode="decode", B=4, L=1048576, H_q=64, H_kv=8, top_k=16, seed=3,
                      needles=16, amp=4.0),
    "decode_ragged": dict(mode="decode", B=64, L=(4096, 262144), H_q=64, H_kv=8, top_k=16,
                          seed=4, needles=8, amp=4.0),
}

_CHUNK = 1 << 26  # elements drawn per generator call (fixed so draws are reproducible)


@dataclass
class Workload:
    name: str
    B: int
    Sq: int
    H_q: int
    H_kv: int
    top_k: int
    lens: torch.Tensor          # int32 [B] on device
    kv_offsets: torch.Tensor    # int64 [B] on device
    q_idx: torch.Tensor
    k_idx: torch.Tensor
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    lens_host: list = field(default_factory=list)
    needle_blocks: dict = field(default_factory=dict)   # b -> list of block ids
    block: int = BLOCK
    D: int = HEAD_DIM
    d_idx: int = INDEX_DIM

    @property
    def kv_capacity(self) -> int:
        return int(self.k.shape[0])

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


def _randn_bf16(shape, gen, device, std=1.0):
    """i.i.d. N(0, std^2) rounded to bf16, drawn in fixed-size chunks."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        x = torch.randn(hi - lo, generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[lo:hi].copy_(x)
    return out.view(*shape)


def ragged_lens(B: int, lo: int, hi: int, seed: int) -> list:
    """Log-uniform lengths floor(exp(U[ln lo, ln hi])) from a seeded CPU draw."""
    g = torch.Generator().manual_seed(seed)
    u = torch.rand(B, generator=g, dtype=torch.float64)
    a, b = math.log(lo), math.log(hi)
    return [int(math.floor(math.exp(a + float(x) * (b - a)))) for x in u]


def make_inputs(*, B, Sq, lens, H_q, H_kv, top_k, seed, device, name="custom",
                D=HEAD_DIM, d_idx=INDEX_DIM, block=BLOCK, needles=0, amp=4.0,
                padded_to=None) -> Workload:
    """Draw one workload.  ``lens`` is a list of B context lengths (each >= Sq).
    ``padded_to`` lays sequence b at offset b*padded_to instead of packing."""
    lens = [int(x) for x in lens]
    assert len(lens) == B and all(L >= Sq for L in lens)
    if padded_to is not None:
        assert all(L <= padded_to for L in lens)
        offs = [b * padded_to for b in range(B)]
        T = B * padded_to
    else:
        offs, acc = [], 0
        for L in lens:
            offs.append(acc)
            acc += L
        T = acc
    device = torch.device(device)
    gen = torch.Generator(device=device).manual_seed(int(seed))
    q_idx = _randn_bf16((B, Sq, H_kv, d_idx), gen, device)
    q = _randn_bf16((B, Sq, H_q, D), gen, device)
    k_idx = _randn_bf16((T, H_kv, d_idx), gen, device)
    k = _randn_bf16((T, H_kv, D), gen, device)
    v = _randn_bf16((T, H_kv, D), gen, device)
    needle_blocks = {}
    if needles:
        cpu_gen = torch.Generator().manual_seed(int(seed) * 1000003 + 17)
        for b in range(B):
            own = (lens[b] - 1) // block          # the last query's own block
            n_here = min(needles, own)
            if n_here <= 0:
                continue
            picks = torch.randperm(own, generator=cpu_gen)[:n_here].sort().values.tolist()
            needle_blocks[b] = picks
            qn = q_idx[b, Sq - 1].float()                          # [H_kv, d_idx]
            qn = qn / qn.norm(dim=-1, keepdim=True)
            for j in picks:
                t0 = offs[b] + j * block
                noise = torch.randn(block, H_kv, d_idx, generator=gen, device=device,
                                    dtype=torch.float32) * 0.1
                k_idx[t0:t0 + block].copy_(amp * qn.unsqueeze(0) + noise)
    return Workload(
        name=name, B=B, Sq=Sq, H_q=H_q, H_kv=H_kv, top_k=top_k,
        lens=torch.tensor(lens, dtype=torch.int32, device=device),
        kv_offsets=torch.tensor(offs, dtype=torch.int64, device=device),
        q_idx=q_idx, k_idx=k_idx, q=q, k=k, v=v, lens_host=lens,
        needle_blocks=needle_blocks, block=block, D=D, d_idx=d_idx)


def make_workload(name: str, device) -> Workload:
    """One of the five named workloads at full size."""
    c = WORKLOADS[name]
    if c["mode"] == "prefill":
        B, Sq, lens = c["B"], c["n"], [c["n"]] * c["B"]
    elif isinstance(c["L"], tuple):
        B, Sq = c["B"], 1
        lens = ragged_lens(B, c["L"][0], c["L"][1], c["seed"])
    else:
        B, Sq, lens = c["B"], 1, [c["L"]] * c["B"]
    return make_inputs(B=B, Sq=Sq, lens=lens, H_q=c["H_q"], H_kv=c["H_kv"], top_k=c["top_k"],
                       seed=c["seed"], device=device, name=name,
                       needles=c.get("needles", 0), amp=c.get("amp", 4.0))


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 view of its bits (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def quantize_e4m3_rows(x):
    """FP8 E4M3 codes of x with one fp32 scale per row of the last dim: scale =
    max|x| / 448 (the largest E4M3 magnitude), codes = x / scale rounded by
    torch's E4M3 cast.  Returns (uint8 codes shaped like x, float32 scales
    shaped like x without its last dim).  Input preparation only."""
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (xf / scale.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()
