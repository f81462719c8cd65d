"""Python binding of libmsa.so, the B200 MiniMax Sparse Attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/msa.h.  PyTorch provides device
memory and streams.  There is no CPU fallback: if libmsa.so is missing or
cannot be loaded, importing this package raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmsa.so")

MSA_OK = 0
STATUS_NAMES = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED",
                3: "MSA_ERR_WORKSPACE", 4: "MSA_ERR_CUDA", 5: "MSA_ERR_DEVICE_TIMEOUT",
                6: "MSA_ERR_BAD_LENS", 7: "MSA_ERR_MISALIGNED"}

# Every entry point include/msa.h declares.
EXPORTS = ("msa_index_topk_workspace_size", "msa_index_topk", "msa_index_topk_fp8",
           "msa_sparse_attention_workspace_size", "msa_sparse_attention",
           "msa_index_topk_paged", "msa_sparse_attention_paged", "msa_kv_append",
           "msa_index_topk_static", "msa_sparse_attention_backward_workspace_size",
           "msa_sparse_attention_backward", "msa_decode_step_workspace_size",
           "msa_decode_step", "msa_decode_step_paged", "msa_read_device_status",
           "msa_set_wait_controls", "msa_trace_enable",
           "msa_trace_read",
           "msa_status_string")


class msa_shape_t(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("q_len", ctypes.c_int32),
                ("max_kv_len", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("index_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("kv_capacity", ctypes.c_int64),
                ("num_index_heads", ctypes.c_int32), ("index_key_format", ctypes.c_int32)]


# msa_index_key_format_t
INDEX_KEYS_BF16, INDEX_KEYS_BF16_SHARED, INDEX_KEYS_FP8, INDEX_KEYS_FP8_SHARED = 0, 1, 2, 3


class MSAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python block_sparse_attention_43_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, Z, S = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(msa_shape_t)
    lib.msa_index_topk_workspace_size.argtypes = [S]
    lib.msa_index_topk_workspace_size.restype = Z
    lib.msa_sparse_attention_workspace_size.argtypes = [S]
    lib.msa_sparse_attention_workspace_size.restype = Z
    lib.msa_index_topk.argtypes = [S, P, P, P, P, P, P, P, Z, P]
    lib.msa_index_topk.restype = ctypes.c_int
    lib.msa_index_topk_fp8.argtypes = [S, P, P, P, P, P, P, P, P, Z, P]
    lib.msa_index_topk_fp8.restype = ctypes.c_int
    lib.msa_sparse_attention.argtypes = [S, P, P, P, P, P, P, ctypes.c_float, P, P, Z, P]
    lib.msa_sparse_attention.restype = ctypes.c_int
    I32 = ctypes.c_int32
    lib.msa_index_topk_paged.argtypes = [S, P, P, P, P, I32, P, P, P, Z, P]
    lib.msa_index_topk_paged.restype = ctypes.c_int
    lib.msa_sparse_attention_paged.argtypes = [S, P, P, P, P, P, P, I32, ctypes.c_float, P, P, Z, P]
    lib.msa_sparse_attention_paged.restype = ctypes.c_int
    lib.msa_kv_append.argtypes = [S, I32, P, P, P, P, P, P, I32, P, P, P, P, P]
    lib.msa_kv_append.restype = ctypes.c_int
    lib.msa_index_topk_static.argtypes = [S, P, P, P, P, P, P, P]
    lib.msa_index_topk_static.restype = ctypes.c_int
    lib.msa_sparse_attention_backward_workspace_size.argtypes = [S]
    lib.msa_sparse_attention_backward_workspace_size.restype = Z
    lib.msa_sparse_attention_backward.argtypes = [S, P, P, P, P, P, P, ctypes.c_float, P, P, P, P,
                                                  P, Z, P]
    lib.msa_sparse_attention_backward.restype = ctypes.c_int
    lib.msa_decode_step_workspace_size.argtypes = [S]
    lib.msa_decode_step_workspace_size.restype = Z
    lib.msa_decode_step.argtypes = [S, P, P, P, P, P, P, P, ctypes.c_float, P, P, P, P, Z, P]
    lib.msa_decode_step.restype = ctypes.c_int
    lib.msa_decode_step_paged.argtypes = [S, P, P, P, P, P, P, P, I32, ctypes.c_float, P, P, P, P,
                                          Z, P]
    lib.msa_decode_step_paged.restype = ctypes.c_int
    lib.msa_read_device_status.argtypes = [P, P]
    lib.msa_read_device_status.restype = ctypes.c_int
    lib.msa_set_wait_controls.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
    lib.msa_set_wait_controls.restype = ctypes.c_int
    lib.msa_trace_enable.argtypes = [ctypes.c_int]
    lib.msa_trace_enable.restype = ctypes.c_int
    lib.msa_trace_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float),
                                   ctypes.c_int]
    lib.msa_trace_read.restype = ctypes.c_int
    lib.msa_status_string.argtypes = [ctypes.c_int]
    lib.msa_status_string.restype = ctypes.c_char_p
    return lib


lib = _load()


def make_shape(*, batch, q_len, max_kv_len, num_q_heads, num_kv_heads, top_k, kv_capacity,
               head_dim=128, index_dim=128, block_size=128, num_index_heads=0,
               index_key_format=INDEX_KEYS_BF16) -> msa_shape_t:
    return msa_shape_t(batch, q_len, max_kv_len, num_q_heads, num_kv_heads, head_dim, index_dim,
                       block_size, top_k, kv_capacity, num_index_heads, index_key_format)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code, where):
    if code != MSA_OK:
        raise MSAError(code, where)


def msa_index_topk_workspace_size(shape: msa_shape_t) -> int:
    return lib.msa_index_topk_workspace_size(ctypes.byref(shape))


def msa_sparse_attention_workspace_size(shape: msa_shape_t) -> int:
    return lib.msa_sparse_attention_workspace_size(ctypes.byref(shape))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A caller-owned workspace buffer (256-byte aligned via the caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def msa_index_topk(shape, q_idx, k_idx, lens, kv_offsets, block_ids, block_scores, workspace,
                   stream=None) -> None:
    """Index branch through the C ABI; see include/msa.h for the contract."""
    _check(lib.msa_index_topk(ctypes.byref(shape), _ptr(q_idx), _ptr(k_idx), _ptr(lens),
                              _ptr(kv_offsets), _ptr(block_ids), _ptr(block_scores),
                              _ptr(workspace), workspace.numel(), _stream(stream)),
           "msa_index_topk")


def msa_index_topk_fp8(shape, q_idx, k_idx_fp8, k_idx_scale, lens, kv_offsets, block_ids,
                       block_scores, workspace, stream=None) -> None:
    """Index branch on FP8 E4M3 index keys (uint8 codes) with fp32 per-row
    scales, decode only; see include/msa.h."""
    _check(lib.msa_index_topk_fp8(ctypes.byref(shape), _ptr(q_idx), _ptr(k_idx_fp8),
                                  _ptr(k_idx_scale), _ptr(lens), _ptr(kv_offsets), _ptr(block_ids),
                                  _ptr(block_scores), _ptr(workspace), workspace.numel(),
                                  _stream(stream)),
           "msa_index_topk_fp8")


def msa_sparse_attention(shape, q, k_cache, v_cache, block_ids, lens, kv_offsets, softmax_scale,
                         out, workspace, stream=None) -> None:
    """Sparse branch through the C ABI; see include/msa.h for the contract."""
    _check(lib.msa_sparse_attention(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(block_ids), _ptr(lens), _ptr(kv_offsets),
                                    float(softmax_scale), _ptr(out), _ptr(workspace),
                                    workspace.numel(), _stream(stream)),
           "msa_sparse_attention")


def msa_index_topk_paged(shape, q_idx, k_idx_pool, lens, page_table, block_ids, block_scores,
                         workspace, stream=None) -> None:
    """Index branch on paged caches; page_table is int32 [B, pages_per_seq]."""
    _check(lib.msa_index_topk_paged(ctypes.byref(shape), _ptr(q_idx), _ptr(k_idx_pool), _ptr(lens),
                                    _ptr(page_table), int(page_table.shape[-1]), _ptr(block_ids),
                                    _ptr(block_scores), _ptr(workspace), workspace.numel(),
                                    _stream(stream)),
           "msa_index_topk_paged")


def msa_sparse_attention_paged(shape, q, k_pool, v_pool, block_ids, lens, page_table,
                               softmax_scale, out, workspace, stream=None) -> None:
    """Sparse branch on paged caches; page_table is int32 [B, pages_per_seq]."""
    _check(lib.msa_sparse_attention_paged(ctypes.byref(shape), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                          _ptr(block_ids), _ptr(lens), _ptr(page_table),
                                          int(page_table.shape[-1]), float(softmax_scale),
                                          _ptr(out), _ptr(workspace), workspace.numel(),
                                          _stream(stream)),
           "msa_sparse_attention_paged")


def msa_kv_append(shape, new_k_idx, new_k, new_v, lens, k_idx_cache, k_cache, v_cache, *,
                  kv_offsets=None, page_table=None, device_status=None, stream=None) -> None:
    """Writes [B, n_new, H_kv, 128] new tokens after each sequence's length."""
    pps = int(page_table.shape[-1]) if page_table is not None else 0
    _check(lib.msa_kv_append(ctypes.byref(shape), int(new_k.shape[1]), _ptr(new_k_idx), _ptr(new_k),
                             _ptr(new_v), _ptr(lens), _ptr(kv_offsets), _ptr(page_table), pps,
                             _ptr(k_idx_cache), _ptr(k_cache), _ptr(v_cache), _ptr(device_status),
                             _stream(stream)),
           "msa_kv_append")


def msa_index_topk_static(shape, q_idx, k_idx, lens, kv_offsets, block_ids, block_scores,
                          stream=None) -> None:
    """Index branch with the library's fixed device scratch instead of a
    workspace (for callers that cannot allocate); see include/msa.h."""
    _check(lib.msa_index_topk_static(ctypes.byref(shape), _ptr(q_idx), _ptr(k_idx), _ptr(lens),
                                     _ptr(kv_offsets), _ptr(block_ids), _ptr(block_scores),
                                     _stream(stream)),
           "msa_index_topk_static")


def msa_sparse_attention_backward_workspace_size(shape: msa_shape_t) -> int:
    return lib.msa_sparse_attention_backward_workspace_size(ctypes.byref(shape))


def msa_sparse_attention_backward(shape, q, k_cache, v_cache, block_ids, lens, kv_offsets,
                                  softmax_scale, d_out, dq, dk, dv, workspace, stream=None) -> None:
    """Backward of the sparse branch: writes dq (bf16), adds into dk and dv
    (float32, [kv_capacity, H_kv, 128]); see include/msa.h."""
    _check(lib.msa_sparse_attention_backward(ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                             _ptr(v_cache), _ptr(block_ids), _ptr(lens),
                                             _ptr(kv_offsets), float(softmax_scale), _ptr(d_out),
                                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                             workspace.numel(), _stream(stream)),
           "msa_sparse_attention_backward")


def msa_decode_step_workspace_size(shape: msa_shape_t) -> int:
    return lib.msa_decode_step_workspace_size(ctypes.byref(shape))


def msa_decode_step(shape, q_idx, k_idx, q, k_cache, v_cache, lens, kv_offsets, softmax_scale,
                    block_ids, block_scores, out, workspace, stream=None) -> None:
    """Index branch, top-k and sparse branch of a decode step in one launch;
    see include/msa.h."""
    _check(lib.msa_decode_step(ctypes.byref(shape), _ptr(q_idx), _ptr(k_idx), _ptr(q),
                               _ptr(k_cache), _ptr(v_cache), _ptr(lens), _ptr(kv_offsets),
                               float(softmax_scale), _ptr(block_ids), _ptr(block_scores),
                               _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "msa_decode_step")


def msa_decode_step_paged(shape, q_idx, k_idx_pool, q, k_pool, v_pool, lens, page_table,
                          softmax_scale, block_ids, block_scores, out, workspace,
                          stream=None) -> None:
    """msa_decode_step on paged caches (page_table [B, pages_per_seq])."""
    pps = int(page_table.shape[-1])
    _check(lib.msa_decode_step_paged(ctypes.byref(shape), _ptr(q_idx), _ptr(k_idx_pool), _ptr(q),
                                     _ptr(k_pool), _ptr(v_pool), _ptr(lens), _ptr(page_table), pps,
                                     float(softmax_scale), _ptr(block_ids), _ptr(block_scores),
                                     _ptr(out), _ptr(workspace), workspace.numel(),
                                     _stream(stream)),
           "msa_decode_step_paged")


def msa_read_device_status(workspace, stream=None) -> int:
    return lib.msa_read_device_status(_ptr(workspace), _stream(stream))


# msa_stall_t bits
STALL_NONE, STALL_INDEX_DECODE, STALL_DECODE_STEP = 0, 1, 2


def msa_set_wait_controls(wait_limit_ns: int = 0, stall_mask: int = STALL_NONE) -> None:
    """Testing aid: the bounded device waits' limit (0 = default) and the
    kernels that wait once on something that never happens."""
    _check(lib.msa_set_wait_controls(int(wait_limit_ns), int(stall_mask)), "msa_set_wait_controls")


def msa_trace_enable(on: bool) -> None:
    _check(lib.msa_trace_enable(1 if on else 0), "msa_trace_enable")


def msa_trace_read(max_entries: int = 4096):
    """[(kernel name, milliseconds)] recorded since the last read, in launch order."""
    names = (ctypes.c_char_p * max_entries)()
    ms = (ctypes.c_float * max_entries)()
    n = lib.msa_trace_read(names, ms, max_entries)
    if n < 0:
        raise MSAError(4, "msa_trace_read")
    return [(names[i].decode(), float(ms[i])) for i in range(n)]


def msa_status_string(code: int) -> str:
    return lib.msa_status_string(int(code)).decode()


class MSA:
    """Convenience wrapper owning output and workspace buffers for one shape.
    Holds torch tensors only; every call goes straight to the C ABI."""

    def __init__(self, *, batch, q_len, max_kv_len, num_q_heads, num_kv_heads, top_k,
                 kv_capacity, device="cuda", num_index_heads=0, index_key_format=INDEX_KEYS_BF16):
        self.shape = make_shape(batch=batch, q_len=q_len, max_kv_len=max_kv_len,
                                num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, top_k=top_k,
                                kv_capacity=kv_capacity, num_index_heads=num_index_heads,
                                index_key_format=index_key_format)
        n_idx = msa_index_topk_workspace_size(self.shape)
        n_att = msa_sparse_attention_workspace_size(self.shape)
        if n_idx == 0 or n_att == 0:
            raise MSAError(2, "shape rejected")
        self.device = torch.device(device)
        self.ws_index = alloc_workspace(n_idx, self.device)
        self.ws_attn = alloc_workspace(n_att, self.device)
        sel = (batch, q_len, num_index_heads or num_kv_heads, top_k)
        self.block_ids = torch.empty(sel, dtype=torch.int32, device=self.device)
        self.block_scores = torch.empty(sel, dtype=torch.float32, device=self.device)
        self.out = torch.empty((batch, q_len, num_q_heads, 128), dtype=torch.bfloat16,
                               device=self.device)
        self.softmax_scale = 1.0 / math.sqrt(128)

    def index_topk(self, q_idx, k_idx, lens, kv_offsets, stream=None, k_idx_scale=None):
        """k_idx_scale given: FP8 index keys (msa_index_topk_fp8)."""
        if k_idx_scale is not None:
            msa_index_topk_fp8(self.shape, q_idx, k_idx, k_idx_scale, lens, kv_offsets,
                               self.block_ids, self.block_scores, self.ws_index, stream)
        else:
            msa_index_topk(self.shape, q_idx, k_idx, lens, kv_offsets, self.block_ids,
                           self.block_scores, self.ws_index, stream)
        return self.block_ids, self.block_scores

    def sparse_attention(self, q, k_cache, v_cache, lens, kv_offsets, block_ids=None, stream=None):
        msa_sparse_attention(self.shape, q, k_cache, v_cache,
                             self.block_ids if block_ids is None else block_ids, lens, kv_offsets,
                             self.softmax_scale, self.out, self.ws_attn, stream)
        return self.out

    def forward(self, q_idx, k_idx, q, k_cache, v_cache, lens, kv_offsets, stream=None):
        self.index_topk(q_idx, k_idx, lens, kv_offsets, stream)
        return self.sparse_attention(q, k_cache, v_cache, lens, kv_offsets, stream=stream)

    def decode_step(self, q_idx, k_idx, q, k_cache, v_cache, lens, kv_offsets, stream=None):
        """The fused single-launch decode step (q_len 1); same results as
        forward().  Its workspace is allocated on first use."""
        if getattr(self, "ws_step", None) is None:
            n = msa_decode_step_workspace_size(self.shape)
            if n == 0:
                raise MSAError(2, "shape rejected by msa_decode_step")
            self.ws_step = alloc_workspace(n, self.device)
        msa_decode_step(self.shape, q_idx, k_idx, q, k_cache, v_cache, lens, kv_offsets,
                        self.softmax_scale, self.block_ids, self.block_scores, self.out,
                        self.ws_step, stream)
        return self.out

    def device_status(self, stream=None) -> int:
        a = msa_read_device_status(self.ws_index, stream)
        b = msa_read_device_status(self.ws_attn, stream)
        return a if a != MSA_OK else b
