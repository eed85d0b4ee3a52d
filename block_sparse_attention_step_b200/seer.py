"""ctypes binding of ``libseer.so`` (the C ABI in ``include/seer.h``).

Argument marshalling only: every function takes torch tensors (device memory
for the device arguments), checks dtype and contiguity, passes raw pointers
and the current CUDA stream, and raises ``SeerError`` on a non-zero status.
All computation happens in the library's kernels.  The library must have been
built (``python -m block_sparse_attention_step_b200.build``); there is no
fallback path, a missing library raises at first use.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libseer.so")

SEER_OK = 0
SEER_ERR_CUDA = 3
STATUS_NAMES = {0: "SEER_OK", 1: "SEER_ERR_INVALID_ARG", 2: "SEER_ERR_UNSUPPORTED",
                3: "SEER_ERR_CUDA", 4: "SEER_ERR_WORKSPACE"}
DEV_NONFINITE_SCORE = 1
DEV_BAD_INDEX = 2
DEV_BAD_PAGE = 4
DEV_K_CLAMPED = 8
DEV_TIMEOUT = 16

EXPORTS = (
    "seer_version", "seer_status_string", "seer_last_cuda_error", "seer_dims_default",
    "seer_k_from_sparsity",
    "seer_k_from_budget", "seer_fill_k", "seer_default_splits", "seer_step_workspace_bytes",
    "seer_pool_keys", "seer_gate_scores", "seer_block_select", "seer_block_select_unified",
    "seer_sparse_decode",
    "seer_combine", "seer_decode_step", "seer_decode_step_host", "seer_host_ptr_mapped",
    "seer_decode_step_noalloc",
    "seer_decode_step_fused", "seer_step_workspace_init",
    "seer_prefill_k_max", "seer_prefill_workspace_bytes", "seer_prefill",
    "seer_prefill_attention",
    "seer_block_lse_elems", "seer_sparse_decode_mass", "seer_block_mass",
)
NOALLOC_SCRATCH_BYTES = 16 << 20


class SeerError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = _lib().seer_status_string(status).decode()
        if status == SEER_ERR_CUDA:
            detail += ": " + _lib().seer_last_cuda_error().decode()
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)} ({detail})")


class seer_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("num_pages", ctypes.c_int64), ("stride_page", ctypes.c_int64),
                ("stride_token", ctypes.c_int64), ("stride_head", ctypes.c_int64)]


class seer_step_args(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seqlens", ctypes.c_void_p),
                ("w_gate", ctypes.c_void_p), ("kbar", ctypes.c_void_p),
                ("k_per_seq", ctypes.c_void_p), ("update_kbar", ctypes.c_int32),
                ("force_newest", ctypes.c_int32), ("k_max", ctypes.c_int32),
                ("num_splits", ctypes.c_int32), ("gate_scale", ctypes.c_float),
                ("softmax_scale", ctypes.c_float), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("out", ctypes.c_void_p),
                ("lse_out", ctypes.c_void_p), ("dev_status", ctypes.c_void_p),
                ("block_lse", ctypes.c_void_p), ("block_mass", ctypes.c_void_p),
                ("unified_heads", ctypes.c_int32), ("k_new", ctypes.c_void_p),
                ("v_new", ctypes.c_void_p)]


class seer_prefill_args(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seqlens", ctypes.c_void_p),
                ("w_gate", ctypes.c_void_p), ("kbar", ctypes.c_void_p),
                ("pool_keys", ctypes.c_int32), ("sparsity_permille", ctypes.c_int32),
                ("budget_tokens", ctypes.c_int32), ("k_max", ctypes.c_int32),
                ("gate_scale", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("out", ctypes.c_void_p), ("lse_out", ctypes.c_void_p),
                ("scores_out", ctypes.c_void_p), ("dev_status", ctypes.c_void_p)]


_P = ctypes.c_void_p
_D = ctypes.POINTER(seer_dims)
_I = ctypes.c_int32
_SIGS = {
    "seer_version": (_I, []),
    "seer_status_string": (ctypes.c_char_p, [_I]),
    "seer_last_cuda_error": (ctypes.c_char_p, []),
    "seer_dims_default": (_I, [_I, _I, _I, _I, _I, _I, ctypes.c_int64, _D]),
    "seer_k_from_sparsity": (_I, [_I, _I, ctypes.POINTER(_I)]),
    "seer_k_from_budget": (_I, [_I, _I, _I, ctypes.POINTER(_I)]),
    "seer_fill_k": (_I, [_D, _P, _I, _I, _P, _P]),
    "seer_default_splits": (_I, [_D, _I, _I]),
    "seer_step_workspace_bytes": (ctypes.c_size_t, [_D, _I, _I]),
    "seer_pool_keys": (_I, [_D, _P, _P, _P, _I, _P, _P, _P]),
    "seer_gate_scores": (_I, [_D, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P]),
    "seer_block_select": (_I, [_D, _P, _P, _P, _I, _I, _P, _P, _P, _P]),
    "seer_block_select_unified": (_I, [_D, _P, _P, _P, _I, _I, _P, _P, _P, _P]),
    "seer_sparse_decode": (_I, [_D, _P, _P, _P, _P, _P, _P, _P, _I, _I, ctypes.c_float, _P, _P,
                                _P, _P, _P]),
    "seer_combine": (_I, [_D, _P, _P, _I, _P, _P, _P]),
    "seer_decode_step": (_I, [_D, ctypes.POINTER(seer_step_args), _P]),
    "seer_decode_step_host": (_I, [_D, ctypes.POINTER(seer_step_args), _P, _P, _P, _P]),
    "seer_host_ptr_mapped": (_I, [_P]),
    "seer_decode_step_noalloc": (_I, [_D, ctypes.POINTER(seer_step_args), _P]),
    "seer_decode_step_fused": (_I, [_D, ctypes.POINTER(seer_step_args), _P]),
    "seer_step_workspace_init": (_I, [_D, _I, _I, _P, ctypes.c_size_t, _P]),
    "seer_prefill_k_max": (_I, [_D, _I, _I]),
    "seer_prefill_workspace_bytes": (ctypes.c_size_t, [_D, _I]),
    "seer_prefill": (_I, [_D, ctypes.POINTER(seer_prefill_args), _P]),
    "seer_prefill_attention": (_I, [_D, ctypes.POINTER(seer_prefill_args), _P, _P, _P]),
    "seer_block_lse_elems": (ctypes.c_size_t, [_D]),
    "seer_sparse_decode_mass": (_I, [_D, _P, _P, _P, _P, _P, _P, _P, _I, _I, ctypes.c_float, _P, _P,
                                     _P, _P, _P, _P]),
    "seer_block_mass": (_I, [_D, _P, _P, _I, _P, _P, _P, _P, _P]),
}

_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_sparse_attention_step_b200.build` (no fallback exists)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib_handle = lib
    return _lib_handle


def library():
    """The loaded ctypes library (loads it on first call)."""
    return _lib()


def _check(fn: str, status: int):
    if status != SEER_OK:
        raise SeerError(fn, status)


def _ptr(t, dtype=None, name="tensor", allow_none=False, device=True):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_dims(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks, num_pages,
              stride_page=None, stride_token=None, stride_head=None) -> seer_dims:
    d = seer_dims()
    _check("seer_dims_default", _lib().seer_dims_default(batch, num_q_heads, num_kv_heads, head_dim,
                                                         block_size, max_blocks, num_pages,
                                                         ctypes.byref(d)))
    if stride_page is not None:
        d.stride_page, d.stride_token, d.stride_head = stride_page, stride_token, stride_head
    return d


def version() -> int:
    return _lib().seer_version()


def seer_k_from_sparsity(nb: int, sparsity_permille: int) -> int:
    k = ctypes.c_int32()
    _check("seer_k_from_sparsity", _lib().seer_k_from_sparsity(nb, sparsity_permille, ctypes.byref(k)))
    return k.value


def seer_k_from_budget(nb: int, budget_tokens: int, block_size: int) -> int:
    k = ctypes.c_int32()
    _check("seer_k_from_budget", _lib().seer_k_from_budget(nb, budget_tokens, block_size, ctypes.byref(k)))
    return k.value


def seer_fill_k(d, seqlens, sparsity_permille, budget_tokens, k_per_seq, stream=None):
    _check("seer_fill_k", _lib().seer_fill_k(ctypes.byref(d), _ptr(seqlens, torch.int32, "seqlens"),
                                             sparsity_permille, budget_tokens,
                                             _ptr(k_per_seq, torch.int32, "k_per_seq"), _stream(stream)))


def seer_default_splits(d, k_max: int, num_sms: int = 0) -> int:
    return _lib().seer_default_splits(ctypes.byref(d), k_max, num_sms)


def seer_step_workspace_bytes(d, k_max: int, num_splits: int) -> int:
    return _lib().seer_step_workspace_bytes(ctypes.byref(d), k_max, num_splits)


def seer_pool_keys(d, k_pool, page_table, seqlens, incremental, kbar, dev_status=None, stream=None):
    _check("seer_pool_keys", _lib().seer_pool_keys(
        ctypes.byref(d), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(page_table, torch.int32, "page_table", allow_none=True),
        _ptr(seqlens, torch.int32, "seqlens"), int(incremental), _ptr(kbar, torch.float32, "kbar"),
        _ptr(dev_status, torch.int32, "dev_status", allow_none=True), _stream(stream)))


def seer_gate_scores(d, q, w_gate, kbar, seqlens, gate_scale, scores, dev_status=None, stream=None):
    _check("seer_gate_scores", _lib().seer_gate_scores(
        ctypes.byref(d), _ptr(q, torch.bfloat16, "q"), _ptr(w_gate, torch.float32, "w_gate"),
        _ptr(kbar, torch.float32, "kbar"), _ptr(seqlens, torch.int32, "seqlens"), float(gate_scale),
        _ptr(scores, torch.float32, "scores"),
        _ptr(dev_status, torch.int32, "dev_status", allow_none=True), _stream(stream)))


def seer_block_select(d, scores, seqlens, k_per_seq, force_newest, k_max, idx, n_sel,
                      dev_status=None, stream=None):
    _check("seer_block_select", _lib().seer_block_select(
        ctypes.byref(d), _ptr(scores, torch.float32, "scores"), _ptr(seqlens, torch.int32, "seqlens"),
        _ptr(k_per_seq, torch.int32, "k_per_seq"), int(bool(force_newest)), int(k_max),
        _ptr(idx, torch.int32, "idx"), _ptr(n_sel, torch.int32, "n_sel"),
        _ptr(dev_status, torch.int32, "dev_status", allow_none=True), _stream(stream)))


def seer_block_select_unified(d, scores, seqlens, k_per_seq, force_newest, k_max, idx, n_sel,
                      dev_status=None, stream=None):
    _check("seer_block_select_unified", _lib().seer_block_select_unified(
        ctypes.byref(d), _ptr(scores, torch.float32, "scores"), _ptr(seqlens, torch.int32, "seqlens"),
        _ptr(k_per_seq, torch.int32, "k_per_seq"), int(bool(force_newest)), int(k_max),
        _ptr(idx, torch.int32, "idx"), _ptr(n_sel, torch.int32, "n_sel"),
        _ptr(dev_status, torch.int32, "dev_status", allow_none=True), _stream(stream)))


def seer_sparse_decode(d, q, k_pool, v_pool, page_table, seqlens, idx, n_sel, k_max, num_splits,
                       softmax_scale, o_part, lse_part, dev_status=None, stream=None, *,
                       work_counter=None):
    """work_counter: None (round-robin items) or 2 zeroed int32 words on the device."""
    _check("seer_sparse_decode", _lib().seer_sparse_decode(
        ctypes.byref(d), _ptr(q, torch.bfloat16, "q"), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(v_pool, torch.bfloat16, "v_pool"),
        _ptr(page_table, torch.int32, "page_table", allow_none=True),
        _ptr(seqlens, torch.int32, "seqlens"), _ptr(idx, torch.int32, "idx"),
        _ptr(n_sel, torch.int32, "n_sel"), int(k_max), int(num_splits), float(softmax_scale),
        _ptr(o_part, torch.float32, "o_part"), _ptr(lse_part, torch.float32, "lse_part"),
        _ptr(work_counter, torch.int32, "work_counter", allow_none=True),
        _ptr(dev_status, torch.int32, "dev_status", allow_none=True), _stream(stream)))


def seer_combine(d, o_part, lse_part, num_splits, out, lse_out=None, stream=None):
    _check("seer_combine", _lib().seer_combine(
        ctypes.byref(d), _ptr(o_part, torch.float32, "o_part"),
        _ptr(lse_part, torch.float32, "lse_part"), int(num_splits),
        _ptr(out, torch.bfloat16, "out"), _ptr(lse_out, torch.float32, "lse_out", allow_none=True),
        _stream(stream)))


def step_args(q, k_pool, v_pool, page_table, seqlens, w_gate, kbar, k_per_seq, *, update_kbar,
              force_newest, k_max, num_splits, gate_scale, softmax_scale, workspace, out,
              lse_out=None, dev_status=None, block_lse=None, block_mass=None,
              unified_heads=False, k_new=None, v_new=None) -> seer_step_args:
    a = seer_step_args()
    a.q = _ptr(q, torch.bfloat16, "q", allow_none=True)
    a.k_pool = _ptr(k_pool, torch.bfloat16, "k_pool")
    a.v_pool = _ptr(v_pool, torch.bfloat16, "v_pool")
    a.page_table = _ptr(page_table, torch.int32, "page_table", allow_none=True)
    a.seqlens = _ptr(seqlens, torch.int32, "seqlens")
    a.w_gate = _ptr(w_gate, torch.float32, "w_gate")
    a.kbar = _ptr(kbar, torch.float32, "kbar")
    a.k_per_seq = _ptr(k_per_seq, torch.int32, "k_per_seq")
    a.update_kbar = int(update_kbar)
    a.force_newest = int(bool(force_newest))
    a.k_max = int(k_max)
    a.num_splits = int(num_splits)
    a.gate_scale = float(gate_scale)
    a.softmax_scale = float(softmax_scale)
    a.workspace = _ptr(workspace, torch.uint8, "workspace")
    a.workspace_bytes = workspace.numel()
    a.out = _ptr(out, torch.bfloat16, "out")
    a.lse_out = _ptr(lse_out, torch.float32, "lse_out", allow_none=True)
    a.dev_status = _ptr(dev_status, torch.int32, "dev_status", allow_none=True)
    a.block_lse = _ptr(block_lse, torch.float32, "block_lse", allow_none=True)
    a.block_mass = _ptr(block_mass, torch.float32, "block_mass", allow_none=True)
    a.unified_heads = int(bool(unified_heads))
    a.k_new = _ptr(k_new, torch.bfloat16, "k_new", allow_none=True)
    a.v_new = _ptr(v_new, torch.bfloat16, "v_new", allow_none=True)
    return a


def seer_decode_step(d, args: seer_step_args, stream=None):
    _check("seer_decode_step", _lib().seer_decode_step(ctypes.byref(d), ctypes.byref(args),
                                                       _stream(stream)))


def seer_decode_step_fused(d, args: seer_step_args, stream=None):
    _check("seer_decode_step_fused", _lib().seer_decode_step_fused(ctypes.byref(d),
                                                                   ctypes.byref(args),
                                                                   _stream(stream)))


def seer_step_workspace_init(d, k_max, num_splits, workspace, stream=None):
    _check("seer_step_workspace_init", _lib().seer_step_workspace_init(
        ctypes.byref(d), int(k_max), int(num_splits), _ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)))


def seer_decode_step_host(d, args: seer_step_args, q_host, q_dev, out_host, stream=None):
    _check("seer_decode_step_host", _lib().seer_decode_step_host(
        ctypes.byref(d), ctypes.byref(args), _ptr(q_host, torch.bfloat16, "q_host", device=False),
        _ptr(q_dev, torch.bfloat16, "q_dev"), _ptr(out_host, torch.bfloat16, "out_host", device=False),
        _stream(stream)))


def seer_host_ptr_mapped(t) -> bool:
    """True if seer_decode_step_host accesses this host tensor directly from
    its kernels (pinned and mapped into the device), False if it copies."""
    if t.is_cuda:
        raise ValueError("expected a host tensor")
    return bool(_lib().seer_host_ptr_mapped(ctypes.c_void_p(t.data_ptr())))


def seer_decode_step_noalloc(d, args: seer_step_args, stream=None):
    """The step with the library's own fixed 16 MiB device scratch instead of
    ``args.workspace`` (for callers that cannot allocate device memory)."""
    _check("seer_decode_step_noalloc", _lib().seer_decode_step_noalloc(
        ctypes.byref(d), ctypes.byref(args), _stream(stream)))


def seer_block_lse_elems(d) -> int:
    return _lib().seer_block_lse_elems(ctypes.byref(d))


def seer_sparse_decode_mass(d, q, k_pool, v_pool, page_table, seqlens, idx, n_sel, k_max,
                            num_splits, softmax_scale, o_part, lse_part, block_lse,
                            dev_status=None, stream=None, *, work_counter=None):
    _check("seer_sparse_decode_mass", _lib().seer_sparse_decode_mass(
        ctypes.byref(d), _ptr(q, torch.bfloat16, "q"), _ptr(k_pool, torch.bfloat16, "k_pool"),
        _ptr(v_pool, torch.bfloat16, "v_pool"),
        _ptr(page_table, torch.int32, "page_table", allow_none=True),
        _ptr(seqlens, torch.int32, "seqlens"), _ptr(idx, torch.int32, "idx"),
        _ptr(n_sel, torch.int32, "n_sel"), int(k_max), int(num_splits), float(softmax_scale),
        _ptr(o_part, torch.float32, "o_part"), _ptr(lse_part, torch.float32, "lse_part"),
        _ptr(block_lse, torch.float32, "block_lse"),
        _ptr(work_counter, torch.int32, "work_counter", allow_none=True),
        _ptr(dev_status, torch.int32, "dev_status", allow_none=True), _stream(stream)))


def seer_block_mass(d, idx, n_sel, k_max, seqlens, block_lse, lse, mass, stream=None):
    _check("seer_block_mass", _lib().seer_block_mass(
        ctypes.byref(d), _ptr(idx, torch.int32, "idx"), _ptr(n_sel, torch.int32, "n_sel"),
        int(k_max), _ptr(seqlens, torch.int32, "seqlens"),
        _ptr(block_lse, torch.float32, "block_lse"), _ptr(lse, torch.float32, "lse"),
        _ptr(mass, torch.float32, "mass"), _stream(stream)))


def seer_prefill_k_max(d, sparsity_permille, budget_tokens):
    return _lib().seer_prefill_k_max(ctypes.byref(d), int(sparsity_permille), int(budget_tokens))


def seer_prefill_workspace_bytes(d, k_max):
    return _lib().seer_prefill_workspace_bytes(ctypes.byref(d), int(k_max))


def seer_prefill_attention(d, q, k_pool, v_pool, page_table, seqlens, idx, n_sel, *, k_max,
                           softmax_scale, out, lse_out=None, dev_status=None, stream=None):
    a = seer_prefill_args()
    a.q = _ptr(q, torch.bfloat16, "q")
    a.k_pool = _ptr(k_pool, torch.bfloat16, "k_pool")
    a.v_pool = _ptr(v_pool, torch.bfloat16, "v_pool")
    a.page_table = _ptr(page_table, torch.int32, "page_table", allow_none=True)
    a.seqlens = _ptr(seqlens, torch.int32, "seqlens")
    a.k_max = int(k_max)
    a.softmax_scale = float(softmax_scale)
    a.out = _ptr(out, torch.bfloat16, "out")
    a.lse_out = _ptr(lse_out, torch.float32, "lse_out", allow_none=True)
    a.dev_status = _ptr(dev_status, torch.int32, "dev_status", allow_none=True)
    _check("seer_prefill_attention", _lib().seer_prefill_attention(
        ctypes.byref(d), ctypes.byref(a), _ptr(idx, torch.int32, "idx"),
        _ptr(n_sel, torch.int32, "n_sel"), _stream(stream)))


def seer_prefill(d, q, k_pool, v_pool, page_table, seqlens, w_gate, kbar, *, pool_keys,
                 sparsity_permille, budget_tokens, k_max, gate_scale, softmax_scale, workspace,
                 out, lse_out=None, scores_out=None, dev_status=None, stream=None):
    a = seer_prefill_args()
    a.q = _ptr(q, torch.bfloat16, "q")
    a.k_pool = _ptr(k_pool, torch.bfloat16, "k_pool")
    a.v_pool = _ptr(v_pool, torch.bfloat16, "v_pool")
    a.page_table = _ptr(page_table, torch.int32, "page_table", allow_none=True)
    a.seqlens = _ptr(seqlens, torch.int32, "seqlens")
    a.w_gate = _ptr(w_gate, torch.float32, "w_gate")
    a.kbar = _ptr(kbar, torch.float32, "kbar")
    a.pool_keys = int(bool(pool_keys))
    a.sparsity_permille = int(sparsity_permille)
    a.budget_tokens = int(budget_tokens)
    a.k_max = int(k_max)
    a.gate_scale = float(gate_scale)
    a.softmax_scale = float(softmax_scale)
    a.workspace = _ptr(workspace, torch.uint8, "workspace")
    a.workspace_bytes = workspace.numel()
    a.out = _ptr(out, torch.bfloat16, "out")
    a.lse_out = _ptr(lse_out, torch.float32, "lse_out", allow_none=True)
    a.scores_out = _ptr(scores_out, torch.float32, "scores_out", allow_none=True)
    a.dev_status = _ptr(dev_status, torch.int32, "dev_status", allow_none=True)
    _check("seer_prefill", _lib().seer_prefill(ctypes.byref(d), ctypes.byref(a), _stream(stream)))

