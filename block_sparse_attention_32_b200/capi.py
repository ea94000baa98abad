"""Thin ctypes binding of ``libmsa.so`` -- argument marshalling only.

Each function has the name of the C entry point it calls (``include/msa.h``)
and takes torch CUDA tensors; it passes raw device pointers, element strides
and the current CUDA stream, raises ``MSAError`` on a non-OK status, and does
no arithmetic of its own.  If the library is missing this module raises on
first use: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libmsa.so")

BLOCK = 128
TOPK = 16
HEAD_DIM = 128

STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED",
          3: "MSA_ERR_ALIGNMENT", 4: "MSA_ERR_WORKSPACE_TOO_SMALL", 5: "MSA_ERR_CUDA",
          6: "MSA_ERR_SCRATCH_LIMIT"}
DEVERR = {1: "MSA_DEVERR_TIMEOUT", 2: "MSA_DEVERR_BAD_BLOCK", 3: "MSA_DEVERR_BAD_ENTRY"}


class MSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("n_q", ctypes.c_int64), ("n_kv", ctypes.c_int64),
                ("q_pos0", ctypes.c_int64), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32),
                ("h_kidx", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("scale", ctypes.c_float),
                ("q_window", ctypes.c_int32)]


class Tensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("s_batch", ctypes.c_int64), ("s_tok", ctypes.c_int64),
                ("s_head", ctypes.c_int64)]


_lib = None
_lock = threading.Lock()
_P = ctypes.c_void_p
_PD = ctypes.POINTER(Dims)


def load_library(path: str) -> ctypes.CDLL:
    """Load a build of the library from `path` with every signature declared."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with "
            "`python -m block_sparse_attention_32_b200.build` (no CPU fallback exists)")
    L = ctypes.CDLL(path)
    L.msa_num_blocks.argtypes = [_PD]
    L.msa_num_blocks.restype = ctypes.c_int64
    L.msa_num_entries.argtypes = [_PD]
    L.msa_num_entries.restype = ctypes.c_int64
    L.msa_query_window.argtypes = [_PD]
    L.msa_query_window.restype = ctypes.c_int64
    L.msa_num_segments.argtypes = [_PD]
    L.msa_num_segments.restype = ctypes.c_int64
    L.msa_index_score_maxpool.argtypes = [_PD, Tensor, Tensor, _P, ctypes.c_int64, _P, _P]
    L.msa_topk_blocks.argtypes = [_PD, _P, ctypes.c_int64, _P, _P, _P]
    L.msa_block_query_lists_workspace.argtypes = [_PD]
    L.msa_block_query_lists_workspace.restype = ctypes.c_size_t
    L.msa_build_block_query_lists.argtypes = [_PD, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]
    L.msa_build_block_query_lists_noalloc.argtypes = [_PD, _P, _P, _P, _P, _P, _P]
    L.msa_sparse_attn_fwd.argtypes = [_PD, Tensor, Tensor, Tensor, _P, _P, _P, _P, _P, _P]
    L.msa_merge_partials.argtypes = [_PD, _P, _P, _P, _P, _P, _P, _P]
    L.msa_sparse_attn_fwd_compact.argtypes = [_PD, Tensor, Tensor, Tensor, _P, _P, _P, _P, _P,
                                              _P]
    L.msa_merge_partials_compact.argtypes = [_PD, _P, _P, _P, _P, _P, _P, _P]
    L.msa_quantize_e4m3.argtypes = [_P, ctypes.c_int64, _P, _P, _P]
    L.msa_index_score_maxpool_e4m3.argtypes = [_PD, Tensor, Tensor, _P, _P, _P, ctypes.c_int64,
                                               _P, _P]
    L.msa_selection_recall_workspace.argtypes = [_PD, ctypes.c_int64]
    L.msa_selection_recall_workspace.restype = ctypes.c_size_t
    L.msa_selection_recall.argtypes = [_PD, Tensor, Tensor, Tensor, Tensor, _P, _P, ctypes.c_int64,
                                       _P, ctypes.c_int64, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                       _P, _P]
    L.msa_sparse_attn_bwd.argtypes = [_PD, Tensor, Tensor, Tensor, Tensor, Tensor, _P, _P, _P,
                                      _P, _P, _P, _P, _P, _P, _P]
    L.msa_token_select_workspace.argtypes = [_PD, ctypes.c_int64]
    L.msa_token_select_workspace.restype = ctypes.c_size_t
    L.msa_token_select_attention.argtypes = [_PD, Tensor, Tensor, Tensor, Tensor, Tensor, _P,
                                             ctypes.c_int64, ctypes.c_int64, _P, _P, _P, _P,
                                             ctypes.c_size_t, _P, _P]
    L.msa_debug_set_attn_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.msa_debug_set_attn_wait_limit_ns.restype = ctypes.c_uint64
    L.msa_status_string.argtypes = [ctypes.c_int]
    L.msa_status_string.restype = ctypes.c_char_p
    for f in (L.msa_index_score_maxpool, L.msa_topk_blocks, L.msa_build_block_query_lists,
              L.msa_build_block_query_lists_noalloc, L.msa_sparse_attn_fwd, L.msa_merge_partials,
              L.msa_sparse_attn_fwd_compact, L.msa_merge_partials_compact,
              L.msa_selection_recall, L.msa_quantize_e4m3, L.msa_index_score_maxpool_e4m3,
              L.msa_token_select_attention, L.msa_sparse_attn_bwd):
        f.restype = ctypes.c_int
    return L


def lib() -> ctypes.CDLL:
    """Load libmsa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(LIB_PATH)
    return _lib


def make_dims(batch, n_q, n_kv, q_pos0, h_q, h_kv, d_idx, h_kidx=1, scale=None,
              q_window=0) -> Dims:
    if scale is None:
        scale = HEAD_DIM ** -0.5
    return Dims(batch, n_q, n_kv, q_pos0, h_q, h_kv, h_kidx, d_idx, scale, q_window)


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def tensor_btd(t: torch.Tensor) -> Tensor:
    """[B, T, H, D] layout (q, q_idx)."""
    assert t.dim() == 4 and t.stride(3) == 1 and t.dtype == torch.bfloat16 and t.is_cuda
    return Tensor(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


def tensor_bhtd(t: torch.Tensor) -> Tensor:
    """[B, H, T, D] layout (k, v, k_idx)."""
    assert t.dim() == 4 and t.stride(3) == 1 and t.dtype == torch.bfloat16 and t.is_cuda
    return Tensor(t.data_ptr(), t.stride(0), t.stride(2), t.stride(1))


def _check(fn, status):
    if status != 0:
        raise MSAError(fn, status)


def msa_num_blocks(d: Dims) -> int:
    return lib().msa_num_blocks(ctypes.byref(d))


def msa_num_entries(d: Dims) -> int:
    return lib().msa_num_entries(ctypes.byref(d))


def msa_query_window(d: Dims) -> int:
    return lib().msa_query_window(ctypes.byref(d))


def msa_num_segments(d: Dims) -> int:
    return lib().msa_num_segments(ctypes.byref(d))


def msa_debug_set_attn_wait_limit_ns(ns: int) -> int:
    """Time limit (ns) of the attention kernel's barrier waits for later calls;
    returns the previous one (0 restores the default 2 s)."""
    return int(lib().msa_debug_set_attn_wait_limit_ns(ns))


def msa_block_query_lists_workspace(d: Dims) -> int:
    return lib().msa_block_query_lists_workspace(ctypes.byref(d))


def msa_index_score_maxpool(d: Dims, q_idx, k_idx, pooled, pooled_row_stride, dev_err=None):
    _check("msa_index_score_maxpool",
           lib().msa_index_score_maxpool(ctypes.byref(d), tensor_btd(q_idx), tensor_bhtd(k_idx),
                                         _ptr(pooled), pooled_row_stride, _ptr(dev_err), _stream()))


def msa_topk_blocks(d: Dims, pooled, pooled_row_stride, sel, dev_err=None):
    _check("msa_topk_blocks",
           lib().msa_topk_blocks(ctypes.byref(d), _ptr(pooled), pooled_row_stride, _ptr(sel),
                                 _ptr(dev_err), _stream()))


def msa_build_block_query_lists(d: Dims, sel, blk_offsets, entries, entry_pos, ws, dev_err=None):
    """entry_pos (int32, the shape of sel) receives the position in entries of
    each (b, g, query, slot), -1 for an empty slot."""
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("msa_build_block_query_lists",
           lib().msa_build_block_query_lists(ctypes.byref(d), _ptr(sel), _ptr(blk_offsets),
                                             _ptr(entries), _ptr(entry_pos), _ptr(ws), nbytes,
                                             _ptr(dev_err), _stream()))


def msa_build_block_query_lists_noalloc(d: Dims, sel, blk_offsets, entries, entry_pos,
                                        dev_err=None):
    """Same lists as msa_build_block_query_lists, with the library's built-in
    device scratch instead of a caller workspace (nothing is allocated)."""
    _check("msa_build_block_query_lists_noalloc",
           lib().msa_build_block_query_lists_noalloc(ctypes.byref(d), _ptr(sel), _ptr(blk_offsets),
                                                     _ptr(entries), _ptr(entry_pos),
                                                     _ptr(dev_err), _stream()))


def msa_sparse_attn_fwd(d: Dims, q, k, v, blk_offsets, entries, part_ml, part_acc, dev_err=None):
    _check("msa_sparse_attn_fwd",
           lib().msa_sparse_attn_fwd(ctypes.byref(d), tensor_btd(q), tensor_bhtd(k),
                                     tensor_bhtd(v), _ptr(blk_offsets), _ptr(entries),
                                     _ptr(part_ml), _ptr(part_acc), _ptr(dev_err), _stream()))


def msa_sparse_attn_fwd_compact(d: Dims, q, k, v, blk_offsets, entries, part_ml, part_acc16,
                                dev_err=None):
    """As msa_sparse_attn_fwd with compact pieces: part_acc16 bf16 [entries, R, 128]
    holds acc / l."""
    assert part_acc16.dtype == torch.bfloat16
    _check("msa_sparse_attn_fwd_compact",
           lib().msa_sparse_attn_fwd_compact(ctypes.byref(d), tensor_btd(q), tensor_bhtd(k),
                                             tensor_bhtd(v), _ptr(blk_offsets), _ptr(entries),
                                             _ptr(part_ml), _ptr(part_acc16), _ptr(dev_err),
                                             _stream()))


def msa_merge_partials_compact(d: Dims, entry_pos, part_ml, part_acc16, out, lse, dev_err=None):
    assert part_acc16.dtype == torch.bfloat16
    _check("msa_merge_partials_compact",
           lib().msa_merge_partials_compact(ctypes.byref(d), _ptr(entry_pos), _ptr(part_ml),
                                            _ptr(part_acc16), _ptr(out), _ptr(lse),
                                            _ptr(dev_err), _stream()))


def msa_sparse_attn_bwd(d: Dims, q, k, v, o, d_o, lse, blk_offsets, entries, delta, part_dq, dq,
                        dk, dv, dev_err=None):
    """dq [B,n_q,H,128], dk/dv [B,G,n_kv,128] (fp32) for upstream d_o (bf16)."""
    for t in (delta, part_dq, dq, dk, dv):
        assert t.dtype == torch.float32 and t.is_contiguous()
    _check("msa_sparse_attn_bwd",
           lib().msa_sparse_attn_bwd(ctypes.byref(d), tensor_btd(q), tensor_bhtd(k),
                                     tensor_bhtd(v), tensor_btd(o), tensor_btd(d_o), _ptr(lse),
                                     _ptr(blk_offsets), _ptr(entries), _ptr(delta),
                                     _ptr(part_dq), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dev_err),
                                     _stream()))


def msa_merge_partials(d: Dims, entry_pos, part_ml, part_acc, out, lse, dev_err=None):
    """Pieces in list order: slot s of (b, g, query) is at row entry_pos * R + r."""
    _check("msa_merge_partials",
           lib().msa_merge_partials(ctypes.byref(d), _ptr(entry_pos), _ptr(part_ml), _ptr(part_acc),
                                    _ptr(out), _ptr(lse), _ptr(dev_err), _stream()))


def msa_selection_recall_workspace(d: Dims, n_rows: int) -> int:
    return int(lib().msa_selection_recall_workspace(ctypes.byref(d), n_rows))


def msa_selection_recall(d: Dims, q, k, q_idx, k_idx, sel, rows, block_mass, recall, kl_pq, kl_qp,
                         ws, dev_err=None, lse_full=None):
    """Teacher block mass, recall and KL divergences for the sampled rows
    (rows: int64 device tensor of b * n_q + qi; block_mass [n * G, >= nblk]);
    lse_full [n, H] (optional) receives each head's full causal log-normaliser."""
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("msa_selection_recall",
           lib().msa_selection_recall(ctypes.byref(d), tensor_btd(q), tensor_bhtd(k),
                                      tensor_btd(q_idx), tensor_bhtd(k_idx), _ptr(sel), _ptr(rows),
                                      rows.numel(), _ptr(block_mass), block_mass.stride(0),
                                      _ptr(recall), _ptr(kl_pq), _ptr(kl_qp), _ptr(lse_full),
                                      _ptr(ws), nbytes, _ptr(dev_err), _stream()))


def msa_token_select_workspace(d: Dims, n_rows: int) -> int:
    return int(lib().msa_token_select_workspace(ctypes.byref(d), n_rows))


def msa_token_select_attention(d: Dims, q, k, v, q_idx, k_idx, rows, budget, tokens, out, lse, ws,
                               dev_err=None):
    """Top-budget tokens by index score per (sampled row, group) and attention
    over them: tokens int32 [n, G, budget], out fp32 [n, H, 128], lse fp32 [n, H]."""
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    assert tokens.dtype == torch.int32 and out.dtype == torch.float32 and lse.dtype == torch.float32
    _check("msa_token_select_attention",
           lib().msa_token_select_attention(ctypes.byref(d), tensor_btd(q), tensor_bhtd(k),
                                            tensor_bhtd(v), tensor_btd(q_idx), tensor_bhtd(k_idx),
                                            _ptr(rows), rows.numel(), budget, _ptr(tokens),
                                            _ptr(out), _ptr(lse), _ptr(ws), nbytes,
                                            _ptr(dev_err), _stream()))


def tensor_u8(t: torch.Tensor, bhtd: bool) -> Tensor:
    """uint8 [B, T, H, D] (q_idx codes) or [B, H, T, D] (k_idx codes), strides in bytes."""
    assert t.dim() == 4 and t.stride(3) == 1 and t.dtype == torch.uint8 and t.is_cuda
    if bhtd:
        return Tensor(t.data_ptr(), t.stride(0), t.stride(2), t.stride(1))
    return Tensor(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


def msa_quantize_e4m3(x, codes, scale):
    """x bf16 contiguous -> codes uint8 (same numel); scale: 2 device floats."""
    assert x.is_contiguous() and codes.is_contiguous() and codes.numel() == x.numel()
    assert scale.dtype == torch.float32 and scale.numel() >= 2
    _check("msa_quantize_e4m3",
           lib().msa_quantize_e4m3(_ptr(x), x.numel(), _ptr(codes), _ptr(scale), _stream()))


def msa_index_score_maxpool_e4m3(d: Dims, q_idx8, k_idx8, scale_q, scale_k, pooled, stride,
                                 dev_err=None):
    _check("msa_index_score_maxpool_e4m3",
           lib().msa_index_score_maxpool_e4m3(ctypes.byref(d), tensor_u8(q_idx8, False),
                                              tensor_u8(k_idx8, True), _ptr(scale_q),
                                              _ptr(scale_k), _ptr(pooled), stride,
                                              _ptr(dev_err), _stream()))
