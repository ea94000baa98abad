"""CPU oracle for the MSA hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``msa_oracle.c`` (plain C,
double precision, OpenMP over rows) through ctypes and shares no code with
the CUDA library.

Each function cites the page passage it follows in ``msa_oracle.c``:
  * ``index_pooled``  -- index-branch token scores + block max-pool
    ("MSA 稀疏注意力三国杀" page, section "MSA 架构：粗筛 + 精算", steps 1-2;
    "稀疏注意力速览" page, section 4, MSA entry);
  * ``topk`` / ``topk_f32`` -- 16 blocks per query and group, own block
    forced (same section, step 3; "稀疏注意力速览" page, MSA entry);
  * ``attention`` -- exact softmax attention over the selected tokens (same
    section, "第二步：精算"; softmax(QK^T/sqrt(d)) V from the "稀疏注意力架构革命"
    page, section 1.1);
  * ``merge`` -- log-sum-exp combination of per-block softmax pieces (the
    identity the KV-block-outer "Outer Gather Q" scheme relies on);
  * ``block_query_lists`` -- query->block lists inverted into block->query
    lists ("Kernel 创新：Outer Gather Q" section);
  * ``entry_positions`` -- the inverse of those lists, (query, slot) -> entry
    position (no counterpart on the pages: how the library finds a piece
    stored in list order; plain Python over the lists);
  * ``e4m3_value``, ``quantize_e4m3``, ``index_pooled_e4m3`` -- the 8-bit
    (e4m3) variant of steps 1-2: per-tensor scale amax / 448, nearest code
    with ties to even, pooled scores from the codes;
  * ``token_select_attention`` -- the token-level variant at the same
    budget: top-2048 tokens by index score, attention over them, and the full
    causal attention's lse;
  * ``attention_bwd`` -- gradients dQ, dK, dV of the main branch's attention
    over a fixed selection, for sparse training (section "MSA 能力不掉：3T token
    对照实验": MSA-PT and MSA-CPT train through the sparse attention);
  * ``selection_recall`` -- the main branch's attention mass per block (the
    teacher), the recall of the chosen blocks and the KL divergences to the
    index branch's block softmax (section "索引分支训练：KL 对齐").

Parity is pinned by ``tests/test_oracle_pins.py`` (brute force, closed forms,
invariants and hand-derived fixtures under ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmsa_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 128
TOPK = 16
HEAD_DIM = 128


def build(force: bool = False) -> str:
    """Compile ``msa_oracle.c`` into ``libmsa_oracle.so`` next to it."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fopenmp", "-fPIC", "-shared",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64, I32, F64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
            lib.msa_oracle_index_pooled.argtypes = [I64, I32, I32, I64, I32, P, P, P, P, I64, P]
            lib.msa_oracle_topk.argtypes = [I64, I32, P, I64, P, P]
            lib.msa_oracle_topk_f32.argtypes = [I64, I64, P, P, P]
            lib.msa_oracle_attention.argtypes = [I64, I32, I32, I64, P, P, P, P, P, P, F64, P, P]
            lib.msa_oracle_merge.argtypes = [I64, I32, I32, P, P, P, P, P, P]
            lib.msa_oracle_block_query_lists.argtypes = [I64, I32, I64, I64, I64, P, P, P]
            lib.msa_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.msa_oracle_e4m3_value.restype = F64
            lib.msa_oracle_quantize_e4m3.argtypes = [I64, P, P, P]
            lib.msa_oracle_index_pooled_e4m3.argtypes = [I64, I32, I32, I64, I32, P, P, P, P, F64,
                                                         F64, I64, P]
            lib.msa_oracle_token_select_attention.argtypes = [I64, I32, I32, I32, I64, I32, I64,
                                                              P, P, P, P, P, P, P, F64, P, P,
                                                              P, P]
            lib.msa_oracle_attention_bwd.argtypes = [I64, I64, I64, I64, I32, I32, P, P, P, P, P,
                                                     F64, P, P, P, P, P]
            lib.msa_oracle_selection_recall.argtypes = [I64, I32, I32, I32, I64, I32, P, P, P, P,
                                                         P, P, P, F64, I64, P, P, P, P]
            for f in (lib.msa_oracle_index_pooled, lib.msa_oracle_topk, lib.msa_oracle_topk_f32,
                      lib.msa_oracle_attention, lib.msa_oracle_merge,
                      lib.msa_oracle_block_query_lists, lib.msa_oracle_selection_recall,
                      lib.msa_oracle_quantize_e4m3, lib.msa_oracle_index_pooled_e4m3,
                      lib.msa_oracle_token_select_attention, lib.msa_oracle_attention_bwd):
                f.restype = None
            _lib = lib
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def bf16_bits(x) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 torch tensor (or pass uint16 through)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def num_blocks(n_kv: int) -> int:
    return (n_kv + BLOCK - 1) // BLOCK


def index_pooled(q_idx_rows, row_pos, row_batch, k_idx, out_stride=None):
    """Pooled block scores for the given query rows.

    q_idx_rows: uint16 [n_rows, G, d_idx]; row_pos/row_batch: int64 [n_rows];
    k_idx: uint16 [B', h_kidx, n_kv, d_idx].  Returns float64
    [n_rows, G, out_stride] with NaN at c >= own(t).
    """
    lib = _load()
    q = _c(q_idx_rows, np.uint16)
    k = _c(k_idx, np.uint16)
    pos = _c(row_pos, np.int64)
    bat = _c(row_batch, np.int64)
    n_rows, G, d_idx = q.shape
    _, h_kidx, n_kv, d2 = k.shape
    assert d2 == d_idx and d_idx <= 256 and h_kidx in (1, G)
    stride = out_stride or num_blocks(n_kv)
    out = np.empty((n_rows, G, stride), np.float64)
    lib.msa_oracle_index_pooled(n_rows, G, d_idx, n_kv, h_kidx, _p(q), _p(pos), _p(bat),
                                _p(k), stride, _p(out))
    return out


def topk(pooled, row_pos):
    """Selected blocks [n_rows, G, 16] (ascending, -1 padded) from float64 scores."""
    lib = _load()
    s = _c(pooled, np.float64)
    pos = _c(row_pos, np.int64)
    n_rows, G, stride = s.shape
    sel = np.empty((n_rows, G, TOPK), np.int32)
    lib.msa_oracle_topk(n_rows, G, _p(pos), stride, _p(s), _p(sel))
    return sel


def topk_f32(pooled_f32, own):
    """Selection on float32 scores [n_rows, stride] with own block per row."""
    lib = _load()
    s = _c(pooled_f32, np.float32)
    o = _c(own, np.int64)
    n_rows, stride = s.shape
    sel = np.empty((n_rows, TOPK), np.int32)
    lib.msa_oracle_topk_f32(n_rows, stride, _p(o), _p(s), _p(sel))
    return sel


def attention(q_rows, row_pos, row_batch, k, v, sel, scale):
    """Exact softmax attention of the rows over their selected tokens.

    q_rows uint16 [n_rows, H, 128]; k, v uint16 [B', G, n_kv, 128];
    sel int32 [n_rows, G, 16].  Returns (out float64 [n_rows, H, 128],
    lse float64 [n_rows, H]).
    """
    lib = _load()
    q = _c(q_rows, np.uint16)
    kk = _c(k, np.uint16)
    vv = _c(v, np.uint16)
    s = _c(sel, np.int32)
    pos = _c(row_pos, np.int64)
    bat = _c(row_batch, np.int64)
    n_rows, H, D = q.shape
    _, G, n_kv, D2 = kk.shape
    assert D == HEAD_DIM and D2 == HEAD_DIM and H % G == 0 and vv.shape == kk.shape
    assert s.shape == (n_rows, G, TOPK)
    out = np.empty((n_rows, H, HEAD_DIM), np.float64)
    lse = np.empty((n_rows, H), np.float64)
    lib.msa_oracle_attention(n_rows, H, G, n_kv, _p(q), _p(pos), _p(bat), _p(kk), _p(vv),
                             _p(s), float(scale), _p(out), _p(lse))
    return out, lse


def merge(valid, m, l, acc):
    """Log-sum-exp combination of softmax pieces: valid/m/l [n, S], acc [n, S, D]."""
    lib = _load()
    va = _c(valid, np.int32)
    mm = _c(m, np.float64)
    ll = _c(l, np.float64)
    aa = _c(acc, np.float64)
    n, S, D = aa.shape
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    lib.msa_oracle_merge(n, S, D, _p(va), _p(mm), _p(ll), _p(aa), _p(out), _p(lse))
    return out, lse


def query_window(h_q, h_kv, q_window=0):
    """The query window of the block->query lists: q_window when positive,
    else the largest power of two W >= 128 with W * (h_q / h_kv) * 256 bytes
    <= 32 MiB (one window's gathered query rows of one group), the rule the
    library's header states."""
    if q_window > 0:
        return int(q_window)
    R = h_q // h_kv
    w = 128
    while 2 * w * R * 256 <= (32 << 20):
        w *= 2
    return w


def block_query_lists(sel, nblk, window=None):
    """CSR inversion of sel [B, G, n_q, 16] with query windows of `window`
    (default: one window over all queries) -> (offsets int64
    [B*G*nwin*nblk+1], entries int32)."""
    lib = _load()
    s = _c(sel, np.int32)
    B, G, n_q, T = s.shape
    assert T == TOPK
    window = int(window or n_q)
    nwin = (n_q + window - 1) // window
    offsets = np.empty((B * G * nwin * nblk + 1,), np.int64)
    n_ent = int((s >= 0).sum())
    entries = np.empty((max(n_ent, 1),), np.int32)
    lib.msa_oracle_block_query_lists(B, G, n_q, nblk, window, _p(s), _p(offsets), _p(entries))
    return offsets, entries[:n_ent]


def entry_positions(offsets, entries, B, G, n_q, nblk, window=None):
    """Inverse of the block->query lists: pos [B, G, n_q, 16] int32 with
    pos[b, g, i, slot] = p where entries[p] = (i << 4) | slot lies in a
    segment of (b, g), and -1 for every (query, slot) no entry names.

    The pages have no counterpart: it is how the library finds a piece written
    in list order (the position of its entry), written out from its
    definition over the segments ((b * G + g) * nwin + w) * nblk + c."""
    window = int(window or n_q)
    nwin = (n_q + window - 1) // window
    off = np.asarray(offsets, np.int64)
    ent = np.asarray(entries, np.int64)
    pos = np.full((B, G, n_q, TOPK), -1, np.int32)
    for s in range(B * G * nwin * nblk):
        bg = (s // nblk) // nwin
        b, g = bg // G, bg % G
        for p in range(int(off[s]), int(off[s + 1])):
            e = int(ent[p])
            pos[b, g, e >> 4, e & 15] = p
    return pos


def forward_rows(q_rows, q_idx_rows, row_pos, row_batch, k, v, k_idx, scale):
    """Whole path for sampled rows: pooled scores, selection, attention."""
    pooled = index_pooled(q_idx_rows, row_pos, row_batch, k_idx)
    sel = topk(pooled, row_pos)
    out, lse = attention(q_rows, row_pos, row_batch, k, v, sel, scale)
    return pooled, sel, out, lse


def selection_recall(q_rows, q_idx_rows, row_pos, row_batch, k, k_idx, sel, scale, stride=None):
    """Teacher block mass, recall and KL divergences for the given rows.

    q_rows uint16 [n, H, 128]; q_idx_rows uint16 [n, G, d_idx]; k uint16
    [B', G, n_kv, 128]; k_idx uint16 [B', h_kidx, n_kv, d_idx]; sel int32
    [n, G, 16].  Returns (block_mass [n, G, stride], recall [n, G],
    kl_pq [n, G], kl_qp [n, G]) in float64.
    """
    lib = _load()
    q = _c(q_rows, np.uint16)
    qi = _c(q_idx_rows, np.uint16)
    kk = _c(k, np.uint16)
    ki = _c(k_idx, np.uint16)
    s = _c(sel, np.int32)
    pos = _c(row_pos, np.int64)
    bat = _c(row_batch, np.int64)
    n, H, D = q.shape
    _, G, d_idx = qi.shape
    _, G2, n_kv, _ = kk.shape
    h_kidx = ki.shape[1]
    assert D == HEAD_DIM and G2 == G and s.shape == (n, G, TOPK)
    stride = stride or num_blocks(n_kv)
    mass = np.empty((n, G, stride), np.float64)
    rec = np.empty((n, G), np.float64)
    kpq = np.empty((n, G), np.float64)
    kqp = np.empty((n, G), np.float64)
    lib.msa_oracle_selection_recall(n, H, G, d_idx, n_kv, h_kidx, _p(q), _p(qi), _p(pos), _p(bat),
                                    _p(kk), _p(ki), _p(s), float(scale), stride, _p(mass), _p(rec),
                                    _p(kpq), _p(kqp))
    return mass, rec, kpq, kqp


def e4m3_value(code: int) -> float:
    """Value of one e4m3 code."""
    return float(_load().msa_oracle_e4m3_value(int(code) & 0xFF))


def quantize_e4m3(x_bits):
    """bf16 bits (any shape) -> (codes uint8 same shape, scale float)."""
    lib = _load()
    x = _c(x_bits, np.uint16)
    codes = np.empty(x.shape, np.uint8)
    scale = np.zeros((1,), np.float32)
    lib.msa_oracle_quantize_e4m3(x.size, _p(x), _p(scale), _p(codes))
    return codes, float(scale[0])


def index_pooled_e4m3(q_codes_rows, row_pos, row_batch, k_codes, s_q, s_k, out_stride=None):
    """Pooled block scores from e4m3 codes (see index_pooled): float64
    [n_rows, G, out_stride], NaN at c >= own(t)."""
    lib = _load()
    q = _c(q_codes_rows, np.uint8)
    k = _c(k_codes, np.uint8)
    pos = _c(row_pos, np.int64)
    bat = _c(row_batch, np.int64)
    n_rows, G, d_idx = q.shape
    _, h_kidx, n_kv, _ = k.shape
    stride = out_stride or num_blocks(n_kv)
    out = np.empty((n_rows, G, stride), np.float64)
    lib.msa_oracle_index_pooled_e4m3(n_rows, G, d_idx, n_kv, h_kidx, _p(q), _p(pos), _p(bat), _p(k),
                                     float(s_q), float(s_k), stride, _p(out))
    return out


def token_select_attention(q_rows, q_idx_rows, row_pos, row_batch, k, v, k_idx, scale, budget=2048):
    """Top-`budget` tokens by index score per (row, group) (ascending, -1 padded,
    int64 [n, G, budget]), attention over them (out [n, H, 128], lse [n, H]) and
    the full causal lse [n, H], all float64."""
    lib = _load()
    q = _c(q_rows, np.uint16)
    qi = _c(q_idx_rows, np.uint16)
    kk = _c(k, np.uint16)
    vv = _c(v, np.uint16)
    ki = _c(k_idx, np.uint16)
    pos = _c(row_pos, np.int64)
    bat = _c(row_batch, np.int64)
    n, H, _ = q.shape
    _, G, d_idx = qi.shape
    n_kv = kk.shape[2]
    tokens = np.empty((n, G, budget), np.int64)
    out = np.empty((n, H, HEAD_DIM), np.float64)
    lse = np.empty((n, H), np.float64)
    lse_full = np.empty((n, H), np.float64)
    lib.msa_oracle_token_select_attention(n, H, G, d_idx, n_kv, ki.shape[1], budget, _p(q), _p(qi),
                                          _p(pos), _p(bat), _p(kk), _p(vv), _p(ki), float(scale),
                                          _p(tokens), _p(out), _p(lse), _p(lse_full))
    return tokens, out, lse, lse_full


def attention_bwd(q, k, v, dout, sel, scale, q_pos0=0):
    """Gradients of the sparse attention for an upstream dout, the selection
    fixed.  q, dout [B, n_q, H, 128]; k, v [B, G, n_kv, 128] (float64 arrays,
    or bf16 bit patterns as uint16, converted exactly); sel [B, G, n_q, 16]
    int32.  Returns dq [B, n_q, H, 128], dk, dv [B, G, n_kv, 128], lse and
    delta = dO.o [B, n_q, H], all float64."""
    lib = _load()

    def f64(a):
        return _c(bits_to_f64(a) if a.dtype == np.uint16 else a, np.float64)

    qq, kk, vv, do = f64(q), f64(k), f64(v), f64(dout)
    ss = _c(sel, np.int32)
    B, n_q, H, _ = qq.shape
    G, n_kv = kk.shape[1], kk.shape[2]
    assert ss.shape == (B, G, n_q, TOPK) and do.shape == qq.shape and vv.shape == kk.shape
    dq = np.empty_like(qq)
    dk = np.empty_like(kk)
    dv = np.empty_like(vv)
    lse = np.empty((B, n_q, H), np.float64)
    delta = np.empty((B, n_q, H), np.float64)
    lib.msa_oracle_attention_bwd(B, n_q, n_kv, int(q_pos0), H, G, _p(qq), _p(kk), _p(vv), _p(do),
                                 _p(ss), float(scale), _p(dq), _p(dk), _p(dv), _p(lse), _p(delta))
    return dq, dk, dv, lse, delta
