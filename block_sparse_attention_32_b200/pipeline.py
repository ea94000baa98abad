"""The whole MSA hot path as five C-ABI calls on one stream.

``Buffers`` owns the intermediate device tensors (torch allocates them: the
library itself never allocates); ``forward`` enqueues

  msa_index_score_maxpool -> msa_topk_blocks -> msa_build_block_query_lists
  -> msa_sparse_attn_fwd -> msa_merge_partials

and returns the bf16 output and the fp32 log-sum-exp.  Beside it:
``select_e4m3`` (8-bit index branch), ``selection_recall`` (recall / KL
alignment target, optionally the full causal lse), ``token_select_attention``
(token-level selection at the same key budget), ``backward`` with ``Grads``
(dq, dk, dv for an upstream gradient) and ``HostPipeline`` (host buffers,
copies overlapped).  Every step runs in the library's kernels; this module
only marshals arguments.
"""
from __future__ import annotations

import dataclasses

import torch

from . import capi

# kernels each step launches (for launch accounting; with one query per row the
# block lists take 2 launches instead of 6)
LAUNCHES_PER_STEP = {"index": 1, "topk": 1, "block_lists": 6, "attn": 1, "merge": 1}


@dataclasses.dataclass
class Buffers:
    dims: capi.Dims
    pooled: torch.Tensor
    pooled_stride: int
    sel: torch.Tensor
    blk_offsets: torch.Tensor
    entries: torch.Tensor
    entry_pos: torch.Tensor
    ws: torch.Tensor
    part_ml: torch.Tensor
    part_acc: torch.Tensor
    out: torch.Tensor
    lse: torch.Tensor
    dev_err: torch.Tensor
    compact: bool = False

    @staticmethod
    def allocate(d: capi.Dims, device="cuda", compact: bool = False) -> "Buffers":
        """Intermediate buffers of one problem.  compact=True: the pieces' acc
        in bf16 (acc / l), read and written by the compact attention and merge
        calls."""
        B, n_q, G, H = d.batch, d.n_q, d.h_kv, d.h_q
        nblk = capi.msa_num_blocks(d)
        stride = (nblk + 3) // 4 * 4
        n_ent = capi.msa_num_entries(d)
        ws_bytes = capi.msa_block_query_lists_workspace(d)
        dev = torch.device(device)
        return Buffers(
            dims=d,
            pooled=torch.empty((B, G, n_q, stride), dtype=torch.float32, device=dev),
            pooled_stride=stride,
            sel=torch.empty((B, G, n_q, capi.TOPK), dtype=torch.int32, device=dev),
            blk_offsets=torch.empty((capi.msa_num_segments(d) + 1,), dtype=torch.int32,
                                    device=dev),
            entries=torch.empty((max(n_ent, 1),), dtype=torch.int32, device=dev),
            entry_pos=torch.empty((B, G, n_q, capi.TOPK), dtype=torch.int32, device=dev),
            ws=torch.empty(((ws_bytes + 15) // 16 * 4,), dtype=torch.int32, device=dev),
            # pieces in list order, [entries, R, ...]; sized for 16 slots per
            # (query, group), so the fp32 buffer also serves as the backward's
            # dq scratch [B, n_q, G, 16, R, 128]
            part_ml=torch.empty((B * n_q * G * capi.TOPK, H // G, 2), dtype=torch.float32,
                                device=dev),
            part_acc=torch.empty((B * n_q * G * capi.TOPK, H // G, capi.HEAD_DIM),
                                 dtype=torch.bfloat16 if compact else torch.float32, device=dev),
            out=torch.empty((B, n_q, H, capi.HEAD_DIM), dtype=torch.bfloat16, device=dev),
            lse=torch.empty((B, n_q, H), dtype=torch.float32, device=dev),
            dev_err=torch.zeros((4,), dtype=torch.int32, device=dev),
            compact=compact,
        )


def dims_for(w) -> capi.Dims:
    """Dims of a workloads.Workload."""
    return capi.make_dims(w.batch, w.n_q, w.n_kv, w.q_pos0, w.h_q, w.h_kv, w.d_idx,
                          h_kidx=w.h_kidx, scale=w.scale, q_window=w.q_window)


def select(buf: Buffers, q_idx, k_idx):
    """Index scores + max-pool + top-16 selection -> buf.sel."""
    d = buf.dims
    capi.msa_index_score_maxpool(d, q_idx, k_idx, buf.pooled, buf.pooled_stride, buf.dev_err)
    capi.msa_topk_blocks(d, buf.pooled, buf.pooled_stride, buf.sel, buf.dev_err)


def select_e4m3(buf: Buffers, q_idx, k_idx):
    """Selection from 8-bit index scores: per-tensor e4m3 copies of q_idx and
    k_idx, the tcgen05 kind::f8f6f4 score + max-pool kernel, then top-16 ->
    buf.sel.  Returns the codes and the two scales (device)."""
    d = buf.dims
    q8 = torch.empty(q_idx.shape, dtype=torch.uint8, device=q_idx.device)
    k8 = torch.empty(k_idx.shape, dtype=torch.uint8, device=k_idx.device)
    sq = torch.empty((2,), dtype=torch.float32, device=q_idx.device)
    sk = torch.empty((2,), dtype=torch.float32, device=q_idx.device)
    capi.msa_quantize_e4m3(q_idx, q8, sq)
    capi.msa_quantize_e4m3(k_idx, k8, sk)
    capi.msa_index_score_maxpool_e4m3(d, q8, k8, sq, sk, buf.pooled, buf.pooled_stride,
                                      buf.dev_err)
    capi.msa_topk_blocks(d, buf.pooled, buf.pooled_stride, buf.sel, buf.dev_err)
    return q8, k8, sq, sk


def attend(buf: Buffers, q, k, v, sel=None):
    """Block lists + KV-block-outer attention + merge over `sel` (default buf.sel)."""
    d = buf.dims
    s = buf.sel if sel is None else sel
    capi.msa_build_block_query_lists(d, s, buf.blk_offsets, buf.entries, buf.entry_pos, buf.ws,
                                     buf.dev_err)
    if buf.compact:
        capi.msa_sparse_attn_fwd_compact(d, q, k, v, buf.blk_offsets, buf.entries, buf.part_ml,
                                         buf.part_acc, buf.dev_err)
        capi.msa_merge_partials_compact(d, buf.entry_pos, buf.part_ml, buf.part_acc, buf.out,
                                        buf.lse, buf.dev_err)
    else:
        capi.msa_sparse_attn_fwd(d, q, k, v, buf.blk_offsets, buf.entries, buf.part_ml,
                                 buf.part_acc, buf.dev_err)
        capi.msa_merge_partials(d, buf.entry_pos, buf.part_ml, buf.part_acc, buf.out, buf.lse,
                                buf.dev_err)


def forward(buf: Buffers, q, k, v, q_idx, k_idx):
    """The whole hot path; returns (out bf16 [B,n_q,H,128], lse fp32 [B,n_q,H])."""
    select(buf, q_idx, k_idx)
    attend(buf, q, k, v)
    return buf.out, buf.lse


@dataclasses.dataclass
class Grads:
    delta: torch.Tensor
    dq: torch.Tensor
    dk: torch.Tensor
    dv: torch.Tensor

    @staticmethod
    def allocate(d: capi.Dims, device="cuda") -> "Grads":
        B, n_q, n_kv, G, H = d.batch, d.n_q, d.n_kv, d.h_kv, d.h_q
        dev = torch.device(device)
        return Grads(
            delta=torch.empty((B, n_q, H), dtype=torch.float32, device=dev),
            dq=torch.empty((B, n_q, H, capi.HEAD_DIM), dtype=torch.float32, device=dev),
            dk=torch.empty((B, G, n_kv, capi.HEAD_DIM), dtype=torch.float32, device=dev),
            dv=torch.empty((B, G, n_kv, capi.HEAD_DIM), dtype=torch.float32, device=dev),
        )


def backward(buf: Buffers, grads: Grads, q, k, v, d_out):
    """Gradients of the attention for upstream d_out (bf16 [B,n_q,H,128]) after a
    forward on the same buffers (its out, lse and block lists; the selection is
    fixed).  The forward's piece buffer holds the dQ pieces, so it must be the
    fp32 one (Buffers allocated with compact=False).  Returns (dq, dk, dv)."""
    if buf.compact:
        raise ValueError("the backward keeps fp32 dq pieces in the piece buffer: "
                         "allocate the Buffers with compact=False")
    capi.msa_sparse_attn_bwd(buf.dims, q, k, v, buf.out, d_out, buf.lse, buf.blk_offsets,
                             buf.entries, grads.delta, buf.part_acc, grads.dq, grads.dk,
                             grads.dv, buf.dev_err)
    return grads.dq, grads.dk, grads.dv


def selection_recall(buf: Buffers, q, k, q_idx, k_idx, rows, lse_full=None):
    """For sampled rows (int64 device tensor of b * n_q + qi): the main branch's
    block mass [n, G, nblk], the recall of buf.sel and KL(P||Q), KL(Q||P) [n, G].
    A given lse_full [n, H] fp32 receives each head's full causal log-normaliser."""
    d = buf.dims
    n, G = rows.numel(), d.h_kv
    nblk = capi.msa_num_blocks(d)
    dev = rows.device
    mass = torch.empty((n, G, nblk), dtype=torch.float32, device=dev)
    rec = torch.empty((n, G), dtype=torch.float32, device=dev)
    kpq = torch.empty((n, G), dtype=torch.float32, device=dev)
    kqp = torch.empty((n, G), dtype=torch.float32, device=dev)
    ws_bytes = capi.msa_selection_recall_workspace(d, n)
    ws = torch.empty(((ws_bytes + 15) // 16 * 4,), dtype=torch.int32, device=dev)
    capi.msa_selection_recall(d, q, k, q_idx, k_idx, buf.sel, rows, mass.view(n * G, nblk), rec,
                              kpq, kqp, ws, buf.dev_err, lse_full=lse_full)
    return mass, rec, kpq, kqp


def token_select_attention(d, q, k, v, q_idx, k_idx, rows, budget=2048, dev_err=None):
    """Token-level selection at the same key budget for sampled rows: tokens
    int32 [n, G, budget] (ascending, -1 padded), out fp32 [n, H, 128] and lse
    fp32 [n, H] of the attention over them."""
    n, G, H = rows.numel(), d.h_kv, d.h_q
    dev = rows.device
    tokens = torch.empty((n, G, budget), dtype=torch.int32, device=dev)
    out = torch.empty((n, H, 128), dtype=torch.float32, device=dev)
    lse = torch.empty((n, H), dtype=torch.float32, device=dev)
    ws_bytes = capi.msa_token_select_workspace(d, n)
    ws = torch.empty(((ws_bytes + 15) // 16 * 4,), dtype=torch.int32, device=dev)
    capi.msa_token_select_attention(d, q, k, v, q_idx, k_idx, rows, budget, tokens, out, lse, ws,
                                    dev_err)
    return tokens, out, lse


INPUT_NAMES = ("q", "k", "v", "q_idx", "k_idx")


class HostPipeline:
    """The hot path on batches held in pinned host memory, copies overlapped.

    ``run(host_in, host_out)`` takes a list of host input dicts (pinned q, k,
    v, q_idx, k_idx of the problem ``buf`` was allocated for) and a matching
    list of pinned host (out, lse) pairs.  For every batch it enqueues the
    host-to-device copy of the inputs (upload stream), the five library calls
    (the caller's current stream) and the device-to-host copy of out and lse
    (download stream).  Two device sets of inputs and outputs alternate, so
    batch i+1's upload and batch i-1's download run while batch i's kernels
    do; events order the three streams.  On return the caller's stream has
    waited for every download.
    """

    def __init__(self, buf: Buffers, like: dict):
        self.buf = buf
        self.dev_in = [{k: torch.empty_like(like[k]) for k in INPUT_NAMES} for _ in range(2)]
        self.dev_out = [(buf.out, buf.lse), (torch.empty_like(buf.out), torch.empty_like(buf.lse))]
        self.s_up = torch.cuda.Stream()
        self.s_down = torch.cuda.Stream()

    def run(self, host_in, host_out):
        comp = torch.cuda.current_stream()
        n = len(host_in)
        comp_done, down_done = [None] * n, [None] * n
        try:
            for i in range(n):
                slot = i % 2
                dev = self.dev_in[slot]
                out, lse = self.dev_out[slot]
                up = torch.cuda.Event()
                with torch.cuda.stream(self.s_up):
                    if i >= 2:                      # the kernels of batch i-2 read this set
                        self.s_up.wait_event(comp_done[i - 2])
                    for k in INPUT_NAMES:
                        dev[k].copy_(host_in[i][k], non_blocking=True)
                    up.record(self.s_up)
                comp.wait_event(up)
                if i >= 2:                          # batch i-2's output has left this set
                    comp.wait_event(down_done[i - 2])
                self.buf.out, self.buf.lse = out, lse
                forward(self.buf, dev["q"], dev["k"], dev["v"], dev["q_idx"], dev["k_idx"])
                comp_done[i] = torch.cuda.Event()
                comp_done[i].record(comp)
                down_done[i] = torch.cuda.Event()
                with torch.cuda.stream(self.s_down):
                    self.s_down.wait_event(comp_done[i])
                    host_out[i][0].copy_(out, non_blocking=True)
                    host_out[i][1].copy_(lse, non_blocking=True)
                    down_done[i].record(self.s_down)
            if n:
                comp.wait_event(down_done[n - 1])
        finally:
            self.buf.out, self.buf.lse = self.dev_out[0]


def check_device_errors(buf: Buffers):
    """Raise if any kernel reported a device-side error (synchronises)."""
    code = int(buf.dev_err[0].item())
    if code:
        raise capi.MSAError("device", 0) from RuntimeError(capi.DEVERR.get(code, code))
