"""The whole MSA hot path as five C-ABI calls on one stream.

``Buffers`` owns the intermediate device tensors (torch allocates them: the
library itself never allocates); ``forward`` enqueues

  msa_index_score_maxpool -> msa_topk_blocks -> msa_build_block_query_lists
  -> msa_sparse_attn_fwd -> msa_merge_partials

and returns the bf16 output and the fp32 log-sum-exp.  Every step runs in the
library's kernels; this module only marshals arguments.
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
    ws: torch.Tensor
    part_ml: torch.Tensor
    part_acc: torch.Tensor
    out: torch.Tensor
    lse: torch.Tensor
    dev_err: torch.Tensor

    @staticmethod
    def allocate(d: capi.Dims, device="cuda") -> "Buffers":
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
            blk_offsets=torch.empty((B * G * nblk + 1,), dtype=torch.int32, device=dev),
            entries=torch.empty((max(n_ent, 1),), dtype=torch.int32, device=dev),
            ws=torch.empty(((ws_bytes + 15) // 16 * 4,), dtype=torch.int32, device=dev),
            part_ml=torch.empty((B, n_q, G, capi.TOPK, H // G, 2), dtype=torch.float32,
                                device=dev),
            part_acc=torch.empty((B, n_q, G, capi.TOPK, H // G, capi.HEAD_DIM),
                                 dtype=torch.float32, device=dev),
            out=torch.empty((B, n_q, H, capi.HEAD_DIM), dtype=torch.bfloat16, device=dev),
            lse=torch.empty((B, n_q, H), dtype=torch.float32, device=dev),
            dev_err=torch.zeros((4,), dtype=torch.int32, device=dev),
        )


def dims_for(w) -> capi.Dims:
    """Dims of a workloads.Workload."""
    return capi.make_dims(w.batch, w.n_q, w.n_kv, w.q_pos0, w.h_q, w.h_kv, w.d_idx,
                          h_kidx=w.h_kidx, scale=w.scale)


def select(buf: Buffers, q_idx, k_idx):
    """Index scores + max-pool + top-16 selection -> buf.sel."""
    d = buf.dims
    capi.msa_index_score_maxpool(d, q_idx, k_idx, buf.pooled, buf.pooled_stride, buf.dev_err)
    capi.msa_topk_blocks(d, buf.pooled, buf.pooled_stride, buf.sel, buf.dev_err)


def attend(buf: Buffers, q, k, v, sel=None):
    """Block lists + KV-block-outer attention + merge over `sel` (default buf.sel)."""
    d = buf.dims
    s = buf.sel if sel is None else sel
    capi.msa_build_block_query_lists(d, s, buf.blk_offsets, buf.entries, buf.ws, buf.dev_err)
    capi.msa_sparse_attn_fwd(d, q, k, v, buf.blk_offsets, buf.entries, buf.part_ml,
                             buf.part_acc, buf.dev_err)
    capi.msa_merge_partials(d, s, buf.part_ml, buf.part_acc, buf.out, buf.lse, buf.dev_err)


def forward(buf: Buffers, q, k, v, q_idx, k_idx):
    """The whole hot path; returns (out bf16 [B,n_q,H,128], lse fp32 [B,n_q,H])."""
    select(buf, q_idx, k_idx)
    attend(buf, q, k, v)
    return buf.out, buf.lse


def check_device_errors(buf: Buffers):
    """Raise if any kernel reported a device-side error (synchronises)."""
    code = int(buf.dev_err[0].item())
    if code:
        raise capi.MSAError("device", 0) from RuntimeError(capi.DEVERR.get(code, code))
