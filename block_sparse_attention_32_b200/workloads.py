"""Seeded synthetic workloads for the MSA hot path.

This module only draws inputs: it holds none of the method's arithmetic and
is shared by the tests, the smoke check and the benchmark (and, through
them, by both the CUDA path and the CPU oracle).  No dataset, model or
trained weight is involved: every tensor is drawn from a seeded generator
with the shapes of the long-context workloads the MSA pages discuss (1M
context, GQA, 128-token blocks, top-16).

Structure added on top of N(0,1) noise, in fp32 before the bf16 cast (the
pages describe the patterns trained index heads show: a recency band along
the diagonal, an attention sink on the first tokens, and per-group stripes
reaching far back -- "MSA 稀疏注意力三国杀" page, appendix on emergent head
patterns):

* plant(block P, group g, targets T): token i of block P gets
  ``k_idx += a * sum_{t in T, t mod 128 = i} q_idx[t, g]``, so the index
  score of P for each target query is large and P surfaces in its top-k;
* sink: the first block's k_idx is scaled by 2;
* recency: token i of key block c gets ``+ 1.0 * sum_{d=1..4} sum_g
  q_idx[128 (c+d) + i, g]`` (the four blocks before a query lean toward it).
"""
from __future__ import annotations

import dataclasses
import math

import torch

BLOCK = 128
TOPK = 16
HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q: int
    n_kv: int
    q_pos0: int
    h_q: int
    h_kv: int
    d_idx: int
    h_kidx: int = 1
    seed: int = 0
    plants_per_group: int = 0      # planted far blocks per (batch, group)
    plant_targets: int = 0         # target queries per plant (0 = all listed below)
    plant_last_queries: int = 0    # tiny: targets are the last N queries
    plant_amp: float = 3.0
    sink: bool = False
    recency: bool = False
    q_scale: float = 1.0           # >1 gives peaked softmax rows
    q_window: int = 0              # query window of the block->query lists (0: library default)

    @property
    def nblk(self) -> int:
        return (self.n_kv + BLOCK - 1) // BLOCK

    @property
    def group_size(self) -> int:
        return self.h_q // self.h_kv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(HEAD_DIM)


# The five workloads (sizes of the pages' long-context settings).
TINY = Workload("tiny_prefill_4k", 1, 4096, 4096, 0, 4, 1, 64, seed=20261202,
                plants_per_group=2, plant_last_queries=512)
P32 = Workload("prefill_32k", 1, 32768, 32768, 0, 32, 8, 128, seed=20261203,
               plants_per_group=8, plant_targets=128)
P128 = Workload("prefill_128k", 1, 131072, 131072, 0, 64, 8, 128, seed=20261204,
                sink=True, recency=True)
DECODE = Workload("decode_64x256k", 64, 1, 262144, 262143, 64, 8, 128, seed=20261205,
                  plants_per_group=2, plant_targets=1)
M1 = Workload("chunked_prefill_1m", 1, 8192, 1056768, 1048576, 64, 8, 128, seed=20261206,
              plants_per_group=4, plant_targets=128, sink=True, recency=True)

CONFIGS = {w.name: w for w in (TINY, P32, P128, DECODE, M1)}

# Profiling-sized prefill with the 128K workload's structure (R = 8, sink and
# recency): ~2.2 GB of pieces, larger than L2, small enough for hardware
# counter capture.
PROFILE_8K = Workload("profile_8k_r8", 1, 8192, 8192, 0, 32, 4, 128, seed=3, sink=True,
                      recency=True)
# Profiling-sized decode: 4 sequences of the decode workload's shape (k_idx 268 MB,
# K/V 4.3 GB), larger than L2.
PROFILE_DECODE = Workload("profile_decode_b4", 4, 1, 262144, 262143, 64, 8, 128, seed=5,
                          plants_per_group=2, plant_targets=1)
# Profiling-sized backward: 4096 queries with the 128K workload's heads (dq pieces 2.1 GB).
PROFILE_BWD = Workload("profile_bwd_4k_r8", 1, 4096, 4096, 0, 64, 8, 128, seed=9)
ALL = dict(CONFIGS, **{PROFILE_8K.name: PROFILE_8K, PROFILE_DECODE.name: PROFILE_DECODE,
                       PROFILE_BWD.name: PROFILE_BWD})


def small(name, batch, n_q, n_kv, q_pos0, h_q, h_kv, d_idx, seed, **kw) -> Workload:
    """A parity-sized workload (ragged tails, several tiles)."""
    return Workload(name, batch, n_q, n_kv, q_pos0, h_q, h_kv, d_idx, seed=seed, **kw)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, device, dtype=torch.float32):
    return torch.randn(*shape, generator=gen, device=device, dtype=dtype)


def _plant_list(w: Workload, gen_cpu: torch.Generator):
    """(batch, group, block P, target query indices) tuples, drawn on the CPU."""
    plants = []
    if w.plants_per_group == 0:
        return plants
    own_first = w.q_pos0 // BLOCK
    for b in range(w.batch):
        for g in range(w.h_kv):
            for _ in range(w.plants_per_group):
                if w.plant_last_queries:
                    targets = torch.arange(w.n_q - w.plant_last_queries, w.n_q)
                    hi = (w.q_pos0 + w.n_q - w.plant_last_queries) // BLOCK
                    lo = 0
                elif w.plant_targets >= w.n_q:
                    targets = torch.arange(w.n_q)
                    lo, hi = (1 if w.sink else 0), max(own_first - 4, 1)
                else:
                    # targets: random queries; the planted block lies before all of them
                    tq = torch.randint(w.n_q // 2, w.n_q, (w.plant_targets,), generator=gen_cpu)
                    targets = torch.unique(tq)
                    lo = 1 if w.sink else 0
                    hi = max((w.q_pos0 + int(targets.min())) // BLOCK - 4, lo + 1)
                blk = int(torch.randint(lo, hi, (1,), generator=gen_cpu))
                plants.append((b, g, blk, targets))
    return plants


def make_inputs(w: Workload, device="cpu", with_qkv: bool = True):
    """Draw q, k, v, q_idx, k_idx for workload ``w`` on ``device`` (bf16).

    Layouts (innermost dimension contiguous):
      q      [B, n_q, H, 128]         k, v [B, H_kv, n_kv, 128]
      q_idx  [B, n_q, G, d_idx]       k_idx [B, h_kidx, n_kv, d_idx]
    """
    device = torch.device(device)
    gen = _gen(device, w.seed)
    gen_cpu = _gen("cpu", w.seed + 7)
    B, G = w.batch, w.h_kv
    out = {}
    if with_qkv:
        q = _randn((B, w.n_q, w.h_q, HEAD_DIM), gen, device, torch.bfloat16)
        if w.q_scale != 1.0:
            q = (q.float() * w.q_scale).to(torch.bfloat16)
        out["q"] = q
        out["k"] = _randn((B, w.h_kv, w.n_kv, HEAD_DIM), gen, device, torch.bfloat16)
        out["v"] = _randn((B, w.h_kv, w.n_kv, HEAD_DIM), gen, device, torch.bfloat16)
    q_idx = _randn((B, w.n_q, G, w.d_idx), gen, device, torch.bfloat16)
    k_idx = _randn((B, w.h_kidx, w.n_kv, w.d_idx), gen, device, torch.bfloat16)

    # structure, per batch row, in fp32 on the touched slices only
    for b in range(B):
        if w.sink:
            k_idx[b, :, :BLOCK] = (k_idx[b, :, :BLOCK].float() * 2.0).to(torch.bfloat16)
        if w.recency:
            _add_recency(w, q_idx[b], k_idx[b])
    for (b, g, blk, targets) in _plant_list(w, gen_cpu):
        hk = 0 if w.h_kidx == 1 else g
        tq = targets.to(device)
        qv = q_idx[b, tq, g].float()                       # [T, d_idx]
        tok = (w.q_pos0 + tq) % BLOCK                       # token slot in the block
        add = torch.zeros((BLOCK, w.d_idx), device=device)
        add.index_add_(0, tok, qv)
        sl = k_idx[b, hk, blk * BLOCK:(blk + 1) * BLOCK]
        k_idx[b, hk, blk * BLOCK:(blk + 1) * BLOCK] = (
            sl.float() + w.plant_amp * add[: sl.shape[0]]).to(torch.bfloat16)
    out["q_idx"] = q_idx
    out["k_idx"] = k_idx
    return out


def _add_recency(w: Workload, q_idx_b: torch.Tensor, k_idx_b: torch.Tensor):
    """Token i of key block c += sum over groups of q_idx at token i of blocks c+1..c+4."""
    nqb_first = w.q_pos0 // BLOCK
    full = w.n_q // BLOCK
    if full == 0 or w.q_pos0 % BLOCK:
        return
    # per query block: sum over groups, [full, 128, d_idx]
    qs = q_idx_b[: full * BLOCK].float().sum(dim=1).view(full, BLOCK, w.d_idx)
    for hk in range(w.h_kidx):
        for d in range(1, 5):
            # key block c = qb - d for every query block qb
            c0 = nqb_first - d
            lo = max(0, -c0)
            if lo >= full:
                continue
            kb = k_idx_b[hk, (c0 + lo) * BLOCK:(c0 + full) * BLOCK]
            kb = kb.view(full - lo, BLOCK, w.d_idx)
            k_idx_b[hk, (c0 + lo) * BLOCK:(c0 + full) * BLOCK] = (
                kb.float() + qs[lo:]).to(torch.bfloat16).view(-1, w.d_idx)


def upstream_grad(w: Workload, device="cpu", seed_offset: int = 101):
    """A seeded upstream gradient dO [B, n_q, H, 128] (bf16, N(0,1)) for the
    attention's backward."""
    device = torch.device(device)
    return _randn((w.batch, w.n_q, w.h_q, HEAD_DIM), _gen(device, w.seed + seed_offset), device,
                  torch.bfloat16)


def random_selection(w: Workload, device="cpu", seed_offset: int = 202):
    """A seeded valid block selection [B, G, n_q, 16] int32: each query's own
    block and up to 15 distinct earlier blocks drawn uniformly, ascending,
    -1 after the last.  It stands in for the index branch's choice where a
    step takes the selection as an input (the attention and its backward)."""
    device = torch.device(device)
    gen = _gen(device, w.seed + seed_offset)
    B, G, n_q, nblk = w.batch, w.h_kv, w.n_q, w.nblk
    own = (w.q_pos0 + torch.arange(n_q, device=device)) // BLOCK          # [n_q]
    r = torch.rand((B, G, n_q, nblk), generator=gen, device=device)
    blk = torch.arange(nblk, device=device)
    r = torch.where(blk[None, None, None, :] < own[None, None, :, None], r, torch.full_like(r, -1.0))
    k = min(TOPK - 1, nblk)
    vals, idx = r.topk(k, dim=-1) if k > 0 else (r[..., :0], r[..., :0].long())
    big = torch.iinfo(torch.int32).max
    idx = torch.where(vals >= 0, idx, torch.full_like(idx, big))
    sel = torch.cat([idx, own[None, None, :, None].expand(B, G, n_q, 1)], dim=-1)
    if sel.shape[-1] < TOPK:
        pad = torch.full((B, G, n_q, TOPK - sel.shape[-1]), big, device=device, dtype=sel.dtype)
        sel = torch.cat([sel, pad], dim=-1)
    sel = sel.sort(dim=-1).values
    sel = torch.where(sel == big, torch.full_like(sel, -1), sel)
    return sel.to(torch.int32).contiguous()
