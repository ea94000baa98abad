"""Benchmark of the MSA hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
index scores + block max-pool, top-16 selection, block->query lists,
KV-block-outer attention and the log-sum-exp merge, for the 128K-token
prefill workload (batch 1, 131072 tokens, 64 query heads / 8 KV heads,
d_idx 128).  The headline metric is queries/s of that pass; the selected-token
attention TFLOP/s and a decode pass (64 sequences x 256K cached tokens, one
new token each) are reported alongside.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl msa|reference]

With N > 1 (launched by torchrun) every rank runs its own independent
instance of the workload (the problems share nothing: weak scaling, no
collective on the data path); `value` = all ranks' queries / the slowest
rank's time.  `--impl reference` times the CPU oracle on a bounded sample of
rows of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK, "fallback"


def work_counts(w):
    """Algorithmic FLOPs and (query, group, block) entry count of one pass."""
    B, G, R, d_idx = w.batch, w.h_kv, w.h_q // w.h_kv, w.d_idx
    t = w.q_pos0 + np.arange(w.n_q, dtype=np.int64)
    own = t // 128
    # index: every token of every candidate block c < own(t), per group: 2*d_idx FLOP
    idx_flops = float(B * G * 2 * d_idx * 128 * own.sum())
    # attention: 4*128 FLOP per (query, head, selected causal token)
    nsel_full = np.minimum(16, own + 1)
    # selected tokens: own block contributes t%128+1, the others 128 each
    toks = (nsel_full - 1) * 128 + (t % 128) + 1
    attn_flops = float(B * w.h_q * 4 * 128 * toks.sum())
    n_entries = int(B * G * nsel_full.sum())
    return idx_flops, attn_flops, n_entries


def bytes_model(w, n_entries, n_pieces_nonempty, piece_bytes=520):
    """Algorithmic DRAM bytes per launch of each kernel.

    attention: per (query, block) entry the R gathered Q rows (256 B each) and
    the R pieces written (fp32: 512 B acc + 8 B (m, l); compact: 256 + 8); per selected (batch,
    group, block) the 64 KB K/V tile once; the entry list.  block lists: sel
    read twice, the entries and their position map written.  merge: the pieces
    read once, the position map, and the bf16 output + lse written."""
    B, G, R = w.batch, w.h_kv, w.h_q // w.h_kv
    t = w.q_pos0 + np.arange(w.n_q, dtype=np.int64)
    own = t // 128
    rows = B * G * w.n_q
    return {
        "index": float(B * w.n_q * G * w.d_idx * 2 + B * w.h_kidx * w.n_kv * w.d_idx * 2
                       + 4 * B * G * own.sum()),
        "topk": float(4 * B * G * own[own >= 16].sum() + 64 * rows),
        "block_lists": float(64 * rows * 3 + 4 * n_entries * 2),
        "attn": float(n_entries * R * (256 + piece_bytes) + n_pieces_nonempty * 65536
                      + 4 * n_entries),
        "merge": float(n_entries * R * piece_bytes + 64 * rows + B * w.n_q * w.h_q * (256 + 4)),
    }


def source_digest(paths):
    import hashlib
    h = hashlib.sha256()
    for pth in paths:
        with open(pth, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(kernel_files, record, units):
    """DRAM bytes per launch from a committed ncu summary taken on a small case
    of the same kernel: its bytes per unit (a list entry of the attention)
    times the units one launch of this workload processes.  None when the
    kernel sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", record)
    try:
        kv = dict(line.split(":", 1) for line in open(path) if ":" in line)
    except OSError:
        return None
    digest = source_digest([os.path.join(ROOT, "block_sparse_attention_32_b200", "csrc", f)
                            for f in kernel_files])
    if kv.get("source_sha256", "").strip() != digest:
        return None
    try:
        return float(kv["dram_bytes_per_entry"].strip()) * units
    except (KeyError, ValueError):
        return None


def sample_clocks(stop_file, out_path):
    cmd = ["nvidia-smi", "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,"
           "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
           "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
           "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits", "-lms", "200"]
    try:
        return subprocess.Popen(cmd, stdout=open(out_path, "w"), stderr=subprocess.DEVNULL)
    except OSError:
        return None


def summarize_clocks(path, gpu_index):
    sm, mx, reasons = [], [], set()
    try:
        for line in open(path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9 or f[0] != str(gpu_index):
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                  "sw_power_cap"], f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
    except OSError:
        pass
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons)}


class Stages:
    """CUDA events between the C-ABI calls of a step (same stream)."""

    NAMES = ["index", "topk", "block_lists", "attn", "merge"]

    def __init__(self):
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.NAMES) + 1)]

    def ms(self):
        return {n: self.ev[i].elapsed_time(self.ev[i + 1]) for i, n in enumerate(self.NAMES)}


def percentile(xs, q):
    """q-th percentile (0..100) of xs by linear interpolation between order statistics."""
    v = sorted(xs)
    if len(v) == 1:
        return v[0]
    pos = (len(v) - 1) * q / 100.0
    lo = int(math.floor(pos))
    hi = min(lo + 1, len(v) - 1)
    return v[lo] + (v[hi] - v[lo]) * (pos - lo)


def stage_percentiles(per_step):
    """{stage: {p50, p95, p99, min, max}} over the timed steps' event times (ms)."""
    return {n: {"p50": percentile([x[n] for x in per_step], 50),
                "p95": percentile([x[n] for x in per_step], 95),
                "p99": percentile([x[n] for x in per_step], 99),
                "min": min(x[n] for x in per_step), "max": max(x[n] for x in per_step)}
            for n in Stages.NAMES}


def run_step(pipeline, capi, buf, inp, stages=None):
    d = buf.dims
    ev = stages.ev if stages else None
    if ev: ev[0].record()
    capi.msa_index_score_maxpool(d, inp["q_idx"], inp["k_idx"], buf.pooled, buf.pooled_stride,
                                 buf.dev_err)
    if ev: ev[1].record()
    capi.msa_topk_blocks(d, buf.pooled, buf.pooled_stride, buf.sel, buf.dev_err)
    if ev: ev[2].record()
    capi.msa_build_block_query_lists(d, buf.sel, buf.blk_offsets, buf.entries, buf.entry_pos,
                                     buf.ws, buf.dev_err)
    if ev: ev[3].record()
    fwd = capi.msa_sparse_attn_fwd_compact if buf.compact else capi.msa_sparse_attn_fwd
    merge = capi.msa_merge_partials_compact if buf.compact else capi.msa_merge_partials
    fwd(d, inp["q"], inp["k"], inp["v"], buf.blk_offsets, buf.entries, buf.part_ml, buf.part_acc,
        buf.dev_err)
    if ev: ev[4].record()
    merge(d, buf.entry_pos, buf.part_ml, buf.part_acc, buf.out, buf.lse, buf.dev_err)
    if ev: ev[5].record()


def pipeline_launches():
    from block_sparse_attention_32_b200 import pipeline
    return pipeline.LAUNCHES_PER_STEP


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """The maximum of a per-rank float over all ranks (the job's time)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, ms_local, world):
    """Whole-job throughput: units of all ranks / the slowest rank's time."""
    ms = max_over_ranks(ms_local, world)
    return world * units_per_rank / (ms / 1000.0), ms


def bench_workload(w, steps, warmup, world, rank, with_e2e=True, compact=False):
    from block_sparse_attention_32_b200 import capi, pipeline, workloads as wl
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d, compact=compact)
    inp = wl.make_inputs(w, "cuda")
    torch.cuda.synchronize()
    for _ in range(warmup):
        run_step(pipeline, capi, buf, inp)
    torch.cuda.synchronize()
    if int(buf.dev_err[0]) != 0:
        raise RuntimeError(f"device error {int(buf.dev_err[0])} during warm-up")

    stages = [Stages() for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    for s in range(steps):
        run_step(pipeline, capi, buf, inp, stages[s])
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    total_ms = start.elapsed_time(end)
    per_step = [st.ms() for st in stages]
    per_stage = stage_percentiles(per_step)
    per_stage_mean = {n: sum(x[n] for x in per_step) / steps for n in Stages.NAMES}
    if int(buf.dev_err[0]) != 0:
        raise RuntimeError(f"device error {int(buf.dev_err[0])} during timing")

    # (batch, group, block) segments that some query selected: K/V tiles read
    n_pieces = int((buf.blk_offsets[1:] > buf.blk_offsets[:-1]).sum().item())
    e2e = None
    if with_e2e:
        e2e = bench_e2e(w, buf, inp, max(3, steps), world)
    del inp
    del buf
    torch.cuda.empty_cache()
    return total_ms, per_stage, per_stage_mean, e2e, n_pieces


def bench_e4m3(w, reps=3):
    """The 8-bit index branch on the workload: time of quantisation + scores +
    top-k against the bf16 selection step, and how many (query, group) sets
    and selected blocks the two selections share."""
    from block_sparse_attention_32_b200 import pipeline, workloads as wl
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda", with_qkv=False)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    pipeline.select(buf, inp["q_idx"], inp["k_idx"])
    pipeline.select_e4m3(buf, inp["q_idx"], inp["k_idx"])
    torch.cuda.synchronize()
    ev[0].record()
    for _ in range(reps):
        pipeline.select(buf, inp["q_idx"], inp["k_idx"])
    ev[1].record()
    sel16 = buf.sel.clone()
    ev[2].record()
    for _ in range(reps):
        pipeline.select_e4m3(buf, inp["q_idx"], inp["k_idx"])
    ev[3].record()
    torch.cuda.synchronize()
    if int(buf.dev_err[0]) != 0:
        raise RuntimeError(f"device error {int(buf.dev_err[0])} in the e4m3 measurement")
    sel8 = buf.sel
    same_sets = float((sel8 == sel16).all(dim=-1).float().mean())
    # blocks of the 8-bit set that the bf16 set also holds (both ascending, -1 padded)
    valid = sel16 >= 0
    hits = (sel8.unsqueeze(-1) == sel16.unsqueeze(-2)).any(dim=-1) & (sel8 >= 0)
    shared = float(hits.sum()) / float(valid.sum())
    ms16 = ev[0].elapsed_time(ev[1]) / reps
    ms8 = ev[2].elapsed_time(ev[3]) / reps
    idx_flops, _, _ = work_counts(w)
    del buf, inp
    torch.cuda.empty_cache()
    return {"select_ms_bf16": ms16, "select_ms_e4m3": ms8, "speedup": ms16 / ms8,
            "identical_sets": same_sets, "shared_blocks": shared,
            "index_tflops_e4m3_incl_quant_and_topk": idx_flops / (ms8 / 1000.0) / 1e12}


def bench_recall(w, n_rows=64, reps=3):
    """Selection recall and KL alignment target on n_rows sampled rows of the
    workload (the next scoped measurement): mean recall / KL and the kernel time,
    and the bytes it streams into shared memory (every causal K and k_idx block of
    each (row, group), mostly L2 hits since rows share blocks)."""
    from block_sparse_attention_32_b200 import pipeline, workloads as wl
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    pipeline.select(buf, inp["q_idx"], inp["k_idx"])
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(w.batch * w.n_q, size=n_rows, replace=False)).astype(np.int64)
    rows_d = torch.from_numpy(rows).cuda()
    args = (buf, inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], rows_d)
    pipeline.selection_recall(*args)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(reps):
        mass, rec, kpq, kqp = pipeline.selection_recall(*args)
    ev[1].record()
    torch.cuda.synchronize()
    if int(buf.dev_err[0]) != 0:
        raise RuntimeError(f"device error {int(buf.dev_err[0])} in the recall measurement")
    ms = ev[0].elapsed_time(ev[1]) / reps
    # token-level selection at the same key budget (2048 = 16 x 128) on the same
    # rows: its captured share of each head's full attention mass,
    # exp(lse_tokens - lse_full), against the block selection's recall
    lse_full = torch.empty((n_rows, w.h_q), dtype=torch.float32, device="cuda")
    pipeline.selection_recall(*args, lse_full=lse_full)
    targs = (d, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], rows_d, 2048,
             buf.dev_err)
    pipeline.token_select_attention(*targs)
    torch.cuda.synchronize()
    ev[0].record()
    for _ in range(reps):
        _, _, lse_tok = pipeline.token_select_attention(*targs)
    ev[1].record()
    torch.cuda.synchronize()
    if int(buf.dev_err[0]) != 0:
        raise RuntimeError(f"device error {int(buf.dev_err[0])} in the token-level measurement")
    ms_tok = ev[0].elapsed_time(ev[1]) / reps
    tok_share = torch.exp(lse_tok.double() - lse_full.double())          # [n, H]
    tok_rec = tok_share.view(n_rows, w.h_kv, -1).mean(dim=2)             # [n, G]
    token_level = {"budget_tokens": 2048, "mean_recall": float(tok_rec.mean()),
                   "min_recall": float(tok_rec.min()),
                   "block_min_recall": float(rec.min()),
                   "units_token_above_block": float((tok_rec > rec.double()).float().mean()),
                   "ms": ms_tok}
    # every (row, group) streams its causal K and k_idx blocks into shared memory;
    # rows of one batch share those blocks, so DRAM sees each at most once
    nb = (w.q_pos0 + rows % w.n_q) // 128 + 1
    streamed = float(nb.sum()) * w.h_kv * (128 * 128 * 2 + 128 * w.d_idx * 2)
    # token level: each (row, group) streams its causal k_idx blocks for the scores
    # and gathers the K and V rows of its min(2048, t + 1) tokens
    ntok = np.minimum(2048, w.q_pos0 + rows % w.n_q + 1)
    tok_streamed = float(w.h_kv * (nb.sum() * 128 * w.d_idx * 2 + ntok.sum() * 512))
    token_level["streamed_bytes"] = tok_streamed
    token_level["streamed_gbs"] = tok_streamed / (ms_tok / 1000.0) / 1e9
    blocks = int(nb.max())
    unique = float(w.batch * blocks * 128 * (w.h_kv * 128 * 2 + w.h_kidx * w.d_idx * 2))
    out = {"rows": n_rows, "mean_recall": float(rec.mean()),
           "mean_kl_teacher_student": float(kpq.mean()),
           "mean_kl_student_teacher": float(kqp.mean()), "ms": ms,
           "streamed_bytes": streamed, "streamed_gbs": streamed / (ms / 1000.0) / 1e9,
           "dram_bytes_at_most": unique, "token_level": token_level}
    del buf, inp
    torch.cuda.empty_cache()
    return out


def attention_roofline(w, stage_mean, attn_flops, n_ent, n_pieces, nbytes, peaks, peak_src,
                       compact=False):
    """Roofline of the KV-block-outer attention (A4) on the basis the scope
    table fixes: a dense bf16 contraction, so tensor-bound, achieved =
    selected-token FLOPs / its mean event time against the sustained bf16 peak
    (it runs inside a long step).  Beside it: the same over attention + merge,
    the algorithmic bytes (Q read once, the selected K/V blocks once, O written
    once), the measured DRAM traffic per launch when the committed ncu record
    matches the current sources, and the design's own byte model (gathered Q
    rows, fp32 pieces, K/V per segment) as an HBM fraction."""
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK["bf16_tflops_sustained"])
    burst = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
    secs = stage_mean["attn"] / 1000.0
    secs_m = (stage_mean["attn"] + stage_mean["merge"]) / 1000.0
    ach = attn_flops / secs / 1e12
    ach_m = attn_flops / secs_m / 1e12
    qo = float(w.batch * w.n_q * w.h_q * 128 * 2)
    algo = 2 * qo + float(n_pieces) * 65536
    # counters of the fp32-piece kernel on the 8K profiling case, scaled by entries
    traffic = None if compact else measured_traffic(
        ["sparse_attn.cu", "common.cuh"], "sparse_attn_fwd_profile_8k_r8.md", n_ent)
    return {"bound": "tensor", "achieved": ach, "peak": sustained, "unit": "TFLOP/s",
            "frac": ach / sustained, "frac_of_burst": ach / burst,
            "peak_source": f"{peak_src} bf16_tflops_sustained",
            "with_merge": {"achieved": ach_m, "frac": ach_m / sustained},
            "algorithmic_flops": attn_flops,
            "algorithmic_bytes": algo,
            "traffic": traffic,
            "traffic_over_algorithmic": (traffic / algo) if traffic else None,
            "design_bytes": nbytes["attn"],
            "design_bytes_hbm_frac": nbytes["attn"] / secs / 1e9 / hbm,
            "merge_bytes": nbytes["merge"],
            "merge_hbm_frac": nbytes["merge"] / (stage_mean["merge"] / 1000.0) / 1e9 / hbm}


def bench_compact(w, steps, warmup, peaks, peak_src):
    """The same pass with compact pieces (acc / l in bf16, fp32 m and l; an
    opt-in of the library): queries/s, stage times and the attention's
    roofline, with the piece bytes of this format in the design byte model."""
    total_ms, pct, mean, _, n_pieces = bench_workload(w, steps, warmup, 1, 0, with_e2e=False,
                                                      compact=True)
    idx_flops, attn_flops, n_ent = work_counts(w)
    nbytes = bytes_model(w, n_ent, n_pieces, piece_bytes=264)
    roof = attention_roofline(w, mean, attn_flops, n_ent, n_pieces, nbytes, peaks, peak_src,
                              compact=True)
    roof["traffic"] = None
    roof["traffic_over_algorithmic"] = None
    ms = total_ms / steps
    return {"workload": w.name, "pieces": "bf16 acc / l + fp32 (m, l): 264 B per (query, head, block)",
            "queries_per_s": w.batch * w.n_q / (ms / 1000.0), "ms_per_step": ms, "steps": steps,
            "stages_ms": mean, "stages_ms_pct": pct, "attention_roofline": roof,
            "selected_token_attn_tflops": attn_flops / (mean["attn"] / 1000.0) / 1e12,
            "selected_token_attn_merge_tflops":
                attn_flops / ((mean["attn"] + mean["merge"]) / 1000.0) / 1e12}


def bench_config(w, steps, warmup, peaks, with_cpu=True):
    """One more configuration of the pages' long-context workloads timed the
    same way as the headline pass (device-resident inputs, events between the
    five calls): queries/s, per-stage times with percentiles, the index and
    attention contractions against the bf16 peaks, and the CPU oracle's
    queries/s on a bounded sample of the same rows (about 4 s)."""
    total_ms, pct, mean, _, n_pieces = bench_workload(w, steps, warmup, 1, 0, with_e2e=False)
    idx_flops, attn_flops, n_ent = work_counts(w)
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK["bf16_tflops_sustained"])
    burst = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    ms = total_ms / steps
    idx_t = idx_flops / (mean["index"] / 1000.0) / 1e12
    attn_t = attn_flops / (mean["attn"] / 1000.0) / 1e12
    out = {"workload": w.name, "queries_per_s": w.batch * w.n_q / (ms / 1000.0),
           "ms_per_step": ms, "steps": steps, "stages_ms": mean, "stages_ms_pct": pct,
           "index": {"tflops": idx_t, "frac_sustained": idx_t / sustained,
                     "frac_burst": idx_t / burst, "algorithmic_flops": idx_flops},
           "attn": {"tflops": attn_t, "frac_sustained": attn_t / sustained,
                    "algorithmic_flops": attn_flops, "entries": n_ent}}
    if with_cpu:
        out["cpu_baseline"] = CpuOracleSample(w, target_s=4.0).run()
    torch.cuda.empty_cache()
    return out


def bwd_bytes_model(w, n_entries, n_pieces):
    """Algorithmic DRAM bytes of one backward call: per gathered row (entry x
    head) the Q and dO rows (512 B), its lse and D (8 B), its fp32 dq piece
    written and read back by the slot reduction (2 x 512 B); per (query, head)
    o and dO for D (512 B), D (4 B) and dq (512 B); per selected (batch, group,
    block) segment the 64 KB K/V tile; dk and dv written once (fp32); the
    entry list."""
    R = w.h_q // w.h_kv
    rows = n_entries * R
    qh = w.batch * w.n_q * w.h_q
    return float(rows * (512 + 8 + 1024) + qh * (512 + 4 + 512) + n_pieces * 65536
                 + 2 * w.batch * w.h_kv * w.n_kv * 512 + 4 * n_entries)


def bench_backward(w, attn_flops, n_entries, peaks, reps=3):
    """The attention's backward (dq, dk, dv for a seeded upstream gradient,
    selection fixed by the forward) on the workload: its time, TFLOP/s over
    the five products per (row, head, selected causal token) -- S, dP, dV, dK
    and dQ, 2.5x the forward's two -- and its algorithmic bytes against the
    measured HBM bandwidth (the bound at these sizes)."""
    from block_sparse_attention_32_b200 import pipeline, workloads as wl
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    grads = pipeline.Grads.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    d_out = wl.upstream_grad(w, "cuda")
    pipeline.forward(buf, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"])
    args = (buf, grads, inp["q"], inp["k"], inp["v"], d_out)
    pipeline.backward(*args)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(reps):
        pipeline.backward(*args)
    ev[1].record()
    torch.cuda.synchronize()
    if int(buf.dev_err[0]) != 0:
        raise RuntimeError(f"device error {int(buf.dev_err[0])} in the backward measurement")
    ms = ev[0].elapsed_time(ev[1]) / reps
    flops = 2.5 * attn_flops
    n_pieces = int((buf.blk_offsets[1:] > buf.blk_offsets[:-1]).sum().item())
    nbytes = bwd_bytes_model(w, n_entries, n_pieces)
    hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK["bf16_tflops_sustained"])
    tflops = flops / (ms / 1000.0) / 1e12
    gbs = nbytes / (ms / 1000.0) / 1e9
    out = {"workload": w.name, "ms": ms, "tflops": tflops, "algorithmic_flops": flops,
           "bound": "hbm" if nbytes / hbm / 1e9 > flops / sustained / 1e12 else "tensor",
           "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "hbm_frac": gbs / hbm,
           "tensor_frac": tflops / sustained,
           "kernels": "tcgen05 kind::f16 (bf16, fp32 accumulate in TMEM)"}
    del buf, grads, inp, d_out
    torch.cuda.empty_cache()
    return out


def bench_e2e(w, buf, dev_inp, steps, world):
    """The pass through the public API with host buffers: every step uploads its
    inputs from pinned host memory, runs the five calls and downloads the output
    and lse (pipeline.HostPipeline: uploads and downloads of neighbouring steps
    overlap the kernels of the current one), all inside the timed region."""
    from block_sparse_attention_32_b200 import pipeline
    host = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in dev_inp.items()}
    for k, v in dev_inp.items():
        host[k].copy_(v)
    out_h = torch.empty(buf.out.shape, dtype=buf.out.dtype, pin_memory=True)
    lse_h = torch.empty(buf.lse.shape, dtype=buf.lse.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
    runner = pipeline.HostPipeline(buf, dev_inp)
    runner.run([host], [(out_h, lse_h)])            # warm-up of the streams and buffers
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start.record()
    runner.run([host] * steps, [(out_h, lse_h)] * steps)
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / steps, world)
    del runner
    return {"ms_per_step": ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


class CpuOracleSample:
    """The oracle, as it stands, on a bounded sample of the workload's query rows.

    The sample size is calibrated so that one run() takes about `target_s`
    seconds on this host: a first pass over one row per core measures the
    per-row cost, then the row count is fixed for every later run().
    """

    def __init__(self, w, target_s=15.0, seed=0):
        import oracle
        from block_sparse_attention_32_b200 import workloads as wl
        self.oracle, self.w = oracle, w
        inp = wl.make_inputs(w, "cpu")
        bits = oracle.bf16_bits
        self.k, self.v, self.ki = bits(inp["k"]), bits(inp["v"]), bits(inp["k_idx"])
        self.q_all, self.qi_all = inp["q"][0], inp["q_idx"][0]
        self.cores = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
        self.rng = np.random.default_rng(seed)
        self._pick(min(self.cores, w.n_q))
        t0 = time.perf_counter()
        self._forward()
        per_row = (time.perf_counter() - t0) / len(self.rows)
        n = int(max(self.cores, min(w.n_q, target_s / max(per_row, 1e-9))))
        self._pick(n)

    def _pick(self, n):
        w = self.w
        self.rows = np.sort(self.rng.choice(w.n_q, size=n, replace=False)).astype(np.int64)
        bits = self.oracle.bf16_bits
        self.q_rows = bits(self.q_all[self.rows])
        self.qi_rows = bits(self.qi_all[self.rows])
        self.pos = w.q_pos0 + self.rows
        self.bat = np.zeros_like(self.rows)

    def _forward(self):
        _, self.sel, _, _ = self.oracle.forward_rows(self.q_rows, self.qi_rows, self.pos, self.bat,
                                                     self.k, self.v, self.ki, self.w.scale)

    def run_next_rows(self, n=None):
        """The oracle on the first n sampled rows for the selection-recall
        measurement and the token-level variant (rows/s, beside the GPU's)."""
        n = min(len(self.rows), n or 2 * self.cores)
        sl = slice(0, n)
        args = (self.q_rows[sl], self.qi_rows[sl], self.pos[sl], self.bat[sl])
        t0 = time.perf_counter()
        self.oracle.selection_recall(*args, self.k, self.ki, self.sel[sl], self.w.scale)
        t1 = time.perf_counter()
        self.oracle.token_select_attention(*args, self.k, self.v, self.ki, self.w.scale, budget=2048)
        t2 = time.perf_counter()
        desc = f"{n} of the sampled rows of {self.w.name}, all groups, fp64, {self.cores} threads"
        return ({"value": n / (t1 - t0), "unit": "rows/s", "cores": self.cores, "kind": "oracle",
                 "sample": desc},
                {"value": n / (t2 - t1), "unit": "rows/s", "cores": self.cores, "kind": "oracle",
                 "sample": desc})

    def run(self):
        t0 = time.perf_counter()
        self._forward()
        dt = time.perf_counter() - t0
        w = self.w
        return {"value": len(self.rows) / dt, "unit": "queries/s", "cores": self.cores,
                "kind": "oracle",
                "sample": f"{len(self.rows)} random query rows of {w.name} (all {w.h_kv} groups, "
                          f"{w.h_q} heads): fp64 index scores + selection + attention; "
                          f"{dt:.1f} s"}


def cpu_baseline(w, target_s=15.0):
    sample = CpuOracleSample(w, target_s)
    return sample.run(), sample


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-recall", action="store_true")
    ap.add_argument("--no-e4m3", action="store_true")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--no-compact", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from block_sparse_attention_32_b200 import workloads as wl
    w = wl.P128
    idx_flops, attn_flops, n_ent = work_counts(w)
    peaks, peak_src = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return
        sample = CpuOracleSample(w, target_s=6.0)
        vals = []
        for _ in range(args.warmup):
            sample.run()
        for _ in range(args.steps):
            vals.append(sample.run())
        v = statistics.median(x["value"] for x in vals)
        line = {"impl": "reference", "metric": "prefill_128k_queries_per_s", "value": v,
                "unit": "queries/s", "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1000.0 * len(sample.rows) / v, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, "batch": w.batch, "seq_len": w.n_kv,
                           "h_q": w.h_q, "h_kv": w.h_kv, "d_idx": w.d_idx, "topk_blocks": 16,
                           "block": 128},
                "cpu_baseline": dict(vals[-1], value=v),
                "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local),
                                             timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    import __graft_entry__
    __graft_entry__.build()

    clk_path = os.path.join(tempfile.gettempdir(), f"msa_bench_clocks_{os.getpid()}.csv")
    proc = sample_clocks(None, clk_path) if rank == 0 else None
    total_ms, stage_pct, stage_mean, e2e, n_pieces = bench_workload(w, args.steps, args.warmup,
                                                                    world, rank)
    if proc is not None:
        proc.terminate()
        proc.wait()
    clocks = summarize_clocks(clk_path, local) if rank == 0 else None

    qps, ms_step = job_throughput(w.n_q, total_ms / args.steps, world)

    decode = None
    if not args.no_decode:
        dw = wl.DECODE
        dsteps = max(3, args.steps)
        dms, dpct, dmean, _, dpieces = bench_workload(dw, dsteps, args.warmup, world, rank,
                                                      with_e2e=False)
        dtps, dms = job_throughput(dw.batch, dms / dsteps, world)
        kidx_bytes = dw.batch * dw.n_kv * dw.d_idx * 2
        sel_kv_bytes = dpieces * 65536
        read_bytes = kidx_bytes + sel_kv_bytes
        decode = {"workload": dw.name, "tokens_per_s": dtps,
                  "ms_per_step": dms, "stages_ms": dmean, "stages_ms_pct": dpct,
                  "index_scan_gbs": kidx_bytes / (dmean["index"] / 1000.0) / 1e9,
                  "bytes_read_per_step": read_bytes,
                  "hbm_frac_on_bytes_read": read_bytes / (dms / 1000.0) / 1e9
                  / peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])}

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    # the side measurements and the CPU baseline run on a single-GPU run only: with
    # N > 1 every GPU of the job would stay held while rank 0 alone works
    single = world == 1

    def side(enabled, fn):
        # a side measurement that fails is reported in its own key; the headline
        # measurement above is already complete
        if not (single and enabled):
            return None
        try:
            return fn()
        except Exception as exc:  # noqa: BLE001 -- any failure of a side measurement
            print(f"bench: side measurement failed: {exc!r}", file=sys.stderr)
            torch.cuda.empty_cache()
            return {"error": repr(exc)}

    recall = side(not args.no_recall, lambda: bench_recall(w))
    e4m3 = side(not args.no_e4m3, lambda: bench_e4m3(w))
    backward = side(not args.no_bwd, lambda: bench_backward(w, attn_flops, n_ent, peaks))
    compact = side(not args.no_compact,
                   lambda: bench_compact(w, max(3, args.steps // 2), args.warmup, peaks,
                                         peak_src))
    configs = side(not args.no_configs,
                   lambda: {c.name: bench_config(c, max(3, args.steps // 2), args.warmup, peaks,
                                                 with_cpu=not args.no_cpu)
                            for c in (wl.P32, wl.M1)})

    sustained = peaks.get("bf16_tflops_sustained", FALLBACK["bf16_tflops_sustained"])
    burst = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
    nbytes = bytes_model(w, n_ent, n_pieces)
    attn_roof = attention_roofline(w, stage_mean, attn_flops, n_ent, n_pieces, nbytes, peaks,
                                   peak_src)
    # dominant kernel: the longest stage.  Index scoring and the attention are
    # dense bf16 contractions (tensor-bound by the algorithmic work: the FLOPs
    # of the selected tokens); the other stages are HBM-bound on the bytes they must move.
    dom = max(stage_mean, key=stage_mean.get)
    if dom == "attn":
        roof = dict(attn_roof)
        roof["kernel"] = "attn"
    elif dom == "index":
        secs = stage_mean["index"] / 1000.0
        ach = idx_flops / secs / 1e12
        roof = {"kernel": "index", "bound": "tensor", "achieved": ach, "peak": sustained,
                "unit": "TFLOP/s", "frac": ach / sustained,
                "peak_source": f"{peak_src} bf16_tflops_sustained",
                "frac_of_burst": ach / burst, "traffic": None}
    else:
        secs = stage_mean[dom] / 1000.0
        ach = nbytes[dom] / secs / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                "frac": ach / hbm, "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic_bytes": nbytes[dom], "traffic": None}

    attn_tflops = attn_flops / (stage_mean["attn"] / 1000.0) / 1e12
    attn_merge_tflops = attn_flops / ((stage_mean["attn"] + stage_mean["merge"]) / 1000.0) / 1e12
    line = {
        "metric": "prefill_128k_queries_per_s", "value": qps, "unit": "queries/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.n_kv, "h_q": w.h_q,
                   "h_kv": w.h_kv, "d_idx": w.d_idx, "topk_blocks": 16, "block": 128,
                   "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (partials 69 GB per pass)"},
        "selected_token_attn_tflops": attn_tflops,
        "selected_token_attn_merge_tflops": attn_merge_tflops,
        "index_tflops": idx_flops / (stage_mean["index"] / 1000.0) / 1e12,
        "stages_ms": stage_mean,
        "stages_ms_pct": stage_pct,
        "stage_conditions": {"steps": args.steps, "stream": "one stream, events between calls",
                             "sm_mhz_median": clocks["sm_mhz"] if clocks else None,
                             "reasons": clocks["reasons"] if clocks else None},
        "attention_roofline": attn_roof,
        "compact_pieces": compact,
        "decode": decode,
        "configs": configs,
        "selection_recall": recall,
        "index_e4m3": e4m3,
        "backward": backward,
        "roofline": roof,
        "clocks": clocks,
        "gpu_launches": args.steps * sum(pipeline_launches().values()),
        "e2e": {"value": world * w.n_q / (e2e["ms_per_step"] / 1000.0), "unit": "queries/s",
                "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                "d2h_bytes_per_step": e2e["d2h_bytes_per_step"]} if e2e else None,
    }
    if single and not args.no_cpu:
        line["cpu_baseline"], sample = cpu_baseline(w)
        if recall is not None and "error" not in recall:
            rec_cpu, tok_cpu = sample.run_next_rows()
            recall["cpu_oracle"] = rec_cpu
            recall["token_level"]["cpu_oracle"] = tok_cpu
            recall["rows_per_s"] = recall["rows"] / (recall["ms"] / 1000.0)
            recall["token_level"]["rows_per_s"] = recall["rows"] / (recall["token_level"]["ms"]
                                                                   / 1000.0)
    print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
