"""Shared helpers of the GPU parity tests: comparisons against the oracle.

Tolerances (the bar stated for this path):
  * pooled block scores: |gpu - oracle| <= 1e-5 * max_j sum_k |q_k k_jk| over
    the block's tokens (fp32 accumulation of exact bf16 products);
  * selected block sets: bit-exact, except rows whose oracle 15th and 16th
    best candidate scores differ by < 1e-5 relative ("near-ties"), which are
    counted and must still pass the selection certificate;
  * attention output (bf16 vs fp64): max-abs <= 2e-2 and mean-abs <= 2e-3,
    per-row relative L2 error <= 2^-7, lse within 1e-4;
  * near-tie rows: the GPU's set must be one of the correct selections the
    oracle's own scores allow (every candidate above the tie band kept,
    nothing below it); the oracle then evaluates the attention on that set
    and the row's output is held to the same bars.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

POOLED_REL = 1e-5
NEAR_TIE_REL = 1e-5
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
# Per-row relative error ||o - o_ref|| / ||o_ref|| (L2 over the row's 128
# outputs).  The bf16 output alone rounds every element by up to 2^-9 of its
# magnitude; the weights rounded to bf16 for P.V add at most 2^-9 of sum_j p_j |v_j|,
# which for the near-flat rows of N(0,1) inputs is ~30x |o| but averages out over the
# 2048 keys (random signs), to ~2^-9 of |o| again.  2^-7 leaves 2x headroom over
# the sum of the two.
OUT_REL_L2 = 2.0 ** -7
# lse = M + ln L in fp32.  M is a scaled logit summed in fp32 from exact bf16
# products (error ~1e-6 of |M| <= ~20 here) and L sums fp32 weights from ex2.approx
# (relative error ~2^-22 each), so |lse error| stays near 1e-5; 1e-4 is the bar
# (a dropped or doubled own-block token moves lse by ~1/2048 = 5e-4 or more).
LSE_MAX_ABS = 1e-4
BLOCK = 128


def bits(t: torch.Tensor) -> np.ndarray:
    return oracle.bf16_bits(t)


def pooled_tolerance(q_idx_rows_bits, k_idx_bits, row_pos, row_batch, h_kidx):
    """1e-5 * max over the block's tokens of sum_k |q_k k_jk|, per (row, g, block)."""
    qa = np.abs(oracle.bits_to_f64(q_idx_rows_bits))      # [n, G, d]
    ka = np.abs(oracle.bits_to_f64(k_idx_bits))           # [B, hk, n_kv, d]
    n, G, _ = qa.shape
    n_kv = ka.shape[2]
    nblk = (n_kv + BLOCK - 1) // BLOCK
    pad = nblk * BLOCK - n_kv
    out = np.zeros((n, G, nblk))
    for r in range(n):
        if h_kidx == 1:
            s = ka[row_batch[r], 0] @ qa[r].T                 # [n_kv, G]
            s = np.concatenate([s, np.zeros((pad, G))])
            out[r] = s.reshape(nblk, BLOCK, G).max(axis=1).T
        else:
            for g in range(G):
                s = ka[row_batch[r], g] @ qa[r, g]
                s = np.concatenate([s, np.zeros(pad)])
                out[r, g] = s.reshape(nblk, BLOCK).max(axis=1)
    return POOLED_REL * out


def compare_pooled(gpu_pooled, ora_pooled, tol, row_pos):
    """gpu_pooled / ora_pooled: [n, G, >=nblk]; returns max |diff| / tol."""
    worst = 0.0
    n, G = ora_pooled.shape[:2]
    for r in range(n):
        own = row_pos[r] // BLOCK
        if own == 0:
            continue
        d = np.abs(gpu_pooled[r, :, :own].astype(np.float64) - ora_pooled[r, :, :own])
        ratio = d / np.maximum(tol[r, :, :own], 1e-30)
        worst = max(worst, float(ratio.max()))
    return worst


def near_tie_rows(ora_pooled, row_pos):
    """Boolean [n, G]: oracle's last-kept and first-dropped candidates nearly tie."""
    n, G = ora_pooled.shape[:2]
    out = np.zeros((n, G), bool)
    for r in range(n):
        own = row_pos[r] // BLOCK
        if own < 16:
            continue
        for g in range(G):
            s = np.sort(ora_pooled[r, g, :own])[::-1]
            a, b = s[14], s[15]
            if abs(a - b) < NEAR_TIE_REL * max(abs(a), abs(b), 1e-300):
                out[r, g] = True
    return out


def certificate_ok(scores, own, sel_row, rel=NEAR_TIE_REL):
    """Selection invariants and optimality (within `rel`) under oracle scores."""
    chosen = [int(c) for c in sel_row if c >= 0]
    nsel = min(16, own + 1)
    if len(chosen) != nsel or chosen != sorted(set(chosen)) or own not in chosen:
        return False
    if any(c > own for c in chosen) or any(c != -1 for c in sel_row[nsel:]):
        return False
    picked = [c for c in chosen if c != own]
    rejected = [c for c in range(own) if c not in picked]
    if not picked or not rejected:
        return True
    lo = min(scores[c] for c in picked)
    hi = max(scores[c] for c in rejected)
    return hi <= lo + rel * max(abs(lo), abs(hi))


def tie_band_ok(scores, own, sel_row, rel=NEAR_TIE_REL):
    """True when sel_row is one of the correct selections under near-tied
    oracle scores: the oracle's boundary pair (last kept a, first dropped b)
    spans the band [b - tol, a + tol], tol = rel * max(|a|, |b|); every
    candidate scoring above the band is kept, none below it, and the count,
    order, padding and own block are right."""
    nsel = min(16, own + 1)
    chosen = [int(c) for c in sel_row if c >= 0]
    if len(chosen) != nsel or chosen != sorted(set(chosen)) or own not in chosen:
        return False
    if any(c > own for c in chosen) or any(c != -1 for c in sel_row[nsel:]):
        return False
    if own < 16:
        return chosen == list(range(own + 1))
    order = sorted(range(own), key=lambda c: (-scores[c], c))
    a, b = scores[order[14]], scores[order[15]]
    tol = rel * max(abs(a), abs(b))
    picked = set(chosen) - {own}
    for c in range(own):
        if scores[c] > a + tol and c not in picked:
            return False
        if scores[c] < b - tol and c in picked:
            return False
    return True


def compare_sets(gpu_sel, ora_sel, ora_pooled, row_pos):
    """Set comparison with near-tie accounting.

    Returns (n_mismatch_outside_ties, n_near_ties, n_bad_tie_sets, eval_sel):
    eval_sel [n, G, 16] is the selection the oracle's attention is evaluated
    on -- the oracle's own set, or for a near-tie (row, group) where the GPU
    chose differently, the GPU's set once tie_band_ok has shown from the
    oracle's scores that it is one of the correct selections."""
    ties = near_tie_rows(ora_pooled, row_pos)
    n, G = ora_sel.shape[:2]
    bad, bad_tie = 0, 0
    eval_sel = np.array(ora_sel, copy=True)
    for r in range(n):
        own = row_pos[r] // BLOCK
        for g in range(G):
            if (gpu_sel[r, g] == ora_sel[r, g]).all():
                continue
            if ties[r, g]:
                if tie_band_ok(ora_pooled[r, g], own, list(gpu_sel[r, g])):
                    eval_sel[r, g] = gpu_sel[r, g]
                else:
                    bad_tie += 1
            else:
                bad += 1
    return bad, int(ties.sum()), bad_tie, eval_sel


def rows_to_recheck(eval_sel, ora_sel):
    """Row indices whose evaluation set differs from the oracle's own."""
    return np.nonzero((eval_sel != ora_sel).any(axis=(1, 2)))[0]


def compare_out(gpu_out, ora_out):
    d = np.abs(gpu_out.astype(np.float64) - ora_out)
    return float(d.max()), float(d.mean())


def compare_rows(gpu_out, gpu_lse, ora_out, ora_lse):
    """Output and lse errors over rows: dict with max / mean abs error, the
    worst per-row relative L2 error and the worst lse error."""
    d = np.abs(gpu_out.astype(np.float64) - ora_out)
    num = np.sqrt(((gpu_out.astype(np.float64) - ora_out) ** 2).sum(-1))
    den = np.maximum(np.sqrt((ora_out ** 2).sum(-1)), 1e-30)
    res = {"out_max": float(d.max()), "out_mean": float(d.mean()),
           "rel_l2": float((num / den).max())}
    if gpu_lse is not None:
        res["lse_max"] = float(np.abs(gpu_lse.astype(np.float64) - ora_lse).max())
    return res


def assert_rows_ok(res, what=""):
    assert res["out_max"] <= OUT_MAX_ABS and res["out_mean"] <= OUT_MEAN_ABS, (what, res)
    assert res["rel_l2"] <= OUT_REL_L2, (what, res)
    if "lse_max" in res:
        assert res["lse_max"] <= LSE_MAX_ABS, (what, res)


def compare_out(gpu_out, ora_out):
    d = np.abs(gpu_out.astype(np.float64) - ora_out)
    return float(d.max()), float(d.mean())


def sample_rows(n_q, q_pos0, k, seed=0, extra=()):
    """Stratified query indices: first/last, around the 16-block boundary, random."""
    rng = np.random.default_rng(seed)
    cand = {0, n_q - 1, n_q // 2}
    for t in (1920, 2047, 2048, 2049, 4095, 4096):
        i = t - q_pos0
        if 0 <= i < n_q:
            cand.add(i)
    cand.update(int(x) for x in extra if 0 <= x < n_q)
    while len(cand) < min(k, n_q):
        cand.add(int(rng.integers(0, n_q)))
    return np.array(sorted(cand), np.int64)


def scale_of(w):
    return 1.0 / math.sqrt(128)
