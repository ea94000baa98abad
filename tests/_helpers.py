"""Shared helpers of the GPU parity tests: comparisons against the oracle.

Tolerances (the bar stated for this path):
  * pooled block scores: |gpu - oracle| <= 1e-5 * max_j sum_k |q_k k_jk| over
    the block's tokens (fp32 accumulation of exact bf16 products);
  * selected block sets: bit-exact, except rows whose oracle 15th and 16th
    best candidate scores differ by < 1e-5 relative ("near-ties"), which are
    counted and must still pass the selection certificate;
  * attention output (bf16 vs fp64): max-abs <= 2e-2 and mean-abs <= 2e-3.
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
# The kernel sums the fp32 softmax weights into l and rounds them to bf16 only for
# the P.V product; l may still differ from the exact sum by the rounding of the
# bf16 logits' fp32 accumulation and of ex2.approx, far below the bf16 unit
# roundoff 2^-8 of a weight.  The bound log(1 + 2^-8) < 4e-3 covers even a
# normaliser built from bf16-rounded weights.
LSE_MAX_ABS = 4e-3
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


def compare_sets(gpu_sel, ora_sel, ora_pooled, row_pos):
    """Returns (n_mismatch_outside_ties, n_near_ties, n_bad_certificates, ok_mask [n])."""
    ties = near_tie_rows(ora_pooled, row_pos)
    n, G = ora_sel.shape[:2]
    bad, bad_cert = 0, 0
    ok = np.ones(n, bool)
    for r in range(n):
        own = row_pos[r] // BLOCK
        for g in range(G):
            same = (gpu_sel[r, g] == ora_sel[r, g]).all()
            if same:
                continue
            ok[r] = False
            if ties[r, g]:
                if not certificate_ok(ora_pooled[r, g], own, list(gpu_sel[r, g])):
                    bad_cert += 1
            else:
                bad += 1
    return bad, int(ties.sum()), bad_cert, ok


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
