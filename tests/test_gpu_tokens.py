"""Token-level selection at the same key budget on the GPU against the oracle.

The comparison the pages draw between selection granularities ("MSA 稀疏注意力
三国杀" page, section "分歧一：颗粒度——token 级还是块级？"; "稀疏注意力速览" page,
section 4): the top-`budget` keys by index score per (row, group), lower index
first among equal scores, and exact attention over them.

Bars:
  * token sets: bit-exact, except (row, group) units whose chosen and rejected
    keys come within 1e-5 * max_j sum_k |q_k k_jk| of each other under the
    oracle's fp64 scores (the kernel's fp32 accumulation of exact bf16
    products can order those either way); such units must still pass the
    selection certificate (size, order, causality, padding, optimality within
    that tolerance) and are left out of the output comparison;
  * out (fp32 from bf16 operands, weights rounded to bf16 for P.V, against
    fp64): max-abs <= 2e-2, mean-abs <= 2e-3; lse: <= 4e-3 absolute;
  * the full causal lse that msa_selection_recall now also writes: <= 1e-4
    absolute (fp32 sums of per-block log-masses).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_32_b200 import capi, pipeline, workloads as wl
from _helpers import LSE_MAX_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, bits, compare_out

pytestmark = pytest.mark.gpu

SCORE_REL = 1e-5

# (workload, budget, number of extra random rows)
CASES = [
    (wl.TINY, 2048, 6),
    (wl.small("tok_r8_batch2_unaligned", 2, 700, 3100, 2400, 16, 2, 128, seed=61, h_kidx=2),
     2048, 6),
    (wl.small("tok_decode", 3, 1, 4000, 3999, 32, 4, 128, seed=62), 2048, 3),
    (wl.small("tok_r1_budget100", 1, 1800, 1800, 0, 4, 4, 64, seed=63), 100, 8),
    (wl.small("tok_budget1", 1, 900, 900, 0, 8, 2, 64, seed=64), 1, 6),
    (wl.small("tok_budget_over_n", 1, 1000, 1000, 0, 8, 1, 128, seed=65), 4096, 6),
    (wl.small("tok_r2_planted", 1, 3000, 3000, 0, 8, 4, 128, seed=66, plants_per_group=2,
              plant_targets=64), 2048, 6),
]


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _sample_rows(w, extra, seed):
    rng = np.random.default_rng(seed)
    n_all = w.batch * w.n_q
    pick = rng.choice(n_all, size=min(extra, n_all), replace=False)
    return np.unique(np.concatenate([[0, n_all - 1], pick])).astype(np.int64)


def _scores_f64(qi_rows, k_idx_bits, pos, bat):
    """fp64 index scores and their tolerance per (row, group): lists of arrays."""
    ki = oracle.bits_to_f64(k_idx_bits)                    # [B, hk, n_kv, d]
    qa = oracle.bits_to_f64(qi_rows)                       # [n, G, d]
    n, G, _ = qa.shape
    sc, tol = [], []
    for r in range(n):
        row_s, row_t = [], []
        for g in range(G):
            kk = ki[bat[r], 0 if ki.shape[1] == 1 else g, : pos[r] + 1]
            row_s.append(kk @ qa[r, g])
            row_t.append(SCORE_REL * float((np.abs(kk) @ np.abs(qa[r, g])).max()))
        sc.append(row_s)
        tol.append(row_t)
    return sc, tol


def _certificate(scores, tol, gpu_row, budget, t):
    m = min(budget, t + 1)
    chosen = [int(x) for x in gpu_row[:m]]
    if any(x != -1 for x in gpu_row[m:]):
        return False
    if chosen != sorted(set(chosen)) or len(chosen) != m or chosen[0] < 0 or chosen[-1] > t:
        return False
    if m == t + 1:
        return True
    mask = np.zeros(t + 1, bool)
    mask[chosen] = True
    return scores[~mask].max() <= scores[mask].min() + tol


def _compare_tokens(gpu_tok, ora_tok, sc, tol, pos, budget):
    n, G, _ = ora_tok.shape
    bad, ties = 0, 0
    ok = np.ones(n, bool)
    for r in range(n):
        for g in range(G):
            if np.array_equal(gpu_tok[r, g], ora_tok[r, g]):
                continue
            ok[r] = False
            ties += 1
            if not _certificate(sc[r][g], tol[r][g], gpu_tok[r, g], budget, int(pos[r])):
                bad += 1
    return bad, ties, ok


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].name}-b{c[1]}")
def test_token_select_matches_oracle(case):
    _need_gpu()
    w, budget, extra = case
    d = pipeline.dims_for(w)
    inp = wl.make_inputs(w, "cuda")
    rows = _sample_rows(w, extra, w.seed + 1)
    rows_d = torch.from_numpy(rows).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, out, lse = pipeline.token_select_attention(d, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                                    inp["k_idx"], rows_d, budget, err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    b, qi = rows // w.n_q, rows % w.n_q
    pos = w.q_pos0 + qi
    q_rows = bits(inp["q"])[b, qi]
    qi_rows = bits(inp["q_idx"])[b, qi]
    e_tok, e_out, e_lse, _ = oracle.token_select_attention(
        q_rows, qi_rows, pos, b, bits(inp["k"]), bits(inp["v"]), bits(inp["k_idx"]), w.scale,
        budget=budget)
    g_tok = tok.cpu().numpy().astype(np.int64)
    sc, tol = _scores_f64(qi_rows, bits(inp["k_idx"]), pos, b)
    bad, ties, ok = _compare_tokens(g_tok, e_tok, sc, tol, pos, budget)
    assert bad == 0, (bad, ties)
    assert ok.sum() >= (len(rows) + 1) // 2, (ties, ok)
    mx, mean = compare_out(out.cpu().numpy()[ok], e_out[ok])
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (mx, mean)
    assert np.abs(lse.cpu().numpy()[ok] - e_lse[ok]).max() <= LSE_MAX_ABS


def test_token_select_full_size_rows():
    """Three rows of the 128K-token prefill workload (64 heads, 8 groups,
    d_idx 128) in the launch configuration the measurement uses."""
    _need_gpu()
    w = wl.P128
    d = pipeline.dims_for(w)
    inp = wl.make_inputs(w, "cuda")
    rows = np.array([5000, 77777, w.n_q - 1], np.int64)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, out, lse = pipeline.token_select_attention(d, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                                    inp["k_idx"], torch.from_numpy(rows).cuda(),
                                                    2048, err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    pos = w.q_pos0 + rows
    b = np.zeros_like(rows)
    q_rows = bits(inp["q"])[b, rows]
    qi_rows = bits(inp["q_idx"])[b, rows]
    kb, vb, kib = bits(inp["k"]), bits(inp["v"]), bits(inp["k_idx"])
    del inp
    torch.cuda.empty_cache()
    e_tok, e_out, e_lse, _ = oracle.token_select_attention(q_rows, qi_rows, pos, b, kb, vb, kib,
                                                           w.scale, budget=2048)
    sc, tol = _scores_f64(qi_rows, kib, pos, b)
    bad, ties, ok = _compare_tokens(tok.cpu().numpy().astype(np.int64), e_tok, sc, tol, pos, 2048)
    assert bad == 0, (bad, ties)
    assert ok.any()
    mx, mean = compare_out(out.cpu().numpy()[ok], e_out[ok])
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (mx, mean)
    assert np.abs(lse.cpu().numpy()[ok] - e_lse[ok]).max() <= LSE_MAX_ABS


@pytest.mark.parametrize("w", [wl.TINY, CASES[2][0]], ids=lambda w: w.name)
def test_recall_lse_full_matches_oracle(w):
    """msa_selection_recall's optional lse_full output: each head's full causal
    log-normaliser, against the oracle's."""
    _need_gpu()
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    pipeline.select(buf, inp["q_idx"], inp["k_idx"])
    rows = _sample_rows(w, 6, w.seed + 2)
    lse_full = torch.full((len(rows), w.h_q), float("nan"), device="cuda")
    pipeline.selection_recall(buf, inp["q"], inp["k"], inp["q_idx"], inp["k_idx"],
                              torch.from_numpy(rows).cuda(), lse_full=lse_full)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    b, qi = rows // w.n_q, rows % w.n_q
    _, _, _, e_full = oracle.token_select_attention(
        bits(inp["q"])[b, qi], bits(inp["q_idx"])[b, qi], w.q_pos0 + qi, b, bits(inp["k"]),
        bits(inp["v"]), bits(inp["k_idx"]), w.scale, budget=1)
    assert np.abs(lse_full.cpu().numpy() - e_full).max() <= 1e-4


def test_token_select_rejects_bad_arguments():
    _need_gpu()
    w = CASES[4][0]
    d = pipeline.dims_for(w)
    inp = wl.make_inputs(w, "cuda")
    rows = torch.zeros(2, dtype=torch.int64, device="cuda")
    tok = torch.empty((2, w.h_kv, 4), dtype=torch.int32, device="cuda")
    out = torch.empty((2, w.h_q, 128), device="cuda")
    lse = torch.empty((2, w.h_q), device="cuda")
    ws = torch.empty(capi.msa_token_select_workspace(d, 2) // 4 + 4, dtype=torch.int32,
                     device="cuda")
    with pytest.raises(capi.MSAError):                      # budget 0
        capi.msa_token_select_attention(d, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                        inp["k_idx"], rows, 0, tok, out, lse, ws)
    with pytest.raises(capi.MSAError):                      # workspace too small
        capi.msa_token_select_attention(d, inp["q"], inp["k"], inp["v"], inp["q_idx"],
                                        inp["k_idx"], rows, 4, tok, out, lse, ws[:4])


def test_token_select_bad_row_reported():
    """A sampled row outside [0, B * n_q) is reported on the device flag."""
    _need_gpu()
    w = CASES[4][0]
    d = pipeline.dims_for(w)
    inp = wl.make_inputs(w, "cuda")
    rows = torch.tensor([3, w.n_q + 5], dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pipeline.token_select_attention(d, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                                    rows, 8, err)
    torch.cuda.synchronize()
    assert int(err[0]) == 3                                  # MSA_DEVERR_BAD_ENTRY
