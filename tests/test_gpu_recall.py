"""Selection recall and KL alignment target on the GPU against the oracle.

The measurement ("MSA 稀疏注意力三国杀" page, section "索引分支训练：KL 对齐"):
the main branch's full causal attention mass per block is the teacher P, the
index branch's block softmax the student Q; recall is P's mass on the chosen
blocks.  Tolerances: the kernel forms each block's log-mass from fp32 sums of
exact bf16 products and ex2.approx (relative error ~1e-6 per block), so P is
within ~1e-5 relative of the fp64 oracle; block masses are checked to 5e-5
absolute, recall to 2e-4, the KL divergences to 2e-3 absolute + 1e-3 relative.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_32_b200 import pipeline, workloads as wl
from _helpers import compare_sets

pytestmark = pytest.mark.gpu

CASES = [
    wl.TINY,
    wl.small("recall_r8", 1, 2500, 2500, 0, 16, 2, 128, seed=51),
    wl.small("recall_batch2_unaligned", 2, 700, 3100, 2400, 8, 2, 64, seed=52, h_kidx=2),
    wl.small("recall_decode", 3, 1, 4000, 3999, 32, 4, 128, seed=53),
    wl.small("recall_r1", 1, 1800, 1800, 0, 4, 4, 128, seed=54, plants_per_group=2,
             plant_targets=64),
]


def _bits(t):
    return oracle.bf16_bits(t)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_selection_recall_matches_oracle(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    pipeline.select(buf, inp["q_idx"], inp["k_idx"])
    rng = np.random.default_rng(w.seed)
    n_all = w.batch * w.n_q
    rows = np.unique(np.concatenate([[0, n_all - 1], rng.choice(n_all, size=min(6, n_all),
                                                                 replace=False)])).astype(np.int64)
    rows_d = torch.from_numpy(rows).cuda()
    mass, rec, kpq, kqp = pipeline.selection_recall(buf, inp["q"], inp["k"], inp["q_idx"],
                                                    inp["k_idx"], rows_d)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    b = rows // w.n_q
    qi = rows % w.n_q
    pos = w.q_pos0 + qi
    q_rows = _bits(inp["q"])[b, qi]
    qi_rows = _bits(inp["q_idx"])[b, qi]
    # the oracle's own selection of these rows; where a near-tie let the GPU
    # choose another correct set, recall is evaluated on that set
    pooled = oracle.index_pooled(qi_rows, pos, b, _bits(inp["k_idx"]))
    sel = oracle.topk(pooled, pos)
    gpu_sel = buf.sel.cpu().numpy()[b, :, qi]                   # [n, G, 16]
    bad, ties, bad_tie, eval_sel = compare_sets(gpu_sel, sel, pooled, pos)
    assert bad == 0 and bad_tie == 0, (bad, ties, bad_tie)
    e_mass, e_rec, e_kpq, e_kqp = oracle.selection_recall(
        q_rows, qi_rows, pos, b, _bits(inp["k"]), _bits(inp["k_idx"]), eval_sel, w.scale,
        stride=mass.shape[2])
    g_mass = mass.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(g_mass, e_mass, atol=5e-5, rtol=1e-4)
    np.testing.assert_allclose(g_mass.sum(axis=2), 1.0, atol=1e-4)
    np.testing.assert_allclose(rec.cpu().numpy(), e_rec, atol=2e-4)
    np.testing.assert_allclose(kpq.cpu().numpy(), e_kpq, atol=2e-3, rtol=1e-3)
    np.testing.assert_allclose(kqp.cpu().numpy(), e_kqp, atol=2e-3, rtol=1e-3)


def test_selection_recall_full_size_rows():
    """Three rows of the 128K prefill (64 heads, 8 groups, d_idx 128), the
    configuration the measurement uses: block mass, KL and the full causal lse
    against the oracle, recall where the selections agree."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = wl.P128
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    pipeline.select(buf, inp["q_idx"], inp["k_idx"])
    rows = np.array([777, 65536, w.n_q - 1], np.int64)
    lse_full = torch.empty((len(rows), w.h_q), device="cuda")
    mass, rec, kpq, kqp = pipeline.selection_recall(buf, inp["q"], inp["k"], inp["q_idx"],
                                                    inp["k_idx"], torch.from_numpy(rows).cuda(),
                                                    lse_full=lse_full)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    b = np.zeros_like(rows)
    pos = w.q_pos0 + rows
    q_rows = _bits(inp["q"])[0, rows]
    qi_rows = _bits(inp["q_idx"])[0, rows]
    kb, vb, kib = _bits(inp["k"]), _bits(inp["v"]), _bits(inp["k_idx"])
    gpu_sel = buf.sel[0, :, torch.from_numpy(rows).cuda()].permute(1, 0, 2).cpu().numpy()
    g = [x.cpu().numpy() for x in (mass, rec, kpq, kqp, lse_full)]
    del inp, buf
    torch.cuda.empty_cache()
    pooled = oracle.index_pooled(qi_rows, pos, b, kib)
    sel = oracle.topk(pooled, pos)
    bad, ties, bad_tie, eval_sel = compare_sets(gpu_sel, sel, pooled, pos)
    assert bad == 0 and bad_tie == 0, (bad, ties, bad_tie)
    e_mass, e_rec, e_kpq, e_kqp = oracle.selection_recall(q_rows, qi_rows, pos, b, kb, kib,
                                                          eval_sel, w.scale, stride=g[0].shape[2])
    _, _, _, e_full = oracle.token_select_attention(q_rows, qi_rows, pos, b, kb, vb, kib, w.scale,
                                                    budget=1)
    np.testing.assert_allclose(g[0].astype(np.float64), e_mass, atol=5e-5, rtol=1e-4)
    np.testing.assert_allclose(g[1], e_rec, atol=2e-4)
    np.testing.assert_allclose(g[2], e_kpq, atol=2e-3, rtol=1e-3)
    np.testing.assert_allclose(g[3], e_kqp, atol=2e-3, rtol=1e-3)
    assert np.abs(g[4] - e_full).max() <= 1e-4
